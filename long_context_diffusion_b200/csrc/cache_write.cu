// Cache refresh with the block pooling fused into the write.
//
// Focus-dLLM (research.elamur.ai summary): the long context is held in a KV
// cache, and block selection reads one mean key per block.  When a decode
// block is finished its tokens join the cached context; this kernel writes
// them into the paged pools and, in the same pass, recomputes the pooled key
// of every block they touch, so the new keys are not read back a second time
// (the block's other rows are read from the pool).
//
// CTA (k, b, g): the k-th block touched by sequence b's positions
// start[b] .. start[b] + n_new - 1, KV head g.  Thread (row group, 16-byte
// column chunk): its rows of the block, new ones copied from K_new/V_new into
// the pools, old ones read from the K pool, summed in fp64; the row groups'
// sums are added in shared memory and the mean over the block's positions
// below L_ctx is rounded once to fp32 (and, when asked, also written as the
// integer digits of kdigits.cuh).  For bf16 keys the fp64 sum is exact,
// so the result equals dl_pool_keys bit for bit whatever the order; for fp32
// keys the fp64 sum is exact only while the 64 values' exponents are close,
// and the pooled key can then differ from dl_pool_keys' by one fp32 ulp.
#include "common.cuh"
#include "internal.h"
#include "kdigits.cuh"
#include "launch.cuh"

namespace dl {

constexpr int kCwThreads = 256;

template <typename T, int D>
__global__ void __launch_bounds__(kCwThreads)
cache_write_kernel(Shape s, const T* __restrict__ K_new, const T* __restrict__ V_new, int n_new,
                   const int32_t* __restrict__ start, const int32_t* __restrict__ page_table,
                   T* __restrict__ Kp, T* __restrict__ Vp, float* __restrict__ Kbar,
                   int8_t* __restrict__ Kdig, int32_t* __restrict__ Kexp, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPT = Vec16<T>::N;       // elements per 16-byte chunk
  constexpr int TPR = D / EPT;           // chunks per row
  constexpr int RG = kCwThreads / TPR;   // row groups
  constexpr int B = 64;                  // positions per block (= page)
  __shared__ double s_sum[RG][D];
  __shared__ float s_sq[RG][TPR];  // per row group and chunk: max sum of squares
  const int bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int tid = threadIdx.x, c = tid % TPR, rg = tid / TPR;
  const int st = start[b];
  if (st < 0 || (long long)st + n_new > s.L_ctx) {  // 64-bit: start comes from device memory
    if (blockIdx.x == 0 && tid == 0) flag_error(err, ERR_BAD_INDEX);
    return;
  }
  const int j = st / B + blockIdx.x;
  if (j > (st + n_new - 1) / B) return;
  const int slot = page_table[(size_t)b * s.n_pages + j];
  if (slot < 0 || slot >= s.n_slots) {
    if (tid == 0) flag_error(err, ERR_BAD_INDEX);
    return;
  }
  const size_t page_row0 = ((size_t)slot * s.H_kv + g) * B;
  double acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
  float sq_max = 0.0f;
#pragma unroll
  for (int r = rg; r < B; r += RG) {
    const int p = j * B + r;
    if (p >= s.L_ctx) continue;  // past the context: neither written nor pooled
    T* krow = Kp + (page_row0 + r) * D + c * EPT;
    uint4 raw;
    if (p >= st && p < st + n_new) {
      const size_t src = ((size_t)bg * n_new + (p - st)) * D + c * EPT;
      raw = __ldg(reinterpret_cast<const uint4*>(K_new + src));
      *reinterpret_cast<uint4*>(krow) = raw;
      *reinterpret_cast<uint4*>(Vp + (page_row0 + r) * D + c * EPT) =
          __ldg(reinterpret_cast<const uint4*>(V_new + src));
    } else {
      raw = *reinterpret_cast<const uint4*>(krow);
    }
    float v[EPT];
    if constexpr (sizeof(T) == 2) {
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
      for (int q = 0; q < EPT / 2; ++q) {
        const float2 f = __bfloat1622float2(h2[q]);
        v[2 * q] = f.x;
        v[2 * q + 1] = f.y;
      }
    } else {
      const float* f = reinterpret_cast<const float*>(&raw);
#pragma unroll
      for (int q = 0; q < EPT; ++q) v[q] = f[q];
    }
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[e] += (double)v[e];
    float q = 0.0f;
#pragma unroll
    for (int e = 0; e < EPT; ++e) q = __fmaf_rn(v[e], v[e], q);
    sq_max = fmaxf(sq_max, q);
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) s_sum[rg][c * EPT + e] = acc[e];
  s_sq[rg][c] = sq_max;
  __syncthreads();
  const int n_blk = (s.L_ctx + B - 1) / B;
  float mean = 0.0f;
  if (tid < D) {
    double sum = 0.0;
    for (int q = 0; q < RG; ++q) sum += s_sum[q][tid];
    const int n = min(B, s.L_ctx - j * B);
    mean = __double2float_rn(sum / (double)n);
    Kbar[((size_t)bg * n_blk + j) * D + tid] = mean;
  }
  if (Kdig == nullptr) return;  // uniform over the grid
  // the block's pooled key as integer digits (kdigits.cuh): row exponent and
  // inexact count over the D threads of the first D / 32 warps
  __shared__ int s_e[kCwThreads / 32], s_n[kCwThreads / 32];
  const int warp = tid >> 5, lane = tid & 31;
  int E = tid < D ? exp_field_f32(mean) : 1;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) E = max(E, __shfl_xor_sync(0xffffffffu, E, o));
  if (lane == 0) s_e[warp] = E;
  __syncthreads();
  E = 1;
  for (int w = 0; w < D / 32; ++w) E = max(E, s_e[w]);
  int dg[kKeyDigits];
  int inexact = (tid < D && key_digits(mean, E, dg)) ? 1 : 0;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) inexact += __shfl_xor_sync(0xffffffffu, inexact, o);
  if (lane == 0) s_n[warp] = inexact;
  __syncthreads();
  if (tid < D) {
#pragma unroll
    for (int t = 0; t < kKeyDigits; ++t)
      Kdig[(((size_t)bg * kKeyDigits + t) * n_blk + j) * D + tid] = (int8_t)dg[t];
  }
  if (tid == 0) {
    int n = 0;
    for (int w = 0; w < D / 32; ++w) n += s_n[w];
    // norm bound: per chunk the max over the row groups, added in chunk order
    float sq_sum = 0.0f;
    for (int q = 0; q < TPR; ++q) {
      float m = 0.0f;
      for (int r = 0; r < RG; ++r) m = fmaxf(m, s_sq[r][q]);
      sq_sum += m;
    }
    Kexp[(size_t)bg * n_blk + j] = E | (n << 8) | key_norm_field(sq_sum);
  }
}

cudaError_t launch_cache_write(const Shape& s, const void* K_new, const void* V_new, int n_new,
                               const int32_t* start, const int32_t* page_table, void* Kp,
                               void* Vp, float* Kbar, int8_t* Kdig, int32_t* Kexp, unsigned* err,
                               cudaStream_t st) {
  dim3 grid((n_new + 63) / 64 + 1, s.batch * s.H_kv);
#define DL_CACHE_WRITE(T, D_)                                                                  \
  DL_LAUNCH(cache_write_kernel<T, D_>, grid, kCwThreads, 0, st, s,                             \
            reinterpret_cast<const T*>(K_new), reinterpret_cast<const T*>(V_new), n_new,      \
            start, page_table, reinterpret_cast<T*>(Kp), reinterpret_cast<T*>(Vp), Kbar, Kdig,   \
            Kexp, err)
  if (s.dtype == 0) {
    if (s.d == 128) DL_CACHE_WRITE(__nv_bfloat16, 128); else DL_CACHE_WRITE(__nv_bfloat16, 64);
  } else {
    if (s.d == 128) DL_CACHE_WRITE(float, 128); else DL_CACHE_WRITE(float, 64);
  }
#undef DL_CACHE_WRITE
  return cudaGetLastError();
}

}  // namespace dl
