// (a3 + a5) Block scores and selection in one kernel for groups of many
// query rows over few units: one CTA per (b, g).  The chunked prefix is the
// case it serves: every decode row of a head (64) against 32 chunk keys,
// top-8 chunks (Prefilling-dLLM abstract: top-K chunks by relevance).
//
// Same results as block_select.cu / scores.cu + select.cu:
//   l[r][u] = scale * q_r . Kbar_u,   score[u] = sum_r softmax_u(l[r][.]),
//   the sink units kept, then the topK other units of largest score (ties
//   to the lower index), ascending.
//
// With at most 128 units and R * n_units <= 8192 every logit of the (b, g)
// fits in shared memory, so one CTA does it all in fp64 on the CUDA cores:
//   stage   the group's query rows (gathered by q_idx) and its pooled keys by
//           cp.async;
//   dot     warp = (4 rows, 32 units), lane = unit: per 4 dimensions one
//           float4 of the key and one load of each row (the same address for
//           the whole warp); 16 fp64 FMA chains per lane (row x dimension mod
//           4), added in a fixed order (so equal keys give equal logits);
//   softmax warp per row: max, e^(l - max) in fp64, sum, divide;
//   scores  thread per unit sums its column in row order;
//   select  the bitonic sort and ascending write of the fused kernels.
// fp32 query values and fp32 pooled keys are exact in fp64 and their
// products too, so the logits carry only the rounding of the sums.
#include "block_select_common.cuh"
#include "launch.cuh"

namespace dl {

namespace bsw {
constexpr int kThreads = bs::kThreads;  // 512: the selection keeps one unit per thread
constexpr int kWarps = kThreads / 32;
constexpr int kMaxUnits = 128;
constexpr int kMaxRows = 256;
constexpr int kMaxCells = 8192;  // rows x units held as fp64 logits

template <typename T, int D>
struct Layout {
  static constexpr int KP = D + 4;  // pooled-key pitch in floats: rows 16 bytes apart mod 128
  __host__ __device__ static int rows_cap(int R) { return (R + 3) & ~3; }
  __host__ __device__ static int units_cap(int U) { return (U + 31) & ~31; }
  __host__ __device__ static size_t q_bytes(int R) { return (size_t)rows_cap(R) * D * sizeof(T); }
  __host__ __device__ static size_t k_bytes(int U) { return (size_t)units_cap(U) * KP * 4; }
  __host__ __device__ static size_t bytes(int R, int U) {
    return q_bytes(R) + k_bytes(U) + (size_t)rows_cap(R) * units_cap(U) * 8;
  }
};
}  // namespace bsw

template <typename T>
__device__ __forceinline__ void load4(const T* p, double (&v)[4]);
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, double (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <>
__device__ __forceinline__ void load4<float>(const float* p, double (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

template <typename T, int D>
__global__ void __launch_bounds__(bsw::kThreads, 1)
block_select_wide_kernel(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                         const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar,
                         Shape s, int n_units, int max_rows, double* __restrict__ score,
                         int unit_size, int topK, const int32_t* __restrict__ sink_pos,
                         int n_sinks, int32_t* __restrict__ blk_idx,
                         int32_t* __restrict__ blk_cnt, int max_sel, unsigned* err) {
  using namespace bsw;
  using L = Layout<T, D>;
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_b[];
  __shared__ BsSelScratch s_sel;

  const int bg = blockIdx.x;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = n_units, Uc = L::units_cap(U);

  // query rows: every predicted position of every query head of the group
  int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  if (nq * s.G > max_rows) {  // more rows than the caller's bound: reported, rows cut
    if (tid == 0) flag_error(err, ERR_BAD_INDEX);
    nq = max_rows / s.G;
  }
  const int R = nq * s.G;
  T* sQ = reinterpret_cast<T*>(smem_b);                                   // [Rc][D]
  float* sK = reinterpret_cast<float*>(smem_b + L::q_bytes(max_rows));    // [Uc][KP]
  double* sL = reinterpret_cast<double*>(smem_b + L::q_bytes(max_rows) + L::k_bytes(U));  // [Rc][Uc]

  constexpr int QCH = D * (int)sizeof(T) / 16;  // 16-byte chunks per query row
  for (int c = tid; c < L::rows_cap(R) * QCH; c += kThreads) {
    const int r = c / QCH, ch = c % QCH;
    const T* src = Q;
    bool ok = false;
    if (r < R) {
      const int h = g * s.G + r / nq;
      const int i = q_idx ? q_idx[(size_t)b * s.L_q + (r % nq)] : (r % nq);
      if (i >= 0 && i < s.L_q) {
        src = Q + (((size_t)b * s.H + h) * s.L_q + i) * D + ch * (16 / sizeof(T));
        ok = true;
      } else if (ch == 0) {
        flag_error(err, ERR_BAD_INDEX);
      }
    }
    cp_async16(sQ + (size_t)r * D + ch * (16 / sizeof(T)), src, ok);
  }
  constexpr int KCH = D / 4;  // 16-byte chunks per pooled key
  const float* kb = Kbar + (size_t)bg * U * D;
  for (int c = tid; c < Uc * KCH; c += kThreads) {
    const int u = c / KCH, ch = c % KCH;
    const bool ok = u < U;
    cp_async16(sK + u * L::KP + ch * 4, ok ? kb + (size_t)u * D + ch * 4 : Kbar, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // ---- logits: work item = (4 rows, 32 units); lane = unit
  const double sc = s.scale;
  const int n_rg = (R + 3) >> 2, n_ug = Uc >> 5;
  for (int it = warp; it < n_rg * n_ug; it += kWarps) {
    const int r0 = (it / n_ug) * 4, u = (it % n_ug) * 32 + lane;
    const float* kr = sK + u * L::KP;
    // 16 independent chains: row i, dimension phase c (k = c mod 4), so the
    // FMA latency is hidden; the phases are added in a fixed order
    double acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[i][c] = 0.0;
#pragma unroll 4
    for (int k = 0; k < D; k += 4) {
      const float4 kv = *reinterpret_cast<const float4*>(kr + k);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        double q[4];
        load4<T>(sQ + (size_t)(r0 + i) * D + k, q);
        acc[i][0] = fma(q[0], (double)kv.x, acc[i][0]);
        acc[i][1] = fma(q[1], (double)kv.y, acc[i][1]);
        acc[i][2] = fma(q[2], (double)kv.z, acc[i][2]);
        acc[i][3] = fma(q[3], (double)kv.w, acc[i][3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      sL[(size_t)(r0 + i) * Uc + u] = ((acc[i][0] + acc[i][1]) + (acc[i][2] + acc[i][3])) * sc;
  }
  __syncthreads();

  // ---- softmax over the units of each row (padding units excluded)
  for (int r = warp; r < R; r += kWarps) {
    double* lr = sL + (size_t)r * Uc;
    double m = -INFINITY;
    for (int u = lane; u < U; u += 32) m = fmax(m, lr[u]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    double z = 0.0;
    for (int u = lane; u < U; u += 32) {
      const double e = exp(lr[u] - m);
      lr[u] = e;
      z += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const double iz = 1.0 / z;
    for (int u = lane; u < U; u += 32) lr[u] *= iz;
  }
  __syncthreads();

  // ---- column sums in row order, then the selection of the fused kernels
  double my = 0.0;
  if (tid < U) {
    for (int r = 0; r < R; ++r) my += sL[(size_t)r * Uc + tid];
    score[(size_t)bg * U + tid] = my;
  }
  const BsSorted srt = bs_sort(my, U, b, unit_size, sink_pos, n_sinks, s_sel, err);
  bs_write(srt, U, topK, bg, blk_idx, blk_cnt, max_sel, s_sel);
}

bool block_select_wide_supported(const Shape& s, int rows, int n_units) {
  if (n_units < 1 || n_units > bsw::kMaxUnits || rows > bsw::kMaxRows) return false;
  if ((size_t)bsw::Layout<float, 128>::rows_cap(rows) * bsw::Layout<float, 128>::units_cap(n_units) >
      (size_t)bsw::kMaxCells)
    return false;
  return s.d == 64 || s.d == 128;
}

cudaError_t launch_block_select_wide(const Shape& s, const void* Q, const int32_t* q_idx,
                                     const int32_t* q_cnt, const float* Kbar, int n_units,
                                     double* score, int unit_size, int topK,
                                     const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                                     int32_t* blk_cnt, int max_sel, int rows, unsigned* err,
                                     cudaStream_t st) {
  cudaError_t e;
#define DL_BSW(T, D_)                                                                           \
  {                                                                                            \
    auto k = block_select_wide_kernel<T, D_>;                                                  \
    const size_t smem = bsw::Layout<T, D_>::bytes(rows, n_units);                              \
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != \
        cudaSuccess)                                                                           \
      return e;                                                                                \
    DL_LAUNCH(k, s.batch * s.H_kv, bsw::kThreads, smem, st, reinterpret_cast<const T*>(Q), q_idx, \
              q_cnt, Kbar, s, n_units, rows, score, unit_size, topK, sink_pos, n_sinks, blk_idx, \
              blk_cnt, max_sel, err);                                                          \
  }
  if (s.dtype == 0) {
    if (s.d == 128) DL_BSW(__nv_bfloat16, 128) else DL_BSW(__nv_bfloat16, 64)
  } else {
    if (s.d == 128) DL_BSW(float, 128) else DL_BSW(float, 64)
  }
#undef DL_BSW
  return cudaGetLastError();
}

}  // namespace dl
