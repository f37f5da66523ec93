// (a6) Block-sparse bidirectional attention -- the CUDA-core kernel, used for
// fp32 inputs (exact fp32 FMAs keep the 1e-5 tolerance, which TF32 tensor
// cores would not), and the split-KV combine shared with the tensor-core
// kernel.
//
// Focus-dLLM abstract / summary: decode-block queries attend bidirectionally
// to the selected (sink-aware) KV blocks and to the decode block; shallow
// layers attend densely.  Prefilling-dLLM abstract: the same over tokens
// gathered from non-contiguously cached chunks.
//
// Grid (split, b*H_kv), 256 threads.  A CTA walks its share of the (b, g)
// key tiles; each 64-row K/V tile is staged in shared memory as fp32 (K rows
// padded by one word so that lane t reading key t hits bank t); a warp owns 4
// query rows, computes two keys' logits per lane, and keeps an online
// softmax (running max, running sum, fp32 accumulator of d/32 columns per
// lane).  Partials (acc, m, l) go to the workspace; the combine kernel
// merges the splits with log-sum-exp weights and rounds O once.
#include "common.cuh"
#include "internal.h"
#include "tiles.cuh"
#include "launch.cuh"

namespace dl {

constexpr int kSimtRowsPerWarp = 4;
constexpr int kSimtRowsPerPass = 8 * kSimtRowsPerWarp;

template <int D>
__host__ __device__ constexpr size_t simt_smem_bytes() {
  return sizeof(float) * (kTile * (D + 1) + kTile * D + kSimtRowsPerPass * D) +
         sizeof(int) * kTile;
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
attn_simt_kernel(AttnArgs a, int n_split, int tps) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ float smem[];
  float* sK = smem;                              // [64][D+1]
  float* sV = sK + kTile * (D + 1);              // [64][D]
  float* sQ = sV + kTile * D;                    // [32][D]
  int* sOk = reinterpret_cast<int*>(sQ + kSimtRowsPerPass * D);
  const Shape& s = a.s;
  const int bg = blockIdx.y, sp = blockIdx.x;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const T* Q = reinterpret_cast<const T*>(a.Q);
  const T* Kp = reinterpret_cast<const T*>(a.Kp);
  const T* Vp = reinterpret_cast<const T*>(a.Vp);
  const T* Kd = reinterpret_cast<const T*>(a.Kd);
  const T* Vd = reinterpret_cast<const T*>(a.Vd);
  const int n_ctx = ctx_tile_count(a, bg);
  const int n_tiles = n_ctx + (s.L_q + kTile - 1) / kTile;
  const int t0 = sp * tps;
  const int t1 = min(t0 + tps, n_tiles);
  const int R = s.G * s.L_q;
  const float scale = (float)s.scale;
  Partials part = partials_of(a.ws, s, n_split);
  constexpr int CPL = D / 32;   // accumulator columns per lane
  constexpr int EPT = Vec16<T>::N;
  constexpr int VPR = D / EPT;  // 16-byte vectors per row

  for (int r0 = 0; r0 < R; r0 += kSimtRowsPerPass) {
    __syncthreads();
    for (int e = threadIdx.x; e < kSimtRowsPerPass * D; e += blockDim.x) {
      const int rr = e / D, c = e % D, r = r0 + rr;
      float v = 0.0f;
      if (r < R) {
        const int h = g * s.G + r / s.L_q, i = r % s.L_q;
        v = to_f32(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + c]);
      }
      sQ[rr * D + c] = v;
    }
    float m[kSimtRowsPerWarp], l[kSimtRowsPerWarp], acc[kSimtRowsPerWarp][CPL];
#pragma unroll
    for (int q = 0; q < kSimtRowsPerWarp; ++q) {
      m[q] = -INFINITY;
      l[q] = 0.0f;
#pragma unroll
      for (int c = 0; c < CPL; ++c) acc[q][c] = 0.0f;
    }
    for (int tile = t0; tile < t1; ++tile) {
      __syncthreads();
      const bool is_ctx = tile < n_ctx;
      if (threadIdx.x < kTile) {
        const int r = threadIdx.x;
        long long off = is_ctx ? ctx_row_offset(a, b, g, bg, tile, r)
                               : dec_row_offset(s, bg, (tile - n_ctx) * kTile + r);
        sOk[r] = off >= 0;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < kTile * VPR; e += blockDim.x) {
        const int r = e / VPR, c = (e % VPR) * EPT;
        float kv[EPT], vv[EPT];
        if (sOk[r]) {
          long long off = is_ctx ? ctx_row_offset(a, b, g, bg, tile, r)
                                 : dec_row_offset(s, bg, (tile - n_ctx) * kTile + r);
          Vec16<T>::load((is_ctx ? Kp : Kd) + off + c, kv);
          Vec16<T>::load((is_ctx ? Vp : Vd) + off + c, vv);
        } else {
#pragma unroll
          for (int x = 0; x < EPT; ++x) { kv[x] = 0.0f; vv[x] = 0.0f; }
        }
#pragma unroll
        for (int x = 0; x < EPT; ++x) {
          sK[r * (D + 1) + c + x] = kv[x];
          sV[r * D + c + x] = vv[x];
        }
      }
      __syncthreads();
      const bool ok0 = sOk[lane] != 0, ok1 = sOk[lane + 32] != 0;
#pragma unroll
      for (int q = 0; q < kSimtRowsPerWarp; ++q) {
        const int rr = warp * kSimtRowsPerWarp + q;
        if (r0 + rr >= R) break;
        const float* qr = sQ + rr * D;
        float s0 = 0.0f, s1 = 0.0f;
#pragma unroll 8
        for (int c = 0; c < D; ++c) {
          const float qc = qr[c];
          s0 = fmaf(qc, sK[lane * (D + 1) + c], s0);
          s1 = fmaf(qc, sK[(lane + 32) * (D + 1) + c], s1);
        }
        s0 = ok0 ? s0 * scale : -INFINITY;
        s1 = ok1 ? s1 * scale : -INFINITY;
        const float m_new = fmaxf(m[q], warp_max(fmaxf(s0, s1)));
        if (m_new == -INFINITY) continue;
        const float alpha = expf(m[q] - m_new);
        const float p0 = expf(s0 - m_new), p1 = expf(s1 - m_new);
        l[q] = l[q] * alpha + warp_sum(p0 + p1);
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[q][c] *= alpha;
        for (int t = 0; t < kTile; ++t) {
          const float pt = __shfl_sync(0xffffffffu, t < 32 ? p0 : p1, t & 31);
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[q][c] = fmaf(pt, sV[t * D + lane + 32 * c], acc[q][c]);
        }
        m[q] = m_new;
      }
    }
#pragma unroll
    for (int q = 0; q < kSimtRowsPerWarp; ++q) {
      const int r = r0 + warp * kSimtRowsPerWarp + q;
      if (r >= R) break;
      const size_t row = ((size_t)bg * n_split + sp) * R + r;
#pragma unroll
      for (int c = 0; c < CPL; ++c) part.o[row * D + lane + 32 * c] = acc[q][c];
      if (lane == 0) part.ml[row] = make_float2(m[q], l[q]);
    }
  }
}

// Merge the split partials of each (b, g, row): O = sum_s acc_s e^{m_s-M} / L,
// L = sum_s l_s e^{m_s-M}, lse = M + ln L.  One warp per row.
// Partials of (b, g) occupy slots [0, n_valid): all n_split slots for the
// CUDA-core kernel (P == 0); for the persistent tensor-core kernel (S tile
// slots per (b, g) split over P CTAs) the CTAs sharing the (b, g).
template <typename T, int D>
__global__ void __launch_bounds__(256)
attn_combine_kernel(Shape s, int n_split, const void* ws, T* __restrict__ O,
                    float* __restrict__ lse, int S, int P) {
  pdl_trigger();
  pdl_wait();
  const int R = s.G * s.L_q;
  const long long n_rows = (long long)s.batch * s.H_kv * R;
  const long long gw = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (gw >= n_rows) return;
  const int bg = (int)(gw / R), r = (int)(gw % R);
  Partials part = partials_of(const_cast<void*>(ws), s, n_split);
  int n_valid = n_split;
  if (P > 0) {
    const long long U = (long long)s.batch * s.H_kv * S;
    const long long base = (long long)bg * S;
    const long long c0 = ((base + 1) * P + U - 1) / U - 1;
    const long long c1 = ((base + S) * P + U - 1) / U - 1;
    n_valid = (int)(c1 - c0 + 1);
    n_valid = n_valid < n_split ? n_valid : n_split;
  }
  merge_row<T, D>(part, s, n_split, bg, r, n_valid, O, lse, lane);
}

size_t attn_workspace(const Shape& s) {
  const size_t n = (size_t)s.batch * s.H_kv * kMaxSplits * s.G * s.L_q;
  return round256(n * s.d * sizeof(float)) + round256(n * sizeof(float2));
}

int attn_splits(const Shape& s, int max_tiles) {
  const int bgs = s.batch * s.H_kv;
  int n = (2 * 148 + bgs - 1) / bgs;
  n = n < 1 ? 1 : n;
  n = n > kMaxSplits ? kMaxSplits : n;
  n = n > max_tiles ? max_tiles : n;
  return n < 1 ? 1 : n;
}

template <typename T, int D>
static cudaError_t run_combine(const AttnArgs& a, int n_split, cudaStream_t st, int S, int P) {
  const Shape& s = a.s;
  const long long rows = (long long)s.batch * s.H_kv * s.G * s.L_q;
  DL_LAUNCH(attn_combine_kernel<T, D>, (unsigned)((rows + 7) / 8), 256, 0, st, 
      s, n_split, a.ws, reinterpret_cast<T*>(a.O), a.lse, S, P);
  return cudaGetLastError();
}

cudaError_t launch_combine(const AttnArgs& a, int n_split, cudaStream_t st, int S = 0,
                           int P = 0) {
  if (a.s.dtype == 1)
    return a.s.d == 128 ? run_combine<float, 128>(a, n_split, st, S, P)
                        : run_combine<float, 64>(a, n_split, st, S, P);
  return a.s.d == 128 ? run_combine<__nv_bfloat16, 128>(a, n_split, st, S, P)
                      : run_combine<__nv_bfloat16, 64>(a, n_split, st, S, P);
}

template <typename T, int D>
static cudaError_t run_simt(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  const Shape& s = a.s;
  const int n_split = attn_splits(s, max_tiles);
  const int tps = (max_tiles + n_split - 1) / n_split;
  const size_t smem = simt_smem_bytes<D>();
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<T, D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(n_split, s.batch * s.H_kv);
  DL_LAUNCH(attn_simt_kernel<T, D>, grid, 256, smem, st, a, n_split, tps);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_combine(a, n_split, st);
}

static int max_tiles_of(const AttnArgs& a) {
  const Shape& s = a.s;
  const int n_blk = (s.L_ctx + s.page - 1) / s.page;
  int ctx = a.mode == kDense ? n_blk
          : a.mode == kBlocks ? a.max_idx : (a.max_idx + kTile - 1) / kTile;
  return ctx + (s.L_q + kTile - 1) / kTile;
}

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t st) {
  const int mt = max_tiles_of(a);
  if (a.s.dtype == 1) {
    return a.s.d == 128 ? run_simt<float, 128>(a, mt, st) : run_simt<float, 64>(a, mt, st);
  }
  return a.s.d == 128 ? run_simt<__nv_bfloat16, 128>(a, mt, st)
                      : run_simt<__nv_bfloat16, 64>(a, mt, st);
}

bool attn_tc_supported(const AttnArgs& a);
cudaError_t launch_attn_tc(const AttnArgs& a, int max_tiles, cudaStream_t st);

// bf16 block/dense attention runs on the tensor cores (attn_tc.cu); fp32
// inputs (exact FMAs for the 1e-5 bar), gathered tokens and query groups of
// more than 256 rows run on this kernel.
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  if (attn_tc_supported(a)) return launch_attn_tc(a, max_tiles_of(a), st);
  return launch_attn_simt(a, st);
}

}  // namespace dl
