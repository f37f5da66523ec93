// (a3) Block scores: predicted query rows x mean-pooled keys, a softmax over
// blocks per row, summed over the rows (and over the query heads of a KV
// group).
//
// Focus-dLLM (research.elamur.ai summary): predicted queries select the most
// relevant KV blocks.  The score decides which block indices are kept, so it
// is computed in fp64: bf16 (or fp32) query x fp32 pooled-key products are
// exact in fp64 and the remaining rounding (~1e-16 relative) sits far below
// the spacing of neighbouring scores, so the kept set equals the one an
// exact computation gives.
//
// Two kernels.  (1) logits: grid (64-unit tiles, b*H_kv); each thread owns
// one pooled key and 8 query rows (staged in shared memory as fp64) and
// writes scale * q . Kbar in fp64 to the workspace.  (2) softmax: one CTA per (b, g); a warp per row takes its max
// and sum of exponentials by shuffles and writes the probabilities in place;
// then one thread per unit sums its column over the rows in row order.
#include "common.cuh"
#include "internal.h"

namespace dl {

constexpr int kUT = 64;   // units per logits CTA (one per thread column)
constexpr int kRT = 32;   // query rows staged per pass (8 per thread)

// Thread (u, rg): unit u0 + (tid % 64), rows rg*8 .. rg*8+7 of the pass.
// Query rows are staged once as fp64 (exact) and read as broadcasts; the
// pooled key is read 16 bytes at a time and converted once per element; the
// 8 products per key element accumulate with fp64 FMAs.
template <typename T, int D>
__global__ void __launch_bounds__(256)
scores_logits_kernel(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                     const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar,
                     Shape s, int n_units, double* __restrict__ S, unsigned* err) {
  __shared__ __align__(16) double sQ[kRT][D];
  const int bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int u = blockIdx.x * kUT + (threadIdx.x % kUT);
  const int rg = threadIdx.x / kUT;  // 0..3
  const int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  const int R = nq * s.G;
  const int R_max = s.L_q * s.G;
  const bool u_ok = u < n_units;
  const float* kb = Kbar + (((size_t)b * s.H_kv + g) * n_units + (u_ok ? u : 0)) * D;
  for (int r0 = 0; r0 < R; r0 += kRT) {
    __syncthreads();
    for (int e = threadIdx.x; e < kRT * D; e += blockDim.x) {
      const int rr = e / D, c = e % D;
      const int r = r0 + rr;
      double v = 0.0;
      if (r < R) {
        const int h = g * s.G + r / nq;
        const int i = q_idx ? q_idx[(size_t)b * s.L_q + (r % nq)] : (r % nq);
        if (i >= 0 && i < s.L_q)
          v = (double)to_f32(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + c]);
        else if (c == 0)
          flag_error(err, ERR_BAD_INDEX);
      }
      sQ[rr][c] = v;
    }
    __syncthreads();
    if (!u_ok || r0 + rg * 8 >= R) continue;
    double acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0;
#pragma unroll 2
    for (int c0 = 0; c0 < D; c0 += 4) {
      const float4 kv = __ldg(reinterpret_cast<const float4*>(kb + c0));
      const double k0 = kv.x, k1 = kv.y, k2 = kv.z, k3 = kv.w;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const double2 qa = *reinterpret_cast<const double2*>(&sQ[rg * 8 + k][c0]);
        const double2 qb = *reinterpret_cast<const double2*>(&sQ[rg * 8 + k][c0 + 2]);
        acc[k] = fma(qa.x, k0, acc[k]);
        acc[k] = fma(qa.y, k1, acc[k]);
        acc[k] = fma(qb.x, k2, acc[k]);
        acc[k] = fma(qb.y, k3, acc[k]);
      }
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = r0 + rg * 8 + k;
      if (r < R) S[((size_t)bg * R_max + r) * n_units + u] = acc[k] * s.scale;
    }
  }
}

__global__ void __launch_bounds__(512)
scores_softmax_kernel(const int32_t* __restrict__ q_idx, const int32_t* __restrict__ q_cnt,
                      Shape s, int n_units, double* __restrict__ S, double* __restrict__ score) {
  const int bg = blockIdx.x;
  const int b = bg / s.H_kv;
  const int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  const int R = nq * s.G;
  const int R_max = s.L_q * s.G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  double* Sb = S + (size_t)bg * R_max * n_units;
  for (int r = warp; r < R; r += nw) {
    double* row = Sb + (size_t)r * n_units;
    double m = -INFINITY;
    for (int u = lane; u < n_units; u += 32) m = fmax(m, row[u]);
    m = warp_max_d(m);
    double z = 0.0;
    for (int u = lane; u < n_units; u += 32) z += exp(row[u] - m);
    z = warp_sum_d(z);
    for (int u = lane; u < n_units; u += 32) row[u] = exp(row[u] - m) / z;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < n_units; u += blockDim.x) {
    double acc = 0.0;
    for (int r = 0; r < R; ++r) acc += Sb[(size_t)r * n_units + u];
    score[(size_t)bg * n_units + u] = acc;
  }
}

size_t scores_workspace(const Shape& s, int n_units) {
  return round256((size_t)s.batch * s.H_kv * s.G * s.L_q * (size_t)n_units * sizeof(double));
}

cudaError_t launch_scores(const Shape& s, const void* Q, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, int n_units, double* score,
                          void* ws, unsigned* err, cudaStream_t st) {
  double* S = reinterpret_cast<double*>(ws);
  dim3 grid((n_units + kUT - 1) / kUT, s.batch * s.H_kv);
  if (s.dtype == 0) {
    auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
    if (s.d == 128)
      scores_logits_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(q, q_idx, q_cnt, Kbar, s,
                                                                     n_units, S, err);
    else
      scores_logits_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(q, q_idx, q_cnt, Kbar, s,
                                                                    n_units, S, err);
  } else {
    auto* q = reinterpret_cast<const float*>(Q);
    if (s.d == 128)
      scores_logits_kernel<float, 128><<<grid, 256, 0, st>>>(q, q_idx, q_cnt, Kbar, s, n_units, S, err);
    else
      scores_logits_kernel<float, 64><<<grid, 256, 0, st>>>(q, q_idx, q_cnt, Kbar, s, n_units, S, err);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  scores_softmax_kernel<<<s.batch * s.H_kv, 512, 0, st>>>(q_idx, q_cnt, s, n_units, S, score);
  return cudaGetLastError();
}

}  // namespace dl
