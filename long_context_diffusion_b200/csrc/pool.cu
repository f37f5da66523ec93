// (a2) Mean-pooled keys, one per key block (or per chunk).
//
// Focus-dLLM (research.elamur.ai summary): the predicted queries select the
// most relevant key-value pairs; selection works on one mean key per block.
// Prefilling-dLLM (abstract): chunks are ranked for relevance; a chunk's key
// is the mean of its content tokens (the BOS anchor is left out).
//
// HBM-bound: every K row of the unit is read once with 16-byte coalesced
// loads.  Sums are taken in fp64, where the sum of <= 2^16 bf16 (or fp32)
// values of a block is exact, so the result does not depend on the order of
// the additions; it is divided by the token count and rounded once to fp32.
#include "common.cuh"
#include "internal.h"

namespace dl {

template <typename T, int D>
__global__ void __launch_bounds__(256)
pool_kernel(const T* __restrict__ Kp, const int32_t* __restrict__ page_table, Shape s,
            int n_units, int stride, int offset, int len, float* __restrict__ Kbar,
            unsigned* err) {
  constexpr int EPT = Vec16<T>::N;          // elements per 16-byte load
  constexpr int TPR = D / EPT;              // threads per K row
  constexpr int RPI = 256 / TPR;            // rows per iteration
  __shared__ double s_acc[RPI][D];
  const int u = blockIdx.x;
  const int bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int c = threadIdx.x % TPR, r0 = threadIdx.x / TPR;
  const long long lo = (long long)u * stride + offset;
  const long long hi = min(lo + (long long)len, (long long)s.L_ctx);
  double acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
  for (long long t = lo + r0; t < hi; t += RPI) {
    const int lp = (int)(t / s.page);
    const int row = (int)(t % s.page);
    int slot = -1;
    if (lp < s.n_pages) slot = page_table[(size_t)b * s.n_pages + lp];
    if (slot < 0 || slot >= s.n_slots) {
      flag_error(err, ERR_BAD_INDEX);
      continue;
    }
    const T* src = Kp + (((size_t)slot * s.H_kv + g) * s.page + row) * D + c * EPT;
    float v[EPT];
    Vec16<T>::load(src, v);
#pragma unroll
    for (int e = 0; e < EPT; ++e) acc[e] += (double)v[e];
  }
#pragma unroll
  for (int e = 0; e < EPT; ++e) s_acc[r0][c * EPT + e] = acc[e];
  __syncthreads();
  const long long n = hi > lo ? hi - lo : 0;
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    double sum = 0.0;
    for (int r = 0; r < RPI; ++r) sum += s_acc[r][j];
    const float mean = n > 0 ? __double2float_rn(sum / (double)n) : 0.0f;
    Kbar[(((size_t)b * s.H_kv + g) * n_units + u) * D + j] = mean;
  }
}

cudaError_t launch_pool(const Shape& s, const void* Kp, const int32_t* page_table, int n_units,
                        int stride, int offset, int len, float* Kbar, unsigned* err,
                        cudaStream_t st) {
  dim3 grid(n_units, s.batch * s.H_kv);
  if (s.dtype == 0) {
    auto* k = reinterpret_cast<const __nv_bfloat16*>(Kp);
    if (s.d == 128)
      pool_kernel<__nv_bfloat16, 128><<<grid, 256, 0, st>>>(k, page_table, s, n_units, stride,
                                                            offset, len, Kbar, err);
    else
      pool_kernel<__nv_bfloat16, 64><<<grid, 256, 0, st>>>(k, page_table, s, n_units, stride,
                                                           offset, len, Kbar, err);
  } else {
    auto* k = reinterpret_cast<const float*>(Kp);
    if (s.d == 128)
      pool_kernel<float, 128><<<grid, 256, 0, st>>>(k, page_table, s, n_units, stride, offset,
                                                    len, Kbar, err);
    else
      pool_kernel<float, 64><<<grid, 256, 0, st>>>(k, page_table, s, n_units, stride, offset,
                                                   len, Kbar, err);
  }
  return cudaGetLastError();
}

}  // namespace dl
