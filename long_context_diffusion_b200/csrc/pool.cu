// (a2) Mean-pooled keys, one per key block (or per chunk).
//
// Focus-dLLM (research.elamur.ai summary): the predicted queries select the
// most relevant key-value pairs; selection works on one mean key per block.
// Prefilling-dLLM (abstract): chunks are ranked for relevance; a chunk's key
// is the mean of its content tokens (the BOS anchor is left out).
//
// HBM-bound: every K row of the unit is read once with 16-byte loads.  Sums
// are taken in fp64, where the sum of <= 2^16 bf16 values of a block is
// exact, so the result does not depend on the order of the additions; it is
// divided by the token count and rounded once to fp32.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace dl {

// Thread (u, c): unit u of the CTA's run, 16-byte column chunk c.  It walks
// the unit's rows page by page with 8 independent 16-byte loads in flight and
// accumulates in fp64 (exact for bf16 and for fp32 sums of <= 2^16 terms of
// moderate range), so no cross-thread reduction is needed.
template <typename T, int D>
__global__ void __launch_bounds__(256)
pool_kernel(const T* __restrict__ Kp, const int32_t* __restrict__ page_table, Shape s,
            int n_units, int stride, int offset, int len, float* __restrict__ Kbar,
            unsigned* err) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPT = Vec16<T>::N;          // elements per 16-byte load
  constexpr int TPR = D / EPT;              // threads per K row
  constexpr int UPC = 256 / TPR;            // units per CTA
  const int u = blockIdx.x * UPC + threadIdx.x / TPR;
  const int c = threadIdx.x % TPR;
  const int bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  if (u >= n_units) return;
  const long long lo = (long long)u * stride + offset;
  const long long hi = min(lo + (long long)len, (long long)s.L_ctx);
  double acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
  for (long long t = lo; t < hi;) {
    const int lp = (int)(t / s.page);
    const int row0 = (int)(t % s.page);
    const int rows = (int)min((long long)(s.page - row0), hi - t);
    const int slot = lp < s.n_pages ? page_table[(size_t)b * s.n_pages + lp] : -1;
    t += rows;
    if (slot < 0 || slot >= s.n_slots) {
      flag_error(err, ERR_BAD_INDEX);
      continue;
    }
    const T* src = Kp + (((size_t)slot * s.H_kv + g) * s.page + row0) * D + c * EPT;
    int r = 0;
    for (; r + 8 <= rows; r += 8) {
      float v[8][EPT];
#pragma unroll
      for (int q = 0; q < 8; ++q) Vec16<T>::load(src + (size_t)(r + q) * D, v[q]);
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int e = 0; e < EPT; ++e) acc[e] += (double)v[q][e];
    }
    for (; r < rows; ++r) {
      float v[EPT];
      Vec16<T>::load(src + (size_t)r * D, v);
#pragma unroll
      for (int e = 0; e < EPT; ++e) acc[e] += (double)v[e];
    }
  }
  const long long n = hi > lo ? hi - lo : 0;
  float* dst = Kbar + ((size_t)bg * n_units + u) * D + c * EPT;
#pragma unroll
  for (int e = 0; e < EPT; ++e) dst[e] = n > 0 ? __double2float_rn(acc[e] / (double)n) : 0.0f;
}

cudaError_t launch_pool(const Shape& s, const void* Kp, const int32_t* page_table, int n_units,
                        int stride, int offset, int len, float* Kbar, unsigned* err,
                        cudaStream_t st) {
  const int upc = 256 / (s.d / (s.dtype == 0 ? 8 : 4));
  dim3 grid((n_units + upc - 1) / upc, s.batch * s.H_kv);
  if (s.dtype == 0) {
    auto* k = reinterpret_cast<const __nv_bfloat16*>(Kp);
    if (s.d == 128)
      DL_LAUNCH(pool_kernel<__nv_bfloat16, 128>, grid, 256, 0, st, k, page_table, s, n_units, stride,
                                                            offset, len, Kbar, err);
    else
      DL_LAUNCH(pool_kernel<__nv_bfloat16, 64>, grid, 256, 0, st, k, page_table, s, n_units, stride,
                                                           offset, len, Kbar, err);
  } else {
    auto* k = reinterpret_cast<const float*>(Kp);
    if (s.d == 128)
      DL_LAUNCH(pool_kernel<float, 128>, grid, 256, 0, st, k, page_table, s, n_units, stride, offset,
                                                    len, Kbar, err);
    else
      DL_LAUNCH(pool_kernel<float, 64>, grid, 256, 0, st, k, page_table, s, n_units, stride, offset,
                                                   len, Kbar, err);
  }
  return cudaGetLastError();
}

}  // namespace dl
