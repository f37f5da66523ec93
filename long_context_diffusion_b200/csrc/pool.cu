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
// divided by the token count and rounded once to fp32.  Optionally the same
// pooled keys are also written as integer digits with one exponent per unit
// (kdigits.cuh), the form the int8 tensor-core block scores read.
#include "common.cuh"
#include "internal.h"
#include "kdigits.cuh"
#include "launch.cuh"

namespace dl {

// Thread (u, c): unit u of the CTA's run, 16-byte column chunk c.  It walks
// the unit's rows page by page with 8 independent 16-byte loads in flight and
// accumulates in fp64 (exact for bf16 and for fp32 sums of <= 2^16 terms of
// moderate range), so no cross-thread reduction is needed.  With Kdig/Kexp
// the unit's pooled key is also written as integer digits (kdigits.cuh): the
// TPR threads of a unit (consecutive lanes of one warp) take the row
// exponent and the inexact count by shuffles.
template <typename T, int D>
__global__ void __launch_bounds__(256)
pool_kernel(const T* __restrict__ Kp, const int32_t* __restrict__ page_table, Shape s,
            int n_units, int stride, int offset, int len, float* __restrict__ Kbar,
            int8_t* __restrict__ Kdig, int32_t* __restrict__ Kexp, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  constexpr int EPT = Vec16<T>::N;          // elements per 16-byte load
  constexpr int TPR = D / EPT;              // threads per K row
  constexpr int UPC = 256 / TPR;            // units per CTA
  const int u = blockIdx.x * UPC + threadIdx.x / TPR;
  const int c = threadIdx.x % TPR;
  const int bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const bool active = u < n_units;
  const long long lo = (long long)u * stride + offset;
  const long long hi = active ? min(lo + (long long)len, (long long)s.L_ctx) : lo;
  double acc[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) acc[e] = 0.0;
  float sq_max = 0.0f;  // max over the rows of this chunk's sum of squares
  const bool norms = Kdig != nullptr;
  auto sq = [](const float(&v)[EPT]) {
    float q = 0.0f;
#pragma unroll
    for (int e = 0; e < EPT; ++e) q = __fmaf_rn(v[e], v[e], q);
    return q;
  };
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
      if (norms) {
#pragma unroll
        for (int q = 0; q < 8; ++q) sq_max = fmaxf(sq_max, sq(v[q]));
      }
    }
    for (; r < rows; ++r) {
      float v[EPT];
      Vec16<T>::load(src + (size_t)r * D, v);
#pragma unroll
      for (int e = 0; e < EPT; ++e) acc[e] += (double)v[e];
      if (norms) sq_max = fmaxf(sq_max, sq(v));
    }
  }
  const long long n = hi > lo ? hi - lo : 0;
  float mean[EPT];
#pragma unroll
  for (int e = 0; e < EPT; ++e) mean[e] = n > 0 ? __double2float_rn(acc[e] / (double)n) : 0.0f;
  if (active) {
    float* dst = Kbar + ((size_t)bg * n_units + u) * D + c * EPT;
#pragma unroll
    for (int e = 0; e < EPT; ++e) dst[e] = mean[e];
  }
  if (Kdig == nullptr) return;  // uniform over the grid
  int E = 1;
#pragma unroll
  for (int e = 0; e < EPT; ++e) E = max(E, exp_field_f32(mean[e]));
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) E = max(E, __shfl_xor_sync(0xffffffffu, E, o));
  int dg[EPT][kKeyDigits];
  int inexact = 0;
#pragma unroll
  for (int e = 0; e < EPT; ++e) inexact += key_digits(mean[e], E, dg[e]) ? 1 : 0;
#pragma unroll
  for (int o = 1; o < TPR; o <<= 1) inexact += __shfl_xor_sync(0xffffffffu, inexact, o);
  // norm bound: the chunks' maxima added in chunk order (as dl_cache_write)
  const int lane0 = (threadIdx.x & 31) & ~(TPR - 1);
  float sq_sum = 0.0f;
#pragma unroll
  for (int q = 0; q < TPR; ++q) sq_sum += __shfl_sync(0xffffffffu, sq_max, lane0 + q);
  if (!active) return;
#pragma unroll
  for (int t = 0; t < kKeyDigits; ++t) {
    int8_t* plane = Kdig + (((size_t)bg * kKeyDigits + t) * n_units + u) * D + c * EPT;
    if constexpr (EPT == 8) {
      *reinterpret_cast<uint2*>(plane) =
          make_uint2(pack4_i8(dg[0][t], dg[1][t], dg[2][t], dg[3][t]),
                     pack4_i8(dg[4][t], dg[5][t], dg[6][t], dg[7][t]));
    } else {
      *reinterpret_cast<uint32_t*>(plane) = pack4_i8(dg[0][t], dg[1][t], dg[2][t], dg[3][t]);
    }
  }
  if (c == 0) Kexp[(size_t)bg * n_units + u] = E | (inexact << 8) | key_norm_field(sq_sum);
}

cudaError_t launch_pool(const Shape& s, const void* Kp, const int32_t* page_table, int n_units,
                        int stride, int offset, int len, float* Kbar, int8_t* Kdig,
                        int32_t* Kexp, unsigned* err, cudaStream_t st) {
  const int upc = 256 / (s.d / (s.dtype == 0 ? 8 : 4));
  dim3 grid((n_units + upc - 1) / upc, s.batch * s.H_kv);
#define DL_POOL(T, D_)                                                                         \
  DL_LAUNCH(pool_kernel<T, D_>, grid, 256, 0, st, reinterpret_cast<const T*>(Kp), page_table, s, \
            n_units, stride, offset, len, Kbar, Kdig, Kexp, err)
  if (s.dtype == 0) {
    if (s.d == 128) DL_POOL(__nv_bfloat16, 128); else DL_POOL(__nv_bfloat16, 64);
  } else {
    if (s.d == 128) DL_POOL(float, 128); else DL_POOL(float, 64);
  }
#undef DL_POOL
  return cudaGetLastError();
}

}  // namespace dl
