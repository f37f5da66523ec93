// Pooled keys and query rows as base-128 integer digits, for block scores
// taken exactly on the int8 tensor cores (block_select_tc.cu).
//
// A row of d values (one pooled key in fp32, or one query row in bf16) gets
// one exponent: E = the largest biased exponent field of the row (a zero or
// subnormal value counts as field 1).  A value x = sign * m * 2^(e - bias')
// (m its significand with the implicit bit, e its field, at least 1) is
// represented by the integer V = trunc(m * 2^(F - W - (E - e))), negated when
// x < 0, where W is the significand width (24 for fp32, 8 for bf16) and F the
// digit bits (35 for keys, 28 for queries).  Then
//     x~ = V * 2^(E - bias' - (F - W))  and  |x - x~| < 2^(E - bias' - (F - W)),
// x~ = x exactly when the truncation drops no set bit (always when
// E - e <= F - W).  V is written in base 128 with a signed top digit:
//     keys:    V = d0*2^28 + d1*2^21 + d2*2^14 + d3*2^7 + d4,
//     queries: V = d0*2^21 + d1*2^14 + d2*2^7 + d3,
// d0 in [-128, 127] (the arithmetic shift of V), the others in [0, 127]; every
// digit is an int8.  Two's complement keeps the trailing zero digits of a
// short value zero for negative values as well.
//
// Device layouts written by dl_pool_keys / dl_cache_write:
//   Kdig int8  [b][g][kKeyDigits][n_units][d]   digit plane t of every unit
//   Kexp int32 [b][g][n_units]                  E | (inexact values << 8)
//                                               | (norm bound << 16)
// The norm bound is the bf16 bit pattern of an upper bound of the largest
// Euclidean norm of the unit's pooled key rows, max_t ||k_t||_2 (rounded up;
// the sink search bounds its fp32 logits with it).  It is computed as
// sqrt(sum_c max_t s_tc) with s_tc the sum of squares of row t's 16-byte
// column chunk c, which is at least max_t sum_c s_tc.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dl {

constexpr int kKeyDigits = 5;    // key digit planes (35 bits)
constexpr int kQueryDigits = 4;  // query digit planes (28 bits)

// Biased exponent field of an fp32 value, at least 1.
__device__ __forceinline__ int exp_field_f32(float x) {
  const int e = (int)((__float_as_uint(x) >> 23) & 255u);
  return e ? e : 1;
}
// Same for the bits of a bf16 value.
__device__ __forceinline__ int exp_field_bf16(uint32_t h) {
  const int e = (int)((h >> 7) & 255u);
  return e ? e : 1;
}

// The five key digits of fp32 x in a row of exponent E; returns true when
// x~ != x (a set bit was truncated).
__device__ __forceinline__ bool key_digits(float x, int E, int (&dg)[kKeyDigits]) {
  const uint32_t u = __float_as_uint(x);
  const uint32_t e = (u >> 23) & 255u;
  const uint32_t m = e ? ((u & 0x7FFFFFu) | 0x800000u) : (u & 0x7FFFFFu);
  const int sh = E - (e ? (int)e : 1);  // >= 0
  const uint64_t v0 = (uint64_t)m << 11;
  const uint64_t v = sh < 64 ? (v0 >> sh) : 0ull;
  const bool inexact = m != 0u && (sh >= 64 || (v << sh) != v0);
  const int64_t sv = (u >> 31) ? -(int64_t)v : (int64_t)v;
  dg[0] = (int)(sv >> 28);
  dg[1] = (int)((sv >> 21) & 127);
  dg[2] = (int)((sv >> 14) & 127);
  dg[3] = (int)((sv >> 7) & 127);
  dg[4] = (int)(sv & 127);
  return inexact;
}

// The four query digits of a bf16 value (raw 16 bits h) in a row of
// exponent E; returns true when truncated.
__device__ __forceinline__ bool query_digits(uint32_t h, int E, int (&dg)[kQueryDigits]) {
  const uint32_t e = (h >> 7) & 255u;
  const uint32_t m = e ? ((h & 0x7Fu) | 0x80u) : (h & 0x7Fu);
  const int sh = E - (e ? (int)e : 1);
  const uint32_t v0 = m << 20;
  const uint32_t v = sh < 32 ? (v0 >> sh) : 0u;
  const bool inexact = m != 0u && (sh >= 32 || (v << sh) != v0);
  const int32_t sv = ((h >> 15) & 1u) ? -(int32_t)v : (int32_t)v;
  dg[0] = sv >> 21;
  dg[1] = (sv >> 14) & 127;
  dg[2] = (sv >> 7) & 127;
  dg[3] = sv & 127;
  return inexact;
}

// The Kexp norm field from sum_c max_t s_tc (fp32 sums of squares, chunk
// sums added in chunk order): the fp32 rounding of the squares, of the sums
// and of the square root is covered by the factor 1 + 2^-14 on the sum, and
// the result is rounded up to bf16.
__device__ __forceinline__ int key_norm_field(float sq_sum) {
  const float n = sqrtf(sq_sum * (1.0f + 0x1p-14f));
  return (int)__bfloat16_as_ushort(__float2bfloat16_ru(n)) << 16;
}
// The norm bound a Kexp word holds.
__device__ __forceinline__ float key_norm_of(int kexp) {
  return __bfloat162float(__ushort_as_bfloat16((unsigned short)((unsigned)kexp >> 16)));
}

__device__ __forceinline__ uint32_t pack4_i8(int a, int b, int c, int d) {
  return (uint32_t)(a & 255) | ((uint32_t)(b & 255) << 8) | ((uint32_t)(c & 255) << 16) |
         ((uint32_t)(d & 255) << 24);
}

}  // namespace dl
