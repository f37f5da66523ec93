// Key tiles of one (sequence, KV head) for the attention kernels.
//
// The keys a decode block attends to are a sequence of 64-row tiles: first
// the context tiles (a selected block, every block in dense mode, or 64
// gathered tokens), then ceil(L_q/64) tiles of the decode block's own keys.
// A row resolves to an element offset into the pool (through the page table)
// or into K_dec/V_dec, or to "invalid" (past the context end, a padding row,
// or an out-of-range index -- the latter also raises the device error word).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace dl {

__device__ __forceinline__ int n_blocks(const Shape& s) { return (s.L_ctx + s.page - 1) / s.page; }

__device__ __forceinline__ int ctx_tile_count(const AttnArgs& a, int bg) {
  if (a.mode == kDense) return n_blocks(a.s);
  int c = a.cnt[bg];
  c = c < 0 ? 0 : (c > a.max_idx ? a.max_idx : c);
  return a.mode == kBlocks ? c : (c + kTile - 1) / kTile;
}

// Element offset of row r of context tile `tile` of (b, g) in the pool, or
// -1 when the row holds no key.
__device__ __forceinline__ long long ctx_row_offset(const AttnArgs& a, int b, int g, int bg,
                                                    int tile, int r) {
  const Shape& s = a.s;
  long long pos;
  if (a.mode == kDense) {
    pos = (long long)tile * kTile + r;
  } else if (a.mode == kBlocks) {
    const int j = a.idx[(size_t)bg * a.max_idx + tile];
    if (j < 0 || j >= n_blocks(s)) {
      if (r == 0) flag_error(a.err, ERR_BAD_INDEX);
      return -1;
    }
    pos = (long long)j * kTile + r;
  } else {
    const int e = tile * kTile + r;
    int c = a.cnt[bg];
    c = c > a.max_idx ? a.max_idx : c;
    if (e >= c) return -1;
    pos = a.idx[(size_t)bg * a.max_idx + e];
    if (pos < 0 || pos >= s.L_ctx) {
      flag_error(a.err, ERR_BAD_INDEX);
      return -1;
    }
  }
  if (pos >= s.L_ctx) return -1;
  const int lp = (int)(pos / s.page);
  const int slot = a.page_table[(size_t)b * s.n_pages + lp];
  if (slot < 0 || slot >= s.n_slots) {
    flag_error(a.err, ERR_BAD_INDEX);
    return -1;
  }
  return (((long long)slot * s.H_kv + g) * s.page + (pos % s.page)) * s.d;
}

// Element offset of decode key i of (b, g) in K_dec/V_dec, or -1.
__device__ __forceinline__ long long dec_row_offset(const Shape& s, int bg, int i) {
  if (i >= s.L_q) return -1;
  return ((long long)bg * s.L_q + i) * s.d;
}

// Split-KV partials in the workspace: for each (b, g), split and query row
// r = (h in the group, i), the unnormalised output row, and (running max in
// natural-log units, running sum of exponentials).
struct Partials {
  float* o;    // [bg][split][R][d]
  float2* ml;  // [bg][split][R]
};

__host__ __device__ inline Partials partials_of(void* ws, const Shape& s, int n_split) {
  const size_t R = (size_t)s.G * s.L_q;
  const size_t n = (size_t)s.batch * s.H_kv * n_split * R;
  Partials p;
  p.o = reinterpret_cast<float*>(ws);
  p.ml = reinterpret_cast<float2*>(reinterpret_cast<char*>(ws) + round256(n * s.d * sizeof(float)));
  return p;
}

// Merge the split partials of one (b, g, row r) into O and lse: O = sum_s
// acc_s e^{m_s-M} / L, L = sum_s l_s e^{m_s-M}, lse = M + ln L, over slots
// [0, n_valid) of the n_split allocated.  One warp per row (lane = columns
// lane, lane + 32, ...).
template <typename T, int D>
__device__ __forceinline__ void merge_row(const Partials& part, const Shape& s, int n_split,
                                          int bg, int r, int n_valid, T* __restrict__ O,
                                          float* __restrict__ lse, int lane) {
  const int R = s.G * s.L_q;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int h = g * s.G + r / s.L_q, i = r % s.L_q;
  constexpr int CPL = D / 32;
  constexpr int SB = 4;  // slots per batch: their loads are all issued before any is used
  float o[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) o[c] = 0.0f;
  float M = -INFINITY, L = 0.0f;
  for (int s0 = 0; s0 < n_valid; s0 += SB) {
    float2 ml[SB];
    float ov[SB][CPL];
#pragma unroll
    for (int q = 0; q < SB; ++q) {
      const size_t row = ((size_t)bg * n_split + s0 + q) * R + r;
      const bool ok = s0 + q < n_valid;
      ml[q] = ok ? part.ml[row] : make_float2(-INFINITY, 0.0f);
#pragma unroll
      for (int c = 0; c < CPL; ++c)
        ov[q][c] = (ok && O) ? part.o[row * D + lane + 32 * c] : 0.0f;
    }
    // merge this batch into the running (M, L, o), as the partials themselves
    float Mb = M;
#pragma unroll
    for (int q = 0; q < SB; ++q) Mb = fmaxf(Mb, ml[q].x);
    if (Mb == -INFINITY) continue;
    const float a = M == -INFINITY ? 0.0f : expf(M - Mb);
    L *= a;
#pragma unroll
    for (int c = 0; c < CPL; ++c) o[c] *= a;
#pragma unroll
    for (int q = 0; q < SB; ++q) {
      // an empty run (m = -inf) wrote no output row: skip it, never 0 * garbage
      if (ml[q].x == -INFINITY) continue;
      const float wgt = expf(ml[q].x - Mb);
      L += ml[q].y * wgt;
#pragma unroll
      for (int c = 0; c < CPL; ++c) o[c] = fmaf(ov[q][c], wgt, o[c]);
    }
    M = Mb;
  }
  if (O) {  // O == nullptr: the row LSEs only
    const float inv = L > 0.0f ? 1.0f / L : 0.0f;
    T* dst = O + (((size_t)b * s.L_q + i) * s.H + h) * D;
#pragma unroll
    for (int c = 0; c < CPL; ++c) dst[lane + 32 * c] = from_f32<T>(o[c] * inv);
  }
  if (lse && lane == 0) lse[((size_t)b * s.H + h) * s.L_q + i] = L > 0.0f ? M + logf(L) : -INFINITY;
}

}  // namespace dl
