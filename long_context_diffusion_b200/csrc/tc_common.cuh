// Pieces shared by the tensor-core attention kernels (attn_tc.cu: query rows
// on the MMA's M side; attn_tc_kt.cu: keys on the M side): the persistent
// work split over tile slots, context-tile lookup, and the host-side tensor
// maps and launch plan.
#pragma once

#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "tiles.cuh"

namespace dl {

constexpr int kTcMaxTiles = 1024;  // tiles of one CTA (tile table in shared memory)
constexpr int kMaxSegs = 64;       // (b, g) segments of one CTA

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Block index of context tile `tile` of (b, g), or -1 (bad index, flagged).
__device__ __forceinline__ int ctx_tile_block(const AttnArgs& a, int bg, int tile) {
  if (a.mode == kDense) return tile;
  const int j = a.idx[(size_t)bg * a.max_idx + tile];
  if (j < 0 || j >= n_blocks(a.s)) {
    flag_error(a.err, ERR_BAD_INDEX);
    return -1;
  }
  return j;
}

// Persistent work split over tile slots: slot u = (bg, t) = (u / S, u % S)
// with S = the largest tile count of any (b, g); the slot holds a tile when
// t < n_tiles(bg).  CTA c owns slots [c*U/P, (c+1)*U/P) of U = n_bg*S, so the
// CTAs share the work within one tile.  The run of one (b, g) inside a CTA is
// a segment: one accumulator and one partial, at partial slot c - first(bg),
// where first(bg) is the CTA owning slot (bg, 0); a CTA whose run of a (b, g)
// holds no tile writes an empty marker (m = -inf) there instead.
struct TcPlan {
  int S;      // tile slots per (b, g)
  int nslot;  // partial slots per (b, g) (at most ceil(P / n_bg) + 1)
};

// CTA owning tile slot u when U slots are split over P CTAs.
__host__ __device__ inline int tc_owner(long long u, long long U, int P) {
  return (int)(((u + 1) * P + U - 1) / U) - 1;
}

// TMA row coordinate and valid-key count (bit 15: decode tile) of tile
// `tile` of (b, g); a context tile whose block or page is out of range is
// flagged and gets 0 valid keys.
__device__ __forceinline__ int2 tc_tile_info(const AttnArgs& a, int bg, int tile, int n_ctx) {
  const Shape& s = a.s;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  int y = 0, valid = 0;
  if (tile < n_ctx) {
    const int j = ctx_tile_block(a, bg, tile);
    if (j >= 0) {
      const int slot = a.page_table[(size_t)b * s.n_pages + j];
      if (slot < 0 || slot >= s.n_slots) {
        flag_error(a.err, ERR_BAD_INDEX);
      } else {
        valid = min(64, s.L_ctx - j * 64);
        y = (slot * s.H_kv + g) * 64;
      }
    }
  } else {
    const int td = tile - n_ctx;
    valid = min(64, s.L_q - td * 64) | (1 << 15);
    y = td * 64;
  }
  return make_int2(y, valid);
}

// ---- host side (attn_tc.cu) ----
// bf16 rows of `inner` elements, boxes of 64 x box_rows, 128-byte swizzle.
bool tc_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);
// decode block K/V: [bg][L_q][d], boxes of 64 x 64 x 1 (rows past L_q read 0)
bool tc_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t L_q, uint64_t n_bg);
// int8 planes [planes][rows][inner] (inner = 128 bytes), boxes of
// inner x box_rows x 1, 128-byte swizzle.
bool tc_map_i8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t planes, uint32_t box_rows);
int tc_sm_count();

struct TcLaunch {
  TcPlan plan;
  int grid;
};
// One CTA per SM (fewer when a CTA's tile table or segment list would
// overflow, or the partial slots exceed the workspace's kMaxSplits).
TcLaunch tc_plan(int n_bg, int max_tiles, int sms);

cudaError_t launch_combine(const AttnArgs& a, int n_split, cudaStream_t st, int S = 0, int P = 0);

}  // namespace dl
