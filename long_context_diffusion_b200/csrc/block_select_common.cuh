// Shared by the two fused score + select kernels of one (b, g) per CTA:
// the fp64 scoring of block_select.cu (also the exact fallback of the int8
// tensor-core kernel, block_select_tc.cu) and the selection both end with.
//
// Focus-dLLM (research.elamur.ai summary): the predicted queries score every
// KV block against the block's mean key, and the most relevant blocks are
// kept; the abstract adds that the attention sinks are always kept.
//   l[r][u] = scale * q_r . Kbar_u,   score[u] = sum_r softmax_u(l[r][.]),
//   keep the sink units, then the topK other units of largest score (ties to
//   the lower index), ascending.
#pragma once

#include "common.cuh"
#include "internal.h"
#include "score_common.cuh"

namespace dl {

namespace bs {
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kChunk = kWarps * 8;  // pooled keys per chunk: one 8-key MMA tile per warp
constexpr int kMaxChunks = 4;
constexpr int kMaxUnits = kChunk * kMaxChunks;  // 512, = kThreads (one key per thread)
constexpr int kMaxRows = 32;

template <typename T, int D>
struct Smem {
  static constexpr int QP = D + 2;                    // fp64 query pitch
  static constexpr int K_BYTES = kChunk * D * 4;      // one chunk of fp32 pooled keys
  static constexpr int Q_BYTES = kMaxRows * QP * 8;
  static constexpr int RAW_BYTES = kMaxRows * D * (int)sizeof(T);
  static constexpr int RAW_OFF = 2 * K_BYTES + Q_BYTES - RAW_BYTES;  // copied rows, in the fp64 area
  static constexpr int BYTES = 2 * K_BYTES + Q_BYTES;
  static_assert(RAW_BYTES <= Q_BYTES && RAW_OFF % 16 == 0, "raw query rows inside the fp64 area");
};
}  // namespace bs

// Selection scratch of one CTA of kThreads threads (one unit per thread).
struct BsSelScratch {
  uint64_t key[bs::kMaxUnits];
  int idx[bs::kMaxUnits];
  uint8_t sink[bs::kMaxUnits], keep[bs::kMaxUnits];
  int warp[33];
};

// Position i's entry after the sort by (score desc, index asc), sinks and
// padding last; n_sb sink units, n_cand = the other units.
struct BsSorted {
  uint64_t key;
  int idx;
  int n_sb;
  int n_cand;
};

// Marks the sink units and sorts (as select_shfl_kernel): thread i holds
// unit i's score on entry (units past n_units are ignored).  Every thread of
// the CTA (kThreads) calls it.  NW: the network's width, a power of two
// >= n_units and >= 32; each NW-aligned group of threads is sorted on its
// own, so threads 0 .. NW-1 hold the result (a narrow network skips the
// shared-memory stages a 512-wide one needs).
template <int NW = bs::kThreads>
__device__ __forceinline__ BsSorted bs_sort(double my_score, int n_units, int b, int unit_size,
                                            const int32_t* __restrict__ sink_pos, int n_sinks,
                                            BsSelScratch& sc, unsigned* err) {
  using namespace bs;
  const int i = threadIdx.x;
  sc.sink[i] = 0;
  sc.keep[i] = 0;
  __syncthreads();
  for (int q = i; q < n_sinks; q += kThreads) {
    const int p = sink_pos[(size_t)b * n_sinks + q];
    if (p >= 0) {
      const long long u = p / unit_size;
      if (u < n_units) sc.sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  const bool is_sink = i < n_units && sc.sink[i];
  BsSorted r;
  r.n_sb = __syncthreads_count(is_sink);
  uint64_t key = (i < n_units && !is_sink) ? desc_key(my_score) : ~0ull;
  int idx = i;
  static_assert(NW >= 32 && NW <= kThreads && (NW & (NW - 1)) == 0, "network width");
  for (int k = 2; k <= NW; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      uint64_t pk;
      int px;
      if (j >= 32) {
        sc.key[i] = key;
        sc.idx[i] = idx;
        __syncthreads();
        pk = sc.key[i ^ j];
        px = sc.idx[i ^ j];
        __syncthreads();
      } else {
        pk = __shfl_xor_sync(0xffffffffu, key, j);
        px = __shfl_xor_sync(0xffffffffu, idx, j);
      }
      const bool keep_min = ((i & j) == 0) == ((i & k) == 0);
      const bool p_less = pk < key || (pk == key && px < idx);
      if (keep_min == p_less) {
        key = pk;
        idx = px;
      }
    }
  }
  r.key = key;
  r.idx = idx;
  r.n_cand = n_units - r.n_sb;
  return r;
}

// Keeps the first topK sorted candidates and the sinks; writes the ascending
// list and the count.
__device__ __forceinline__ void bs_write(const BsSorted& r, int n_units, int topK, int bg,
                                         int32_t* __restrict__ blk_idx,
                                         int32_t* __restrict__ blk_cnt, int max_sel,
                                         BsSelScratch& sc) {
  using namespace bs;
  const int i = threadIdx.x;
  const int take = topK < r.n_cand ? topK : r.n_cand;
  if (i < take) sc.keep[r.idx] = 1;
  __syncthreads();
  const bool keep = i < n_units && (sc.keep[i] || sc.sink[i]);
  int total = 0;
  const int pos = block_exclusive_count(keep, sc.warp, &total);
  int32_t* out = blk_idx + (size_t)bg * max_sel;
  if (keep && pos < max_sel) out[pos] = i;
  for (int e = total + i; e < max_sel; e += kThreads) out[e] = -1;
  if (i == 0) blk_cnt[bg] = total < max_sel ? total : max_sel;
}

// The score a key of desc_key() came from.
__device__ __forceinline__ double score_of_desc_key(uint64_t k) {
  const uint64_t mono = ~k;
  const uint64_t b = (mono >> 63) ? (mono & 0x7FFFFFFFFFFFFFFFull) : ~mono;
  return __longlong_as_double((long long)b);
}

template <typename T, int D, int MT>
__device__ __forceinline__ void
block_select_fp64(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                    const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar, Shape s,
                    int n_units, double* __restrict__ score, int unit_size, int topK,
                    const int32_t* __restrict__ sink_pos, int n_sinks,
                    int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt, int max_sel,
                    unsigned* err, uint8_t* smem_b) {
  using namespace bs;
  using L = Smem<T, D>;
  constexpr int KG = D / 16;               // k-groups of 16 dimensions
  constexpr int CPR = D * sizeof(T) / 16;  // 16-byte chunks per query row
  constexpr int NP = kMaxRows * (D / 2) / kThreads;  // query pairs converted per thread
  float* sK = reinterpret_cast<float*>(smem_b);                         // [2][kChunk][D]
  double* sQ = reinterpret_cast<double*>(smem_b + 2 * L::K_BYTES);      // [kMaxRows][QP]
  T* sRaw = reinterpret_cast<T*>(smem_b + L::RAW_OFF);                  // [kMaxRows][D]
  __shared__ double s_red[kWarps][kMaxRows];
  __shared__ double s_M[kMaxRows], s_Zi[kMaxRows];
  __shared__ double s_score[kMaxUnits];
  __shared__ BsSelScratch s_sel;

  const int bg = blockIdx.x;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gi = lane >> 2, t = lane & 3;
  const int nch = (n_units + kChunk - 1) / kChunk;

  auto load_chunk = [&](int c) {
    float* dst = sK + (c & 1) * kChunk * D;
    const float* src = Kbar + ((size_t)bg * n_units + (size_t)c * kChunk) * D;
    for (int e = tid; e < kChunk * (D / 4); e += kThreads) {
      const int j = e / (D / 4), col = (e % (D / 4)) * 4;
      const bool ok = c * kChunk + j < n_units;
      cp_async16(dst + j * D + key_chunk(j, col >> 2) * 4, ok ? src + (size_t)j * D + col : Kbar,
                 ok);
    }
    cp_async_commit();
  };
  load_chunk(0);

  // query rows: every predicted position of every query head of the group
  int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  if (nq * s.G > 8 * MT) {  // more rows than the caller's bound: reported, rows cut
    if (tid == 0) flag_error(err, ERR_BAD_INDEX);
    nq = 8 * MT / s.G;
  }
  const int R = nq * s.G;  // <= 8 * MT <= kMaxRows
  for (int c = tid; c < kMaxRows * CPR; c += kThreads) {
    const int r = c / CPR, ch = c % CPR;
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
    cp_async16(sRaw + r * D + ch * (16 / sizeof(T)), src, ok);
  }
  cp_async_commit();
  if (nch > 1) load_chunk(1);
  if (nch > 1) cp_async_wait<1>(); else cp_async_wait<0>();  // chunk 0 and the rows
  __syncthreads();
  {  // rows to fp64 (the copied rows share the area: read all, sync, write)
    float2 v[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int c = tid + q * kThreads;
      v[q] = load_pair(sRaw + (c / (D / 2)) * D + (c % (D / 2)) * 2);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int c = tid + q * kThreads;
      *reinterpret_cast<double2*>(sQ + (c / (D / 2)) * L::QP + (c % (D / 2)) * 2) =
          make_double2(v[q].x, v[q].y);
    }
  }
  __syncthreads();

  // ---- logits: acc[c][m][i] = row 8m + gi, key c*128 + 8*warp + 2t + i, for
  // the MT row tiles of the launch (a compile-time count: a predicate on
  // every MMA measured 30 % slower; tiles past R hold zero rows)
  double acc[kMaxChunks][kMaxRows / 8][2];
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
    for (int m = 0; m < kMaxRows / 8; ++m) acc[c][m][0] = acc[c][m][1] = 0.0;
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c) {
    if (c < nch) {
      if (c > 0) {
        if (c + 1 < nch) cp_async_wait<1>(); else cp_async_wait<0>();
        __syncthreads();
      }
      const float* sKc = sK + (c & 1) * kChunk * D + (warp * 8 + gi) * D;
#pragma unroll 2
      for (int kg = 0; kg < KG; ++kg) {
        const float4 bv = *reinterpret_cast<const float4*>(sKc + key_chunk(gi, 4 * kg + t) * 4);
        double a[MT][4];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const double* qa = sQ + (8 * m + gi) * L::QP + 16 * kg + 4 * t;
          const double2 a01 = *reinterpret_cast<const double2*>(qa);
          const double2 a23 = *reinterpret_cast<const double2*>(qa + 2);
          a[m][0] = a01.x; a[m][1] = a01.y; a[m][2] = a23.x; a[m][3] = a23.y;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const double bk = i == 0 ? bv.x : i == 1 ? bv.y : i == 2 ? bv.z : bv.w;
#pragma unroll
          for (int m = 0; m < MT; ++m) dmma_m8n8k4(acc[c][m], a[m][i], bk);
        }
      }
      __syncthreads();  // every warp is done with this buffer
      if (c + 2 < nch) load_chunk(c + 2);
    }
  }

  // ---- softmax over the keys of each row, then the column sums
  // scale; keys past the end take -inf
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
    for (int m = 0; m < kMaxRows / 8; ++m)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const int u = c * kChunk + warp * 8 + 2 * t + i;
        acc[c][m][i] = (c < nch && u < n_units) ? acc[c][m][i] * s.scale : -INFINITY;
      }
#pragma unroll
  for (int m = 0; m < kMaxRows / 8; ++m) {
    double mx = -INFINITY;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c) mx = fmax(mx, fmax(acc[c][m][0], acc[c][m][1]));
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    if (t == 0) s_red[warp][8 * m + gi] = mx;
  }
  __syncthreads();
  if (tid < kMaxRows) {
    double mx = s_red[0][tid];
    for (int w = 1; w < kWarps; ++w) mx = fmax(mx, s_red[w][tid]);
    s_M[tid] = mx;
  }
  __syncthreads();
#pragma unroll
  for (int m = 0; m < kMaxRows / 8; ++m) {
    const double M = s_M[8 * m + gi];
    double z = 0.0;
#pragma unroll
    for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
      for (int i = 0; i < 2; ++i) {
        const double p = (m < MT && acc[c][m][i] != -INFINITY) ? exp(acc[c][m][i] - M) : 0.0;
        acc[c][m][i] = p;
        z += p;
      }
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    if (t == 0) s_red[warp][8 * m + gi] = z;
  }
  __syncthreads();
  if (tid < kMaxRows) {
    double z = 0.0;
    for (int w = 0; w < kWarps; ++w) z += s_red[w][tid];
    s_Zi[tid] = (tid < R && z > 0.0) ? 1.0 / z : 0.0;
  }
  __syncthreads();
#pragma unroll
  for (int c = 0; c < kMaxChunks; ++c)
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      double col = 0.0;
#pragma unroll
      for (int m = 0; m < kMaxRows / 8; ++m) col += acc[c][m][i] * s_Zi[8 * m + gi];
      col += __shfl_xor_sync(0xffffffffu, col, 4);
      col += __shfl_xor_sync(0xffffffffu, col, 8);
      col += __shfl_xor_sync(0xffffffffu, col, 16);
      const int u = c * kChunk + warp * 8 + 2 * t + i;
      if (gi == 0 && c < nch && u < n_units) s_score[u] = col;
    }
  __syncthreads();

  // ---- selection (as select_shfl_kernel, on the scores in shared memory)
  const int i = tid;  // key position in the network, kMaxUnits = kThreads
  if (i < n_units) score[(size_t)bg * n_units + i] = s_score[i];
  // a network as wide as the units (the 512-wide one for at most 32 units
  // spends most of its stages on padding)
  const double my = i < n_units ? s_score[i] : 0.0;
  BsSorted r =
      n_units <= 32    ? bs_sort<32>(my, n_units, b, unit_size, sink_pos, n_sinks, s_sel, err)
      : n_units <= 64  ? bs_sort<64>(my, n_units, b, unit_size, sink_pos, n_sinks, s_sel, err)
      : n_units <= 128 ? bs_sort<128>(my, n_units, b, unit_size, sink_pos, n_sinks, s_sel, err)
      : n_units <= 256 ? bs_sort<256>(my, n_units, b, unit_size, sink_pos, n_sinks, s_sel, err)
                       : bs_sort<512>(my, n_units, b, unit_size, sink_pos, n_sinks, s_sel, err);
  bs_write(r, n_units, topK, bg, blk_idx, blk_cnt, max_sel, s_sel);
}

}  // namespace dl
