// (a3 + a5) Block scores and sink-aware top-K selection of one layer, fused:
// one CTA per (b, g).
//
// Focus-dLLM (research.elamur.ai summary): the predicted queries score every
// KV block against the block's mean key, and the most relevant blocks are
// kept; the abstract adds that the attention sinks are always kept.  The
// computation is the one of scores.cu followed by select.cu:
//   l[r][u] = scale * q_r . Kbar_u,   score[u] = sum_r softmax_u(l[r][.]),
//   keep the sink units, then the topK other units of largest score (ties to
//   the lower index), ascending.
//
// A CTA of 16 warps owns one (b, g) and up to 512 pooled keys (four chunks
// of 128).  Warp w multiplies the query rows (at most 32: four 8-row MMA
// tiles) with keys 8w .. 8w+7 of every chunk on the fp64 m8n8k4 MMA (the
// same k-slot assignment and per-accumulator order as scores.cu, so the
// logits are the same numbers) and keeps its logits in registers.  Chunks of
// pooled keys are double-buffered in shared memory (cp.async).  The row
// maxima and sums are reduced over lanes by shuffles and over warps through
// shared memory, the column sums over rows by shuffles; the scores then stay
// in shared memory for the bitonic selection of select.cu (one key per
// thread, warp shuffles below distance 32).  Larger shapes take the separate
// kernels (launch_scores, launch_select).
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
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

template <typename T, int D, int MT>
__global__ void __launch_bounds__(bs::kThreads, 1)
block_select_kernel(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                    const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar, Shape s,
                    int n_units, double* __restrict__ score, int unit_size, int topK,
                    const int32_t* __restrict__ sink_pos, int n_sinks,
                    int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt, int max_sel,
                    unsigned* err) {
  pdl_trigger();
  pdl_wait();
  using namespace bs;
  using L = Smem<T, D>;
  constexpr int KG = D / 16;               // k-groups of 16 dimensions
  constexpr int CPR = D * sizeof(T) / 16;  // 16-byte chunks per query row
  constexpr int NP = kMaxRows * (D / 2) / kThreads;  // query pairs converted per thread
  extern __shared__ __align__(16) uint8_t smem_b[];
  float* sK = reinterpret_cast<float*>(smem_b);                         // [2][kChunk][D]
  double* sQ = reinterpret_cast<double*>(smem_b + 2 * L::K_BYTES);      // [kMaxRows][QP]
  T* sRaw = reinterpret_cast<T*>(smem_b + L::RAW_OFF);                  // [kMaxRows][D]
  __shared__ double s_red[kWarps][kMaxRows];
  __shared__ double s_M[kMaxRows], s_Zi[kMaxRows];
  __shared__ double s_score[kMaxUnits];
  __shared__ uint64_t s_key[kMaxUnits];
  __shared__ int s_idx[kMaxUnits];
  __shared__ uint8_t s_sink[kMaxUnits], s_keep[kMaxUnits];
  __shared__ int s_warp[33];

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
  s_sink[i] = 0;
  s_keep[i] = 0;
  __syncthreads();
  for (int q = i; q < n_sinks; q += kThreads) {
    const int p = sink_pos[(size_t)b * n_sinks + q];
    if (p >= 0) {
      const long long u = p / unit_size;
      if (u < n_units) s_sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  const bool is_sink = i < n_units && s_sink[i];
  const int n_sb = __syncthreads_count(is_sink);
  uint64_t key = (i < n_units && !is_sink) ? desc_key(s_score[i]) : ~0ull;
  int idx = i;
  for (int k = 2; k <= kThreads; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      uint64_t pk;
      int px;
      if (j >= 32) {
        s_key[i] = key;
        s_idx[i] = idx;
        __syncthreads();
        pk = s_key[i ^ j];
        px = s_idx[i ^ j];
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
  const int n_cand = n_units - n_sb;
  const int take = topK < n_cand ? topK : n_cand;
  if (i < take) s_keep[idx] = 1;
  __syncthreads();
  const bool keep = i < n_units && (s_keep[i] || s_sink[i]);
  int total = 0;
  const int pos = block_exclusive_count(keep, s_warp, &total);
  int32_t* out = blk_idx + (size_t)bg * max_sel;
  if (keep && pos < max_sel) out[pos] = i;
  for (int e = total + i; e < max_sel; e += kThreads) out[e] = -1;
  if (i == 0) blk_cnt[bg] = total < max_sel ? total : max_sel;
}

// Fused when the group's query rows (G x the bound max_q on q_cnt, or x L_q)
// fit four MMA row tiles and the keys one thread each; otherwise block scores
// then selection, as separate kernels.
cudaError_t launch_block_select(const Shape& s, const void* Q, const int32_t* q_idx,
                                const int32_t* q_cnt, const float* Kbar, int n_units,
                                double* score, int unit_size, int topK, const int32_t* sink_pos,
                                int n_sinks, int32_t* blk_idx, int32_t* blk_cnt, int max_sel,
                                int max_q, void* ws, unsigned* err, cudaStream_t st) {
  const int nq_max = (max_q > 0 && max_q < s.L_q && q_idx) ? max_q : s.L_q;
  const int rows = s.G * nq_max;
  if (rows > bs::kMaxRows || n_units > bs::kMaxUnits) {
    cudaError_t e = launch_scores(s, Q, q_idx, q_cnt, Kbar, n_units, score, ws, err, st);
    if (e != cudaSuccess) return e;
    return launch_select(score, s.batch, s.H_kv, n_units, unit_size, topK, sink_pos, n_sinks,
                         blk_idx, blk_cnt, max_sel, err, st);
  }
  cudaError_t e;
#define DL_BLOCK_SELECT_MT(T, D_, MT)                                                          \
  {                                                                                           \
    auto k = block_select_kernel<T, D_, MT>;                                                  \
    constexpr int smem = bs::Smem<T, D_>::BYTES;                                              \
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=   \
        cudaSuccess)                                                                          \
      return e;                                                                               \
    DL_LAUNCH(k, s.batch * s.H_kv, bs::kThreads, smem, st, reinterpret_cast<const T*>(Q), q_idx, \
              q_cnt, Kbar, s, n_units, score, unit_size, topK, sink_pos, n_sinks, blk_idx,    \
              blk_cnt, max_sel, err);                                                         \
  }
  // row tiles for the largest group the caller can produce (one kernel per count)
#define DL_BLOCK_SELECT(T, D_)                                                                 \
  switch ((rows + 7) / 8) {                                                                   \
    case 0:                                                                                   \
    case 1: DL_BLOCK_SELECT_MT(T, D_, 1) break;                                               \
    case 2: DL_BLOCK_SELECT_MT(T, D_, 2) break;                                               \
    case 3: DL_BLOCK_SELECT_MT(T, D_, 3) break;                                               \
    default: DL_BLOCK_SELECT_MT(T, D_, 4) break;                                              \
  }
  if (s.dtype == 0) {
    if (s.d == 128) DL_BLOCK_SELECT(__nv_bfloat16, 128) else DL_BLOCK_SELECT(__nv_bfloat16, 64)
  } else {
    if (s.d == 128) DL_BLOCK_SELECT(float, 128) else DL_BLOCK_SELECT(float, 64)
  }
#undef DL_BLOCK_SELECT
#undef DL_BLOCK_SELECT_MT
  return cudaGetLastError();
}

}  // namespace dl
