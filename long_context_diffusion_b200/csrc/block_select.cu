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
#include "block_select_common.cuh"
#include "launch.cuh"

namespace dl {

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
  extern __shared__ __align__(16) uint8_t smem_b[];
  block_select_fp64<T, D, MT>(Q, q_idx, q_cnt, Kbar, s, n_units, score, unit_size, topK,
                              sink_pos, n_sinks, blk_idx, blk_cnt, max_sel, err, smem_b);
}

// The int8 tensor-core kernel (block_select_tc.cu) when the caller passes the
// key digits and the shape fits it; else fused on the fp64 MMA when the
// group's query rows (G x the bound max_q on q_cnt, or x L_q) fit four MMA
// row tiles and the keys one thread each; else, for more rows over at most
// 128 units, the kernel of block_select_wide.cu; otherwise block
// scores then selection, as separate kernels.
cudaError_t launch_block_select(const Shape& s, const void* Q, const int32_t* q_idx,
                                const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                                const int32_t* Kexp, int n_units, double* score, int unit_size,
                                int topK, const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                                int32_t* blk_cnt, int max_sel, int max_q, void* ws,
                                unsigned* err, cudaStream_t st) {
  const int nq_max = (max_q > 0 && max_q < s.L_q && q_idx) ? max_q : s.L_q;
  const int rows = s.G * nq_max;
  if (Kdig && Kexp && block_select_tc_supported(s, rows, n_units))
    return launch_block_select_tc(s, Q, q_idx, q_cnt, Kbar, Kdig, Kexp, n_units, score, unit_size,
                                  topK, sink_pos, n_sinks, blk_idx, blk_cnt, max_sel, rows, err,
                                  st);
  if (rows > bs::kMaxRows && block_select_wide_supported(s, rows, n_units))
    return launch_block_select_wide(s, Q, q_idx, q_cnt, Kbar, n_units, score, unit_size, topK,
                                    sink_pos, n_sinks, blk_idx, blk_cnt, max_sel, rows, err, st);
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
