// (a5) Sink-aware top-K block selection.
//
// Focus-dLLM abstract: sink-aware pruning removes redundant attention while
// the attention sinks are always kept.  Per (b, g): the sink blocks are kept,
// the topK other blocks of largest fp64 score are added (ties -> lower
// index), and the union is written ascending.
//
// One CTA per (b, g).  Scores are staged in shared memory; a block's rank is
// the number of candidates ordered before it by (score desc, index asc),
// counted with an early exit once it reaches topK.  The ascending compaction
// is a ballot/popc prefix count over the unit indices.
#include "common.cuh"
#include "internal.h"

namespace dl {

constexpr int kSelThreads = 1024;

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const double* __restrict__ score, int H_kv, int n_units, int unit_size, int topK,
              const int32_t* __restrict__ sink_pos, int n_sinks, int32_t* __restrict__ blk_idx,
              int32_t* __restrict__ blk_cnt, int max_sel, unsigned* err) {
  extern __shared__ unsigned char smem[];
  double* s_score = reinterpret_cast<double*>(smem);
  uint8_t* s_sink = reinterpret_cast<uint8_t*>(s_score + n_units);
  __shared__ int s_warp[33];
  __shared__ int s_base;
  const int bg = blockIdx.x;
  const int b = bg / H_kv;
  const double* sc = score + (size_t)bg * n_units;
  for (int u = threadIdx.x; u < n_units; u += blockDim.x) {
    s_score[u] = sc[u];
    s_sink[u] = 0;
  }
  __syncthreads();
  if (threadIdx.x < n_sinks) {
    const int p = sink_pos[(size_t)b * n_sinks + threadIdx.x];
    if (p >= 0) {
      const long long u = p / unit_size;
      if (u < n_units) s_sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }
  if (threadIdx.x == 0) s_base = 0;
  __syncthreads();
  int32_t* out = blk_idx + (size_t)bg * max_sel;
  for (int u0 = 0; u0 < n_units; u0 += blockDim.x) {
    const int u = u0 + threadIdx.x;
    bool keep = false;
    if (u < n_units) {
      if (s_sink[u]) {
        keep = true;
      } else {
        const double v = s_score[u];
        int rank = 0;
        for (int j = 0; j < n_units && rank < topK; ++j)
          rank += (!s_sink[j]) && ranks_before(s_score[j], j, v, u);
        keep = rank < topK;
      }
    }
    int total = 0;
    const int pos = block_exclusive_count(keep, s_warp, &total);
    if (keep && s_base + pos < max_sel) out[s_base + pos] = u;
    __syncthreads();
    if (threadIdx.x == 0) s_base += total;
    __syncthreads();
  }
  const int cnt = s_base;
  for (int e = cnt + threadIdx.x; e < max_sel; e += blockDim.x) out[e] = -1;
  if (threadIdx.x == 0) blk_cnt[bg] = cnt < max_sel ? cnt : max_sel;
}

cudaError_t launch_select(const double* score, int batch, int H_kv, int n_units, int unit_size,
                          int topK, const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                          int32_t* blk_cnt, int max_sel, unsigned* err, cudaStream_t st) {
  const size_t smem = (size_t)n_units * (sizeof(double) + 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  select_kernel<<<batch * H_kv, kSelThreads, smem, st>>>(score, H_kv, n_units, unit_size, topK,
                                                         sink_pos, n_sinks, blk_idx, blk_cnt,
                                                         max_sel, err);
  return cudaGetLastError();
}

}  // namespace dl
