// (a1) Past-confidence-guided query prediction.
//
// Focus-dLLM (research.elamur.ai summary; key point 1): the previous step's
// confidence over still-masked positions predicts the next unmasked positions
// (top-k, k = 4 in the paper's measurement); each guess is widened into a
// local window.  One CTA per sequence, one thread per decode position: the
// top-k test is a rank count on (confidence desc, position asc), the window
// union is a neighbourhood test, and the ascending compaction is a ballot /
// popc prefix count.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace dl {

__global__ void __launch_bounds__(1024)
predict_kernel(const float* __restrict__ conf, const uint8_t* __restrict__ masked, int L_q,
               int k, int w, int32_t* __restrict__ q_idx, int32_t* __restrict__ q_cnt) {
  pdl_trigger();
  pdl_wait();
  __shared__ float s_conf[1024];
  __shared__ uint8_t s_mask[1024];
  __shared__ uint8_t s_chosen[1024];
  __shared__ int s_warp[33];
  const int b = blockIdx.x;
  const int i = threadIdx.x;
  const size_t base = (size_t)b * L_q;
  if (i < L_q) {
    s_conf[i] = conf[base + i];
    s_mask[i] = masked[base + i] != 0;
  }
  __syncthreads();
  bool chosen = false;
  if (i < L_q && s_mask[i]) {
    const float ci = s_conf[i];
    int rank = 0;
    for (int j = 0; j < L_q && rank < k; ++j) {
      if (s_mask[j]) {
        const float cj = s_conf[j];
        rank += (cj > ci) || (cj == ci && j < i);
      }
    }
    chosen = rank < k;
  }
  if (i < L_q) s_chosen[i] = chosen;
  __syncthreads();
  bool mark = false;
  if (i < L_q) {
    const int lo = max(0, i - w), hi = min(L_q - 1, i + w);
    for (int j = lo; j <= hi && !mark; ++j) mark = s_chosen[j] != 0;
  }
  int total = 0;
  const int pos = block_exclusive_count(mark, s_warp, &total);
  if (mark) q_idx[base + pos] = i;
  if (i >= total && i < L_q) q_idx[base + i] = -1;
  if (i == 0) q_cnt[b] = total;
}

cudaError_t launch_predict(const float* conf, const uint8_t* masked, int batch, int L_q, int k,
                           int w, int32_t* q_idx, int32_t* q_cnt, cudaStream_t st) {
  const int threads = ((L_q + 31) / 32) * 32;
  DL_LAUNCH(predict_kernel, batch, threads, 0, st, conf, masked, L_q, k, w, q_idx, q_cnt);
  return cudaGetLastError();
}

}  // namespace dl
