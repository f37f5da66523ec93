// (a7) Intra-chunk token selection over a chunked, paged prefix.
//
// Prefilling-dLLM abstract: the prefix is split into chunks cached once; the
// top-K chunks are kept with intra-chunk token sparsity; the BOS token
// prepended to each chunk acts as an attention anchor.  Per selected chunk,
// every decode query of the KV group ranks the chunk's content tokens by
// softmax mass over the chunk; the top-T tokens and the chunk's BOS are kept.
//
// One CTA per (b, g, selected chunk), one thread per content token (key row
// in registers).  For 32 query rows at a time: logits in fp32, warp-shuffle
// max/sum per row, a cross-warp pass through shared memory, then each thread
// adds its softmax probability to its token's mass.  The top-T cut is a rank
// count on (mass desc, position asc) and the kept tokens are compacted in
// ascending position order.
#include <cstdlib>

#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace dl {

constexpr int kTokThreads = 1024;
constexpr int kTokRows = 32;

template <typename T, int D>
__global__ void __launch_bounds__(kTokThreads)
token_select_kernel(Shape s, const T* __restrict__ Q, const T* __restrict__ Kp,
                    const int32_t* __restrict__ page_table, const int32_t* __restrict__ chunk_idx,
                    int n_sel, int stride, int content, int topT, int32_t* __restrict__ tok_pos,
                    int32_t* __restrict__ tok_cnt, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sQ[kTokRows * D];
  __shared__ float sRed[kTokRows][33];
  __shared__ float sStat[kTokRows];
  __shared__ float sTau[kTokThreads];
  __shared__ int s_warp[33];
  const int sel = blockIdx.x, bg = blockIdx.y;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int c = chunk_idx[(size_t)bg * n_sel + sel];
  const long long base = (long long)c * stride;
  const int per = topT + 1;
  int32_t* out = tok_pos + ((size_t)bg * n_sel + sel) * per;
  if (c < 0 || base + content >= (long long)s.L_ctx) {
    if (t == 0) flag_error(err, ERR_BAD_INDEX);
    for (int e = t; e < per; e += blockDim.x) out[e] = -1;
    if (t == 0 && sel == 0) tok_cnt[bg] = n_sel * per;
    return;
  }
  // key row of content token t (logical position base + 1 + t); it is
  // re-read (16 bytes at a time) for every pass of 32 query rows so that
  // only the 32 running dot products live in registers.
  const T* src = nullptr;
  bool ok = t < content;
  if (ok) {
    const long long pos = base + 1 + t;
    const int slot = page_table[(size_t)b * s.n_pages + pos / s.page];
    if (slot < 0 || slot >= s.n_slots) {
      flag_error(err, ERR_BAD_INDEX);
      ok = false;
    } else {
      src = Kp + (((size_t)slot * s.H_kv + g) * s.page + pos % s.page) * D;
    }
  }
  const int R = s.G * s.L_q;
  const float scale = (float)s.scale;
  float tau = 0.0f;
  for (int r0 = 0; r0 < R; r0 += kTokRows) {
    const int nr = min(kTokRows, R - r0);
    __syncthreads();
    for (int e = t; e < kTokRows * D; e += blockDim.x) {
      const int rr = e / D, x = e % D, r = r0 + rr;
      float v = 0.0f;
      if (r < R) {
        const int h = g * s.G + r / s.L_q, i = r % s.L_q;
        v = to_f32(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + x]);
      }
      sQ[rr * D + x] = v;
    }
    __syncthreads();
    float lg[kTokRows];
#pragma unroll
    for (int rr = 0; rr < kTokRows; ++rr) lg[rr] = 0.0f;
    if (ok) {
      constexpr int EPT = Vec16<T>::N;
      for (int x0 = 0; x0 < D; x0 += EPT) {
        float kv[EPT];
        Vec16<T>::load(src + x0, kv);
#pragma unroll
        for (int rr = 0; rr < kTokRows; ++rr)
#pragma unroll
          for (int x = 0; x < EPT; ++x) lg[rr] = fmaf(sQ[rr * D + x0 + x], kv[x], lg[rr]);
      }
    }
#pragma unroll
    for (int rr = 0; rr < kTokRows; ++rr) {
      lg[rr] = (ok && rr < nr) ? lg[rr] * scale : -INFINITY;
      const float m = warp_max(lg[rr]);
      if (lane == 0) sRed[rr][warp] = m;
    }
    __syncthreads();
    if (warp < kTokRows) {   // warp rr reduces row rr over the 32 warps
      const float m = warp_max(sRed[warp][lane]);
      if (lane == 0) sStat[warp] = m;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kTokRows; ++rr) {
      const float e = lg[rr] == -INFINITY ? 0.0f : expf(lg[rr] - sStat[rr]);
      lg[rr] = e;
      const float z = warp_sum(e);
      if (lane == 0) sRed[rr][warp] = z;
    }
    __syncthreads();
    if (warp < kTokRows) {
      const float z = warp_sum(sRed[warp][lane]);
      if (lane == 0) sRed[warp][32] = z;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < kTokRows; ++rr)
      if (rr < nr) tau += lg[rr] / sRed[rr][32];
  }
  sTau[t] = ok ? tau : -INFINITY;
  __syncthreads();
  bool keep = false;
  if (t < content) {
    int rank = 0;
    for (int j = 0; j < content && rank < topT; ++j) {
      const float v = sTau[j];
      rank += (v > sTau[t]) || (v == sTau[t] && j < t);
    }
    keep = rank < topT;
  }
  int total = 0;
  const int p = block_exclusive_count(keep, s_warp, &total);
  if (keep) out[1 + p] = (int)(base + 1 + t);
  if (t == 0) {
    out[0] = (int)base;
    if (sel == 0) tok_cnt[bg] = n_sel * per;
  }
  for (int e = 1 + total + t; e < per; e += blockDim.x) out[e] = -1;
}

bool token_select_tc_supported(const Shape& s, int chunk_stride, int chunk_content);
cudaError_t launch_token_select_tc(const Shape& s, const void* Q, const void* Kp,
                                   const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                                   int chunk_stride, int chunk_content, int topT,
                                   const int32_t* Kexp, int32_t* tok_pos, int32_t* tok_cnt,
                                   unsigned* err, cudaStream_t st);

// bf16, d 128, page-aligned chunks of at most 64 rows per group: the tensor
// cores (token_select_tc.cu); otherwise the CUDA-core kernel above.
cudaError_t launch_token_select(const Shape& s, const void* Q, const void* Kp,
                                const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                                int chunk_stride, int chunk_content, int topT,
                                const int32_t* Kexp, int32_t* tok_pos, int32_t* tok_cnt,
                                unsigned* err, cudaStream_t st) {
  if (token_select_tc_supported(s, chunk_stride, chunk_content) && !(kernel_flags() & DL_FLAG_TOKEN_SIMT))
    return launch_token_select_tc(s, Q, Kp, page_table, chunk_idx, n_sel, chunk_stride,
                                  chunk_content, topT, Kexp, tok_pos, tok_cnt, err, st);
  dim3 grid(n_sel, s.batch * s.H_kv);
  if (s.dtype == 0) {
    auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
    auto* k = reinterpret_cast<const __nv_bfloat16*>(Kp);
    if (s.d == 128)
      DL_LAUNCH(token_select_kernel<__nv_bfloat16, 128>, grid, kTokThreads, 0, st, 
          s, q, k, page_table, chunk_idx, n_sel, chunk_stride, chunk_content, topT, tok_pos,
          tok_cnt, err);
    else
      DL_LAUNCH(token_select_kernel<__nv_bfloat16, 64>, grid, kTokThreads, 0, st, 
          s, q, k, page_table, chunk_idx, n_sel, chunk_stride, chunk_content, topT, tok_pos,
          tok_cnt, err);
  } else {
    auto* q = reinterpret_cast<const float*>(Q);
    auto* k = reinterpret_cast<const float*>(Kp);
    if (s.d == 128)
      DL_LAUNCH(token_select_kernel<float, 128>, grid, kTokThreads, 0, st, 
          s, q, k, page_table, chunk_idx, n_sel, chunk_stride, chunk_content, topT, tok_pos,
          tok_cnt, err);
    else
      DL_LAUNCH(token_select_kernel<float, 64>, grid, kTokThreads, 0, st, 
          s, q, k, page_table, chunk_idx, n_sel, chunk_stride, chunk_content, topT, tok_pos,
          tok_cnt, err);
  }
  return cudaGetLastError();
}

}  // namespace dl
