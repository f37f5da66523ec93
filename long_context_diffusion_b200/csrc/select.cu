// (a5) Sink-aware top-K block selection.
//
// Focus-dLLM abstract: sink-aware pruning removes redundant attention while
// the attention sinks are always kept.  Per (b, g): the sink blocks are kept,
// the topK other blocks of largest fp64 score are added (ties -> lower
// index), and the union is written ascending.
//
// One CTA per (b, g).  The candidates are sorted by (score desc, index asc)
// -- the score's bits made order-preserving and inverted, the index as the
// tie-break -- with sinks and padding sorted last; the first topK entries
// are kept.  Up to 1024 units: a bitonic sort with one key per thread held
// in registers, partners at distance < 32 exchanged by warp shuffles and
// farther ones through shared memory.  Up to 4096: the same network entirely
// in shared memory.  Larger unit counts use a rank count (the number of
// candidates ordered before each unit).  The ascending compaction is a
// ballot/popc prefix count over the unit indices.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "score_common.cuh"

namespace dl {

constexpr int kSelThreads = 1024;
constexpr int kShflMax = 1024;
constexpr int kBitonicMax = 4096;


// blockDim.x = n2, a power of two in [32, 1024] with n2 >= n_units; thread
// i holds the key at position i of the network.
__global__ void __launch_bounds__(kShflMax)
select_shfl_kernel(const double* __restrict__ score, int H_kv, int n_units, int unit_size,
                   int topK, const int32_t* __restrict__ sink_pos, int n_sinks,
                   int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt, int max_sel,
                   unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ uint64_t s_key[kShflMax];
  __shared__ int s_idx[kShflMax];
  __shared__ uint8_t s_sink[kShflMax];
  __shared__ uint8_t s_keep[kShflMax];
  __shared__ int s_warp[33];
  const int n2 = blockDim.x;
  const int i = threadIdx.x;
  const int bg = blockIdx.x;
  const int b = bg / H_kv;
  s_sink[i] = 0;
  s_keep[i] = 0;
  __syncthreads();
  for (int t = i; t < n_sinks; t += n2) {
    const int p = sink_pos[(size_t)b * n_sinks + t];
    if (p >= 0) {
      const long long u = p / unit_size;
      if (u < n_units) s_sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  const bool is_sink = i < n_units && s_sink[i];
  const int n_sb = __syncthreads_count(is_sink);
  uint64_t key = (i < n_units && !is_sink) ? desc_key(score[(size_t)bg * n_units + i]) : ~0ull;
  int idx = i;
  for (int k = 2; k <= n2; k <<= 1) {
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
      // Ascending runs where (i & k) == 0; the lower position of a pair
      // keeps the smaller key there and the larger one elsewhere.
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
  for (int e = total + i; e < max_sel; e += n2) out[e] = -1;
  if (i == 0) blk_cnt[bg] = total < max_sel ? total : max_sel;
}

__global__ void __launch_bounds__(kSelThreads)
select_bitonic_kernel(const double* __restrict__ score, int H_kv, int n_units, int n2,
                      int unit_size, int topK, const int32_t* __restrict__ sink_pos, int n_sinks,
                      int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt, int max_sel,
                      unsigned* err) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) unsigned char smem[];
  uint64_t* s_key = reinterpret_cast<uint64_t*>(smem);
  int* s_idx = reinterpret_cast<int*>(s_key + n2);
  uint8_t* s_sink = reinterpret_cast<uint8_t*>(s_idx + n2);
  uint8_t* s_keep = s_sink + n2;
  __shared__ int s_warp[33];
  __shared__ int s_nsb;
  __shared__ int s_base;
  const int bg = blockIdx.x;
  const int b = bg / H_kv;
  const double* sc = score + (size_t)bg * n_units;
  for (int u = threadIdx.x; u < n2; u += blockDim.x) {
    s_sink[u] = 0;
    s_keep[u] = 0;
  }
  if (threadIdx.x == 0) { s_nsb = 0; s_base = 0; }
  __syncthreads();
  for (int t = threadIdx.x; t < n_sinks; t += blockDim.x) {
    const int p = sink_pos[(size_t)b * n_sinks + t];
    if (p >= 0) {
      const long long u = p / unit_size;
      if (u < n_units) s_sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }
  __syncthreads();
  for (int u = threadIdx.x; u < n2; u += blockDim.x) {
    const bool cand = u < n_units && !s_sink[u];
    s_key[u] = cand ? desc_key(sc[u]) : ~0ull;
    s_idx[u] = u;
    if (u < n_units && s_sink[u]) atomicAdd(&s_nsb, 1);
  }
  __syncthreads();
  for (int k = 2; k <= n2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n2; i += blockDim.x) {
        const int l = i ^ j;
        if (l > i) {
          const uint64_t ki = s_key[i], kl = s_key[l];
          const int ii = s_idx[i], il = s_idx[l];
          const bool i_after = ki > kl || (ki == kl && ii > il);
          if (((i & k) == 0) == i_after) {
            s_key[i] = kl; s_key[l] = ki;
            s_idx[i] = il; s_idx[l] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
  const int n_cand = n_units - s_nsb;
  const int take = topK < n_cand ? topK : n_cand;
  for (int t = threadIdx.x; t < take; t += blockDim.x) s_keep[s_idx[t]] = 1;
  __syncthreads();
  int32_t* out = blk_idx + (size_t)bg * max_sel;
  for (int u0 = 0; u0 < n_units; u0 += blockDim.x) {
    const int u = u0 + threadIdx.x;
    const bool keep = u < n_units && (s_keep[u] || s_sink[u]);
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

__global__ void __launch_bounds__(kSelThreads)
select_kernel(const double* __restrict__ score, int H_kv, int n_units, int unit_size, int topK,
              const int32_t* __restrict__ sink_pos, int n_sinks, int32_t* __restrict__ blk_idx,
              int32_t* __restrict__ blk_cnt, int max_sel, unsigned* err) {
  pdl_trigger();
  pdl_wait();
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
  if (n_units <= kShflMax) {
    int n2 = 32;
    while (n2 < n_units) n2 <<= 1;
    DL_LAUNCH(select_shfl_kernel, batch * H_kv, n2, 0, st, score, H_kv, n_units, unit_size, topK,
                                                     sink_pos, n_sinks, blk_idx, blk_cnt, max_sel,
                                                     err);
    return cudaGetLastError();
  }
  if (n_units <= kBitonicMax) {
    int n2 = 2;
    while (n2 < n_units) n2 <<= 1;
    const size_t smem = (size_t)n2 * (sizeof(uint64_t) + sizeof(int) + 2);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(select_bitonic_kernel,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    const int threads = n2 / 2 < 32 ? 32 : (n2 / 2 > kSelThreads ? kSelThreads : n2 / 2);
    DL_LAUNCH(select_bitonic_kernel, batch * H_kv, threads, smem, st, 
        score, H_kv, n_units, n2, unit_size, topK, sink_pos, n_sinks, blk_idx, blk_cnt, max_sel,
        err);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)n_units * (sizeof(double) + 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  DL_LAUNCH(select_kernel, batch * H_kv, kSelThreads, smem, st, score, H_kv, n_units, unit_size, topK,
                                                         sink_pos, n_sinks, blk_idx, blk_cnt,
                                                         max_sel, err);
  return cudaGetLastError();
}

}  // namespace dl
