// Allocation-free entry point for the block scores.
//
// dl_block_scores needs a scratch buffer for its fp64 logits, which the
// caller normally allocates and passes in as a workspace.  Some callers have
// no way to do that: a runtime that owns every device allocation and cannot
// hand out a workspace, code running where cudaMalloc is forbidden because it
// may synchronise the device (a latency-critical serving loop, a host
// callback), or a process that must not change its device-memory footprint
// after start-up.  dl_block_scores_noalloc serves them: its scratch is a
// fixed array compiled into this library, so the call allocates nothing.
//
// The array holds kScratchBytes (32 MiB) on every GPU that loads the library,
// until the process exits.  All calls on a device share it: the contents left
// by the previous call are kept, every cell the kernels read is written first
// in the same call, and two calls whose kernels overlap on the GPU (different
// streams without ordering) race on it.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
static __device__ __align__(256) double g_scores_scratch[kScratchBytes / sizeof(double)];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  The first
// call on a device looks it up (cudaGetSymbolAddress), so that first call
// should be made before any stream capture begins.
dl_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return dl::api_fail(DL_ERR_CUDA, "cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return dl::api_fail(DL_ERR_UNSUPPORTED, "device id too large");
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scores_scratch);
    if (e != cudaSuccess || p == nullptr)
      return dl::api_fail(DL_ERR_CUDA, "cudaGetSymbolAddress of the built-in scratch failed");
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return DL_OK;
}

}  // namespace

extern "C" dl_status dl_block_scores_noalloc(const dl_attn_desc* desc, const void* Q_dec,
                                             const int32_t* q_idx, const int32_t* q_cnt,
                                             const float* Kbar, int n_units, double* score,
                                             void* stream) {
  dl::Shape s;
  dl_status st = dl::api_check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !Kbar || !score || (q_idx && !q_cnt))
    return dl::api_fail(DL_ERR_INVALID_ARG, "dl_block_scores_noalloc: NULL pointer");
  if (n_units < 1 || n_units > (1 << 20))
    return dl::api_fail(DL_ERR_INVALID_ARG, "dl_block_scores_noalloc: n_units out of range");
  if (dl::scores_workspace(s, n_units) > kScratchBytes)
    return dl::api_fail(DL_ERR_WORKSPACE,
                        "dl_block_scores_noalloc: the block-score scratch for these sizes exceeds the "
                        "built-in 32 MiB scratch; use dl_block_scores with a workspace");
  void* scratch = nullptr;
  if ((st = scratch_address(&scratch)) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = dl::api_error_word(&err)) != DL_OK) return st;
  cudaError_t e = dl::launch_scores(s, Q_dec, q_idx, q_cnt, Kbar, n_units, score, scratch, err,
                                    reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return dl::api_fail(DL_ERR_CUDA, cudaGetErrorString(e));
  return dl::api_ok();
}
