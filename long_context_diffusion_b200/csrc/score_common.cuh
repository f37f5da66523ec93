// Device helpers shared by the block-score kernels (scores.cu) and the fused
// score-and-select kernel (block_select.cu), and the selection order shared
// with select.cu.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace dl {

// D (8x8) += A (8x4, row-major) * B (4x8, column-major) in fp64.  Lane l
// holds A[l/4][l%4], B[l%4][l/4] and D[l/4][2(l%4) .. 2(l%4)+1].
__device__ __forceinline__ void dmma_m8n8k4(double (&d)[2], double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
      : "+d"(d[0]), "+d"(d[1])
      : "d"(a), "d"(b));
}

__device__ __forceinline__ float2 load_pair(const __nv_bfloat16* p) {
  return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
}
__device__ __forceinline__ float2 load_pair(const float* p) {
  return *reinterpret_cast<const float2*>(p);
}

// 16-byte global -> shared copy; zero-fills when !ok (src is then not read).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, bool ok) {
  const uint32_t sp = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(sp), "l"(src),
               "r"(ok ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Staged pooled keys: fp32 rows of D, the 16-byte chunk index XOR-ed with
// 4 * (row & 1) so that the float4 loads of two rows in one quarter-warp hit
// distinct banks.
__device__ __forceinline__ int key_chunk(int j, int chunk) { return chunk ^ ((j & 1) << 2); }

// Ascending order of the result equals descending order of x (IEEE bits made
// monotone, then inverted); the selection breaks ties by the lower index.
__device__ __forceinline__ uint64_t desc_key(double x) {
  const uint64_t b = static_cast<uint64_t>(__double_as_longlong(x));
  const uint64_t mono = (b >> 63) ? ~b : (b | 0x8000000000000000ull);
  return ~mono;
}

}  // namespace dl
