// (a3 + a5) Block scores and selection in one kernel for groups of many
// query rows over few units: one CTA per (b, g).  The chunked prefix is the
// case it serves: every decode row of a head (64) against 32 chunk keys,
// top-8 chunks (Prefilling-dLLM abstract: top-K chunks by relevance).
//
// Same results as block_select.cu / scores.cu + select.cu:
//   l[r][u] = scale * q_r . Kbar_u,   score[u] = sum_r softmax_u(l[r][.]),
//   the sink units kept, then the topK other units of largest score (ties
//   to the lower index), ascending.
//
// With at most 128 units and R * n_units <= 8192 every logit of the (b, g)
// fits in shared memory.  A cluster of four CTAs takes one (b, g), each CTA a
// quarter of the rows (softmax rows are independent), in fp64:
//   stage   the group's query rows (gathered by q_idx) and its pooled keys by
//           cp.async, rows padded so that the fragment loads below hit 32
//           distinct banks;
//   dot     fp64 mma.sync m8n8k4 (the CUDA-core fp64 rate is a fraction of
//           the fp64 MMA rate on this part): warp item = 8 rows x 16 units,
//           four accumulators (two 8-unit tiles x even / odd 16-dimension
//           groups), added in a fixed order, so equal keys give equal
//           logits;
//   softmax warp per row: max, e^(l - max) in fp64, sum, divide;
//   scores  thread per unit sums its column over the CTA's rows in row
//           order; the first CTA of the cluster adds the four CTAs' sums in
//           CTA order (reading the others' shared memory);
//   select  that CTA: the bitonic sort and ascending write of the fused
//           kernels, on a network as wide as the units (32, 64 or 128).
// fp32 query values and fp32 pooled keys are exact in fp64 and their
// products too, so the logits carry only the rounding of the sums.
#include <cooperative_groups.h>

#include "block_select_common.cuh"
#include "launch.cuh"

namespace dl {

namespace bsw {
constexpr int kThreads = bs::kThreads;  // 512: the selection keeps one unit per thread
constexpr int kWarps = kThreads / 32;
constexpr int kMaxUnits = 128;
constexpr int kMaxRows = 256;
constexpr int kMaxCells = 8192;  // rows x units held as fp64 logits
constexpr int kCluster = 4;      // CTAs per (b, g), a quarter of the rows each
// rows of one CTA of the cluster: a multiple of the MMA's 8
__host__ __device__ inline int cta_rows(int R) { return ((R + kCluster - 1) / kCluster + 7) & ~7; }

template <typename T, int D>
struct Layout {
  // pitches: bf16 query rows D + 16 elements (288 B at D 128: 8 banks
  // apart, conflict-free 8-byte loads), fp32 rows D + 4 (2-way conflicts,
  // but 256 rows still fit), pooled keys D + 16 floats (16 banks apart)
  static constexpr int QP = D + (sizeof(T) == 2 ? 16 : 4);
  static constexpr int KP = D + 16;
  __host__ __device__ static int rows_cap(int R) { return (R + 7) & ~7; }
  __host__ __device__ static int units_cap(int U) { return (U + 31) & ~31; }
  __host__ __device__ static size_t q_bytes(int R) { return (size_t)rows_cap(R) * QP * sizeof(T); }
  __host__ __device__ static size_t k_bytes(int U) { return (size_t)units_cap(U) * KP * 4; }
  __host__ __device__ static size_t bytes(int R, int U) {
    return q_bytes(R) + k_bytes(U) + (size_t)rows_cap(R) * units_cap(U) * 8;
  }
};
constexpr size_t kSmemLimit = 232448 - sizeof(BsSelScratch);
}  // namespace bsw

template <typename T>
__device__ __forceinline__ void load4(const T* p, double (&v)[4]);
template <>
__device__ __forceinline__ void load4<__nv_bfloat16>(const __nv_bfloat16* p, double (&v)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
  v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
template <>
__device__ __forceinline__ void load4<float>(const float* p, double (&v)[4]) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}

template <typename T, int D>
__global__ void __cluster_dims__(bsw::kCluster, 1, 1) __launch_bounds__(bsw::kThreads, 1)
block_select_wide_kernel(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                         const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar,
                         Shape s, int n_units, int max_rows, double* __restrict__ score,
                         int unit_size, int topK, const int32_t* __restrict__ sink_pos,
                         int n_sinks, int32_t* __restrict__ blk_idx,
                         int32_t* __restrict__ blk_cnt, int max_sel, unsigned* err) {
  using namespace bsw;
  using L = Layout<T, D>;
  pdl_trigger();
  pdl_wait();
  extern __shared__ __align__(16) uint8_t smem_b[];
  __shared__ BsSelScratch s_sel;
  __shared__ double s_part[kMaxUnits];  // this CTA's column sums
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();

  const int bg = blockIdx.x / kCluster;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = n_units, Uc = L::units_cap(U);

  // query rows: every predicted position of every query head of the group
  int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  if (nq * s.G > max_rows) {  // more rows than the caller's bound: reported, rows cut
    if (tid == 0) flag_error(err, ERR_BAD_INDEX);
    nq = max_rows / s.G;
  }
  const int R_all = nq * s.G;
  const int r_lo = rank * cta_rows(R_all);                 // this CTA's rows r_lo ..
  const int R = max(0, min(R_all - r_lo, cta_rows(R_all)));  // .. r_lo + R - 1
  const int cap = cta_rows(max_rows);
  T* sQ = reinterpret_cast<T*>(smem_b);                              // [Rc][QP]
  float* sK = reinterpret_cast<float*>(smem_b + L::q_bytes(cap));    // [Uc][KP]
  double* sL = reinterpret_cast<double*>(smem_b + L::q_bytes(cap) + L::k_bytes(U));  // [Rc][Uc]

  constexpr int QCH = D * (int)sizeof(T) / 16;  // 16-byte chunks per query row
  constexpr int QE = 16 / (int)sizeof(T);       // elements per chunk
  for (int c = tid; c < L::rows_cap(R) * QCH; c += kThreads) {
    const int r = c / QCH, ch = c % QCH;
    const T* src = Q;
    bool ok = false;
    if (r < R) {
      const int h = g * s.G + (r_lo + r) / nq;
      const int i = q_idx ? q_idx[(size_t)b * s.L_q + ((r_lo + r) % nq)] : ((r_lo + r) % nq);
      if (i >= 0 && i < s.L_q) {
        src = Q + (((size_t)b * s.H + h) * s.L_q + i) * D + ch * QE;
        ok = true;
      } else if (ch == 0) {
        flag_error(err, ERR_BAD_INDEX);
      }
    }
    cp_async16(sQ + (size_t)r * L::QP + ch * QE, src, ok);
  }
  constexpr int KCH = D / 4;  // 16-byte chunks per pooled key
  const float* kb = Kbar + (size_t)bg * U * D;
  for (int c = tid; c < Uc * KCH; c += kThreads) {
    const int u = c / KCH, ch = c % KCH;
    const bool ok = u < U;
    cp_async16(sK + u * L::KP + ch * 4, ok ? kb + (size_t)u * D + ch * 4 : Kbar, ok);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  // ---- logits on the fp64 MMA: item = (8-row tile, two 8-unit tiles).  In
  // m8n8k4 lane (gi, t) gives A[gi][t] and B[t][gi] and holds C[gi][2t, 2t+1];
  // k-step i of 16-dimension group kg takes dimension 16 kg + 4 t + i, so a
  // lane reads four consecutive dimensions of its row and of its unit.
  const double sc = s.scale;
  const int gi = lane >> 2, t4 = lane & 3;
  const int n_mt = L::rows_cap(R) >> 3, n_np = Uc >> 4;
  for (int it = warp; it < n_mt * n_np; it += kWarps) {
    const int r0 = (it / n_np) * 8, u0 = (it % n_np) * 16;
    const T* qr = sQ + (size_t)(r0 + gi) * L::QP + 4 * t4;
    const float* k0 = sK + (u0 + gi) * L::KP + 4 * t4;
    const float* k1 = k0 + 8 * L::KP;
    double acc[2][2][2];  // [unit tile][kg parity][C element]
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
      for (int p = 0; p < 2; ++p) acc[a][p][0] = acc[a][p][1] = 0.0;
#pragma unroll 4
    for (int kg = 0; kg < D / 16; ++kg) {
      double q[4];
      load4<T>(qr + 16 * kg, q);
      const float4 b0 = *reinterpret_cast<const float4*>(k0 + 16 * kg);
      const float4 b1 = *reinterpret_cast<const float4*>(k1 + 16 * kg);
      const int p = kg & 1;
      dmma_m8n8k4(acc[0][p], q[0], (double)b0.x);
      dmma_m8n8k4(acc[1][p], q[0], (double)b1.x);
      dmma_m8n8k4(acc[0][p], q[1], (double)b0.y);
      dmma_m8n8k4(acc[1][p], q[1], (double)b1.y);
      dmma_m8n8k4(acc[0][p], q[2], (double)b0.z);
      dmma_m8n8k4(acc[1][p], q[2], (double)b1.z);
      dmma_m8n8k4(acc[0][p], q[3], (double)b0.w);
      dmma_m8n8k4(acc[1][p], q[3], (double)b1.w);
    }
    double* lr = sL + (size_t)(r0 + gi) * Uc + u0 + 2 * t4;
#pragma unroll
    for (int a = 0; a < 2; ++a) {
      lr[8 * a] = (acc[a][0][0] + acc[a][1][0]) * sc;
      lr[8 * a + 1] = (acc[a][0][1] + acc[a][1][1]) * sc;
    }
  }
  __syncthreads();

  // ---- softmax over the units of each row (padding units excluded)
  for (int r = warp; r < R; r += kWarps) {
    double* lr = sL + (size_t)r * Uc;
    double m = -INFINITY;
    for (int u = lane; u < U; u += 32) m = fmax(m, lr[u]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
    double z = 0.0;
    for (int u = lane; u < U; u += 32) {
      const double e = exp(lr[u] - m);
      lr[u] = e;
      z += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    const double iz = 1.0 / z;
    for (int u = lane; u < U; u += 32) lr[u] *= iz;
  }
  __syncthreads();

  // ---- column sums over this CTA's rows in row order; the first CTA adds the
  // four CTAs' sums in CTA order and selects
  if (tid < kMaxUnits) {
    double my = 0.0;
    if (tid < U)
      for (int r = 0; r < R; ++r) my += sL[(size_t)r * Uc + tid];
    s_part[tid] = my;
  }
  cluster.sync();  // every CTA's sums are in its shared memory
  double col = 0.0;
  if (rank == 0 && tid < U) {
#pragma unroll
    for (int q = 0; q < kCluster; ++q) col += *cluster.map_shared_rank(&s_part[tid], q);
    score[(size_t)bg * U + tid] = col;
  }
  cluster.sync();  // the others' shared memory stays until it has been read
  if (rank != 0) return;
  const BsSorted srt =
      U <= 32   ? bs_sort<32>(col, U, b, unit_size, sink_pos, n_sinks, s_sel, err)
      : U <= 64 ? bs_sort<64>(col, U, b, unit_size, sink_pos, n_sinks, s_sel, err)
                : bs_sort<128>(col, U, b, unit_size, sink_pos, n_sinks, s_sel, err);
  bs_write(srt, U, topK, bg, blk_idx, blk_cnt, max_sel, s_sel);
}

bool block_select_wide_supported(const Shape& s, int rows, int n_units) {
  if (n_units < 1 || n_units > bsw::kMaxUnits || rows < 1 || rows > bsw::kMaxRows) return false;
  if ((size_t)bsw::Layout<float, 128>::rows_cap(rows) * bsw::Layout<float, 128>::units_cap(n_units) >
      (size_t)bsw::kMaxCells)
    return false;
  if (s.d != 64 && s.d != 128) return false;
  const int cap = bsw::cta_rows(rows);
  const size_t bytes =
      s.dtype == 0 ? (s.d == 128 ? bsw::Layout<__nv_bfloat16, 128>::bytes(cap, n_units)
                                 : bsw::Layout<__nv_bfloat16, 64>::bytes(cap, n_units))
                   : (s.d == 128 ? bsw::Layout<float, 128>::bytes(cap, n_units)
                                 : bsw::Layout<float, 64>::bytes(cap, n_units));
  return bytes <= bsw::kSmemLimit;
}

cudaError_t launch_block_select_wide(const Shape& s, const void* Q, const int32_t* q_idx,
                                     const int32_t* q_cnt, const float* Kbar, int n_units,
                                     double* score, int unit_size, int topK,
                                     const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                                     int32_t* blk_cnt, int max_sel, int rows, unsigned* err,
                                     cudaStream_t st) {
  cudaError_t e;
#define DL_BSW(T, D_)                                                                           \
  {                                                                                            \
    auto k = block_select_wide_kernel<T, D_>;                                                  \
    const size_t smem = bsw::Layout<T, D_>::bytes(bsw::cta_rows(rows), n_units);               \
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != \
        cudaSuccess)                                                                           \
      return e;                                                                                \
    DL_LAUNCH(k, s.batch * s.H_kv * bsw::kCluster, bsw::kThreads, smem, st,                      \
              reinterpret_cast<const T*>(Q), q_idx,                                            \
              q_cnt, Kbar, s, n_units, rows, score, unit_size, topK, sink_pos, n_sinks, blk_idx, \
              blk_cnt, max_sel, err);                                                          \
  }
  if (s.dtype == 0) {
    if (s.d == 128) DL_BSW(__nv_bfloat16, 128) else DL_BSW(__nv_bfloat16, 64)
  } else {
    if (s.d == 128) DL_BSW(float, 128) else DL_BSW(float, 64)
  }
#undef DL_BSW
  return cudaGetLastError();
}

}  // namespace dl
