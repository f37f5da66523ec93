// (a3) Block scores: predicted query rows x mean-pooled keys, a softmax over
// blocks per row, summed over the rows (and over the query heads of a KV
// group).
//
// Focus-dLLM (research.elamur.ai summary): predicted queries select the most
// relevant KV blocks.  The score decides which block indices are kept, so it
// is computed in fp64: bf16 (or fp32) query x fp32 pooled-key products are
// exact in fp64 and the remaining rounding (~1e-16 relative) sits far below
// the spacing of neighbouring scores, so the kept set equals the one an
// exact computation gives.
//
// Two kernels.  (1) tile: grid (128-unit tiles, 32-row blocks, b*H_kv).
// Each warp owns 16 pooled keys and multiplies them with the block's query
// rows on the fp64 tensor-core MMA (m8n8k4; products of bf16 or fp32 inputs
// are exact in fp64).  The CTA then takes, per row, the max over its 128
// units, writes e = exp(l - m_tile) and records (m_tile, z_tile = sum e).
// (2) reduce: grid (128-unit tiles, b*H_kv).  Per row the tile statistics
// give M and Z and the tile's factor f = exp(m_tile - M) / Z, the row's
// softmax being e * f; four row groups then sum each column (rows g, g + 4,
// ... in order) and the four partial sums are added in group order.  This is
// the two-pass softmax of the definition with its max and sum taken tile by
// tile (online-softmax merging), equal to it up to fp64 rounding.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"
#include "score_common.cuh"

namespace dl {

constexpr int kWarps = 8;              // warps per tile CTA
constexpr int kNT = 2;                 // 8-unit MMA tiles per warp
constexpr int kUT = kWarps * kNT * 8;  // 128 units per CTA
constexpr int kRT = 32;                // query rows per pass (4 MMA row tiles)

__host__ __device__ inline int score_tiles(int n_units) { return (n_units + kUT - 1) / kUT; }

// Lane (gi = lane/4, t = lane%4) of warp w: pooled keys u_w + 8nt + gi as
// MMA B columns, query rows 8m + gi as A rows.  The four k-slots of one MMA
// step take, for k-group kg and step i, the model dimensions
// 16kg + 4t + i (t = the k-slot): A and B use the same assignment, so each
// dot product still runs over every dimension once.  The lane then reads its
// four dimensions as one float4 of the staged pooled key and two double2 of
// the staged query row.  The CTA's 128 pooled keys are copied to shared
// memory once (cp.async, overlapping the query staging); query rows are
// staged 32 at a time as fp64.
// Pooled keys: fp32 rows of D, the 16-byte chunk index XOR-ed with
// 4 * (row & 1) so that the float4 loads of two rows in one quarter-warp hit
// distinct banks.  Query rows: fp64, pitch D + 2 (rows 16 B apart mod 128).
// The rows as copied (bf16 or fp32) sit in the tail of the fp64 area and are
// converted through registers.
template <typename T, int D>
struct TileSmem {
  static constexpr int QP = D + 2;
  static constexpr int K_BYTES = kUT * D * 4;
  static constexpr int Q_BYTES = kRT * QP * 8;
  static constexpr int RAW_BYTES = kRT * D * (int)sizeof(T);
  static constexpr int RAW_OFF = K_BYTES + Q_BYTES - RAW_BYTES;
  static constexpr int BYTES = K_BYTES + Q_BYTES;
  static_assert(RAW_BYTES <= Q_BYTES && RAW_OFF % 16 == 0, "raw query rows inside the fp64 area");
};


template <typename T, int D>
__global__ void __launch_bounds__(kWarps * 32, 2)
scores_tile_kernel(const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                   const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar, Shape s,
                   int n_units, double* __restrict__ E, double2* __restrict__ stats,
                   unsigned* err) {
  pdl_trigger();
  pdl_wait();
  using L = TileSmem<T, D>;
  constexpr int KG = D / 16;               // k-groups of 16 dimensions
  constexpr int CPR = D * sizeof(T) / 16;  // 16-byte chunks per query row
  extern __shared__ __align__(16) uint8_t smem_s[];
  float* sK = reinterpret_cast<float*>(smem_s);                   // [kUT][D], swizzled
  double* sQ = reinterpret_cast<double*>(smem_s + L::K_BYTES);    // [kRT][QP]
  T* sRaw = reinterpret_cast<T*>(smem_s + L::RAW_OFF);            // [kRT][D]
  __shared__ double s_red[kWarps][kRT];
  __shared__ double s_row[kRT];
  const int bg = blockIdx.z;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int tile = blockIdx.x, n_tiles = gridDim.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gi = lane >> 2, t = lane & 3;
  const size_t pitch = (size_t)n_tiles * kUT;
  const int u_t = tile * kUT;
  const int u_w = u_t + warp * (kNT * 8);

  {  // the tile's pooled keys (zeros past the last unit), in flight from the start
    const float* src = Kbar + ((size_t)bg * n_units + u_t) * D;
    for (int c = threadIdx.x; c < kUT * (D / 4); c += blockDim.x) {
      const int j = c / (D / 4), col = (c % (D / 4)) * 4;
      const bool ok = u_t + j < n_units;
      cp_async16(sK + j * D + key_chunk(j, col >> 2) * 4, ok ? src + (size_t)j * D + col : Kbar,
                 ok);
    }
  }
  const int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  const int R = nq * s.G;
  const int R_max = s.L_q * s.G;
  const int r0 = blockIdx.y * kRT;  // this CTA's rows r0 .. r0 + kRT - 1
  if (r0 >= R) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;
  }
  {
    // query rows r0 .. r0+31 as copied (zeros past R or for a bad index)
    for (int c = threadIdx.x; c < kRT * CPR; c += blockDim.x) {
      const int rr = c / CPR, ch = c % CPR;
      const int r = r0 + rr;
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
      cp_async16(sRaw + rr * D + ch * (16 / sizeof(T)), src, ok);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    // to fp64 (the copied rows share the area: read all, sync, then write)
    constexpr int NP = kRT * (D / 2) / (kWarps * 32);
    float2 v[NP];
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int c = threadIdx.x + q * kWarps * 32;
      v[q] = load_pair(sRaw + (c / (D / 2)) * D + (c % (D / 2)) * 2);
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      const int c = threadIdx.x + q * kWarps * 32;
      *reinterpret_cast<double2*>(sQ + (c / (D / 2)) * L::QP + (c % (D / 2)) * 2) =
          make_double2(v[q].x, v[q].y);
    }
    __syncthreads();
    const int mt = min(kRT / 8, (R - r0 + 7) / 8);  // row tiles holding valid rows
    double acc[kRT / 8][kNT][2];
#pragma unroll
    for (int m = 0; m < kRT / 8; ++m)
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt) acc[m][nt][0] = acc[m][nt][1] = 0.0;
#pragma unroll 2
    for (int kg = 0; kg < KG; ++kg) {
      float4 bv[kNT];
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
        bv[nt] = *reinterpret_cast<const float4*>(
            sK + (warp * (kNT * 8) + nt * 8 + gi) * D + key_chunk(gi, 4 * kg + t) * 4);
      double a[kRT / 8][4];
#pragma unroll
      for (int m = 0; m < kRT / 8; ++m) {
        if (m < mt) {
          const double* qa = sQ + (8 * m + gi) * L::QP + 16 * kg + 4 * t;
          const double2 a01 = *reinterpret_cast<const double2*>(qa);
          const double2 a23 = *reinterpret_cast<const double2*>(qa + 2);
          a[m][0] = a01.x; a[m][1] = a01.y; a[m][2] = a23.x; a[m][3] = a23.y;
        }
      }
      // k-step outermost: the kRT/8 x kNT accumulator chains advance in turn.
#pragma unroll
      for (int i = 0; i < 4; ++i) {
#pragma unroll
        for (int m = 0; m < kRT / 8; ++m) {
          if (m < mt) {
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) {
              const float bk = i == 0 ? bv[nt].x : i == 1 ? bv[nt].y : i == 2 ? bv[nt].z : bv[nt].w;
              dmma_m8n8k4(acc[m][nt], a[m][i], (double)bk);
            }
          }
        }
      }
    }
    // Scale; units past the end take -inf so that they drop out of max and sum.
#pragma unroll
    for (int m = 0; m < kRT / 8; ++m)
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i)
          acc[m][nt][i] = u_w + nt * 8 + 2 * t + i < n_units ? acc[m][nt][i] * s.scale : -INFINITY;
    // Row max over the tile's 128 units: lanes t, then warps.
#pragma unroll
    for (int m = 0; m < kRT / 8; ++m) {
      double v = fmax(fmax(acc[m][0][0], acc[m][0][1]), fmax(acc[m][1][0], acc[m][1][1]));
      v = fmax(v, __shfl_xor_sync(0xffffffffu, v, 1));
      v = fmax(v, __shfl_xor_sync(0xffffffffu, v, 2));
      if (t == 0) s_red[warp][8 * m + gi] = v;
    }
    __syncthreads();
    if (threadIdx.x < kRT) {
      double v = s_red[0][threadIdx.x];
#pragma unroll
      for (int w = 1; w < kWarps; ++w) v = fmax(v, s_red[w][threadIdx.x]);
      s_row[threadIdx.x] = v;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < kRT / 8; ++m) {
      const int rr = 8 * m + gi;
      const double mx = s_row[rr];
      double z = 0.0;
#pragma unroll
      for (int nt = 0; nt < kNT; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          acc[m][nt][i] = m < mt ? exp(acc[m][nt][i] - mx) : 0.0;
          z += acc[m][nt][i];
        }
      z += __shfl_xor_sync(0xffffffffu, z, 1);
      z += __shfl_xor_sync(0xffffffffu, z, 2);
      if (t == 0) s_red[warp][rr] = z;
      if (r0 + rr < R) {
        double* row = E + ((size_t)bg * R_max + r0 + rr) * pitch + u_w + 2 * t;
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt)
          *reinterpret_cast<double2*>(row + nt * 8) = make_double2(acc[m][nt][0], acc[m][nt][1]);
      }
    }
    __syncthreads();
    if (threadIdx.x < kRT && r0 + threadIdx.x < R) {
      double z = 0.0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) z += s_red[w][threadIdx.x];
      stats[((size_t)bg * R_max + r0 + threadIdx.x) * n_tiles + tile] =
          make_double2(s_row[threadIdx.x], z);
    }
  }
}

// Grid (128-unit tiles, b*H_kv).  Thread per row (every row's statistics
// loaded at once): M = max of the tile maxima, Z = sum_t z_t exp(m_t - M)
// in tile order, and the factor of this CTA's tile
// f = exp(m_tile - M) / Z (dynamic shared memory, G * L_q doubles; the
// statistics are only read).
// Then thread = (row group rg, unit): the sum over the rows rg, rg + 4, ...
// in order of e[r][u] * f[r], and the four groups' sums added in order.
constexpr int kRedGroups = 4;

__global__ void __launch_bounds__(kRedGroups * kUT)
scores_reduce_kernel(const int32_t* __restrict__ q_idx, const int32_t* __restrict__ q_cnt,
                     Shape s, int n_units, const double* __restrict__ E,
                     const double2* __restrict__ stats, double* __restrict__ score) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ double s_f[];  // [G * L_q]
  __shared__ double s_part[kRedGroups][kUT];
  const int tile = blockIdx.x, bg = blockIdx.y;
  const int b = bg / s.H_kv;
  const int nq = q_idx ? min(max(q_cnt[b], 0), s.L_q) : s.L_q;
  const int R = nq * s.G;
  const int R_max = s.L_q * s.G;
  const int n_tiles = score_tiles(n_units);
  const size_t pitch = (size_t)n_tiles * kUT;
  const double2* st = stats + (size_t)bg * R_max * n_tiles;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    const double2* row = st + (size_t)r * n_tiles;
    double M = -INFINITY;
    for (int t = 0; t < n_tiles; ++t) M = fmax(M, row[t].x);
    double Z = 0.0;
    for (int t = 0; t < n_tiles; ++t) Z += row[t].y * exp(row[t].x - M);
    s_f[r] = exp(row[tile].x - M) / Z;
  }
  __syncthreads();
  const int rg = threadIdx.x / kUT, ul = threadIdx.x % kUT;
  const int u = tile * kUT + ul;
  const double* Eb = E + (size_t)bg * R_max * pitch + u;
  double acc = 0.0;
  int r = rg;
  for (; r + 8 * kRedGroups <= R; r += 8 * kRedGroups) {  // 8 loads in flight, sums in order
    double e[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) e[q] = Eb[(size_t)(r + q * kRedGroups) * pitch];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc += e[q] * s_f[r + q * kRedGroups];
  }
  for (; r < R; r += kRedGroups) acc += Eb[(size_t)r * pitch] * s_f[r];
  s_part[rg][ul] = acc;
  __syncthreads();
  if (rg == 0 && u < n_units) {
    double sc = s_part[0][ul];
#pragma unroll
    for (int q = 1; q < kRedGroups; ++q) sc += s_part[q][ul];
    score[(size_t)bg * n_units + u] = sc;
  }
}

static size_t scores_e_bytes(const Shape& s, int n_units) {
  return round256((size_t)s.batch * s.H_kv * s.G * s.L_q * (size_t)score_tiles(n_units) * kUT *
                  sizeof(double));
}

size_t scores_workspace(const Shape& s, int n_units) {
  return scores_e_bytes(s, n_units) +
         round256((size_t)s.batch * s.H_kv * s.G * s.L_q * (size_t)score_tiles(n_units) *
                  sizeof(double2));
}

cudaError_t launch_scores(const Shape& s, const void* Q, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, int n_units, double* score,
                          void* ws, unsigned* err, cudaStream_t st) {
  double* E = reinterpret_cast<double*>(ws);
  double2* stats =
      reinterpret_cast<double2*>(reinterpret_cast<char*>(ws) + scores_e_bytes(s, n_units));
  dim3 grid(score_tiles(n_units), (s.G * s.L_q + kRT - 1) / kRT, s.batch * s.H_kv);
  const dim3 block(kWarps * 32);
  cudaError_t e;
#define DL_TILE(T, D_)                                                                        \
  {                                                                                          \
    auto k = scores_tile_kernel<T, D_>;                                                      \
    constexpr int smem = TileSmem<T, D_>::BYTES;                                                \
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=  \
        cudaSuccess)                                                                         \
      return e;                                                                              \
    DL_LAUNCH(k, grid, block, smem, st, reinterpret_cast<const T*>(Q), q_idx, q_cnt, Kbar, s, n_units, \
                                 E, stats, err);                                             \
  }
  if (s.dtype == 0) {
    if (s.d == 128) DL_TILE(__nv_bfloat16, 128) else DL_TILE(__nv_bfloat16, 64)
  } else {
    if (s.d == 128) DL_TILE(float, 128) else DL_TILE(float, 64)
  }
#undef DL_TILE
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const size_t red_smem = (size_t)s.G * s.L_q * sizeof(double);
  if (red_smem > 48 * 1024 &&
      (e = cudaFuncSetAttribute(scores_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)red_smem)) != cudaSuccess)
    return e;
  DL_LAUNCH(scores_reduce_kernel, dim3(score_tiles(n_units), s.batch * s.H_kv), kRedGroups * kUT,
            red_smem, st, q_idx, q_cnt, s, n_units, E, stats, score);
  return cudaGetLastError();
}

}  // namespace dl
