// (a6) Block-sparse bidirectional attention on the sm_100a tensor cores.
//
// Focus-dLLM abstract / summary: every decode-block query attends to the
// selected (sink-aware) context blocks and to the decode block itself, with
// no causal mask; shallow layers attend to every block.
//
// One CTA per (split, b, g).  Its tiles are 64-key pages: the selected
// context blocks (through the page table) and then the decode block.  Roles:
//   warp 0, one thread : TMA producer -- Q once, then K and V of each tile
//                        into a ring of ST shared-memory stages (128-byte
//                        swizzle; the pool is a 2-D tensor map of 64-row
//                        pages, so a gathered block is just a coordinate);
//   warp 1, one thread : tcgen05.mma issuer -- S = Q K^T into TMEM (two
//                        buffers), then O += P V into TMEM;
//   warps 4.. (128 per M-tile of 128 query rows): softmax -- one thread per
//                        query row reads its S row from TMEM, keeps a running
//                        max (lazy rescale: O and l are rescaled only when the
//                        max grows by more than 2^8) and sum, writes P (bf16)
//                        to shared memory in the MMA's K-major swizzled
//                        layout, and at the end writes its partial (O, m, l).
// The G*L_q query rows of a KV group are padded to M-tiles of 128 rows (the
// path is HBM-bound: padding costs tensor time, not bytes).  Partials of the
// splits of one (b, g) are merged by the combine kernel of attn_simt.cu.
//
// Every wait is bounded: a role that gives up raises the shared abort flag
// and the device error word (ERR_TIMEOUT) and leaves its loop; the CTA then
// frees its TMEM and returns.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "tiles.cuh"

namespace dl {

using namespace sm100;

constexpr int kTcMaxTiles = 1024;  // tiles of one CTA (tile table in shared memory)

template <int D, int NM, int ST, int PB>
struct TcCfg {
  static constexpr int HALVES = D / 64;                    // 128-byte column chunks
  static constexpr int Q_BYTES = NM * HALVES * 128 * 128;  // [m][half][128 rows][128 B]
  static constexpr int KT_BYTES = HALVES * 64 * 128;       // [half][64 rows][128 B]
  static constexpr int STAGE_BYTES = 2 * KT_BYTES;         // K tile, then V tile
  static constexpr int P_TILE = 128 * 128;                 // [128 rows][64 keys bf16]
  static constexpr int P_BYTES = PB * NM * P_TILE;
  static constexpr int BAR_OFF = Q_BYTES + ST * STAGE_BYTES + P_BYTES;
  static constexpr int N_BARS = 2 * ST + 1 + 2 + 2 + 2;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;
  static constexpr int TILE_OFF = MISC_OFF + 16;
  static constexpr int SMEM = TILE_OFF + 2 * kTcMaxTiles * 4 + 1024;  // + alignment slack
  static constexpr int THREADS = 128 + 128 * NM;
  static constexpr uint32_t TMEM_NEED = NM * D + 2 * NM * 64;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TMEM_NEED <= 512, "tensor memory budget");
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Block index of context tile `tile` of (b, g), or -1 (bad index, flagged).
__device__ __forceinline__ int ctx_tile_block(const AttnArgs& a, int bg, int tile) {
  if (a.mode == kDense) return tile;
  const int j = a.idx[(size_t)bg * a.max_idx + tile];
  if (j < 0 || j >= n_blocks(a.s)) {
    flag_error(a.err, ERR_BAD_INDEX);
    return -1;
  }
  return j;
}

template <int D, int NM, int ST, int PB>
__global__ void __launch_bounds__(128 + 128 * NM, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kd,
               const __grid_constant__ CUtensorMap tm_vd, const AttnArgs a, const int n_split,
               const int tps) {
  using C = TcCfg<D, NM, ST, PB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::Q_BYTES;
  uint8_t* sP = sKV + ST * C::STAGE_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty = full + ST;
  uint64_t* qbar = empty + ST;
  uint64_t* s_full = qbar + 1;     // [2]  S buffer written
  uint64_t* p_ready = s_full + 2;  // [2]  P written, O rescaled (128*NM arrivals)
  uint64_t* pv_done = p_ready + 2; // [PB] P V of the buffer's last tile done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  int* t_y = reinterpret_cast<int*>(smem + C::TILE_OFF);
  int* t_valid = t_y + kTcMaxTiles;

  const Shape& s = a.s;
  const int bg = blockIdx.y, sp = blockIdx.x;
  const int b = bg / s.H_kv, g = bg % s.H_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_ctx = ctx_tile_count(a, bg);
  const int n_tiles = n_ctx + (s.L_q + 63) / 64;
  const int t0 = sp * tps;
  const int nt = max(0, min(t0 + tps, n_tiles) - t0);
  const int R = s.G * s.L_q;

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(qbar, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128 * NM);
      mbar_init(&pv_done[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  // Tile table: TMA row coordinate and number of valid keys of every tile.
  for (int t = threadIdx.x; t < nt; t += blockDim.x) {
    const int tile = t0 + t;
    int y = 0, valid = 0;
    if (tile < n_ctx) {
      const int j = ctx_tile_block(a, bg, tile);
      if (j >= 0) {
        const int slot = a.page_table[(size_t)b * s.n_pages + j];
        if (slot < 0 || slot >= s.n_slots) {
          flag_error(a.err, ERR_BAD_INDEX);
        } else {
          valid = min(64, s.L_ctx - j * 64);
          y = (slot * s.H_kv + g) * 64;
        }
      }
    } else {
      const int td = tile - n_ctx;
      valid = min(64, s.L_q - td * 64);
      y = td * 64;
    }
    t_y[t] = y;
    t_valid[t] = valid;
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nt > 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(qbar, C::Q_BYTES);
      const int q_row0 = (b * s.H + g * s.G) * s.L_q;
      for (int m = 0; m < NM; ++m)
        for (int h = 0; h < C::HALVES; ++h)
          tma_load_2d(sQ + (m * C::HALVES + h) * 16384, &tm_q, h * 64, q_row0 + m * 128, qbar);
      for (int i = 0; i < nt; ++i) {
        const int st = i % ST;
        if (i >= ST && !mbar_wait(&empty[st], ((i / ST) - 1) & 1, abort_flag)) break;
        uint8_t* sK = sKV + st * C::STAGE_BYTES;
        uint8_t* sV = sK + C::KT_BYTES;
        if (t_valid[i] > 0) {
          mbar_arrive_expect_tx(&full[st], C::STAGE_BYTES);
          if (t0 + i < n_ctx) {
            for (int h = 0; h < C::HALVES; ++h) {
              tma_load_2d(sK + h * 8192, &tm_k, h * 64, t_y[i], &full[st]);
              tma_load_2d(sV + h * 8192, &tm_v, h * 64, t_y[i], &full[st]);
            }
          } else {
            for (int h = 0; h < C::HALVES; ++h) {
              tma_load_3d(sK + h * 8192, &tm_kd, h * 64, t_y[i], bg, &full[st]);
              tma_load_3d(sV + h * 8192, &tm_vd, h * 64, t_y[i], bg, &full[st]);
            }
          }
        } else {
          mbar_arrive(&full[st]);  // nothing to load: the tile is fully masked
        }
      }
      // do not leave with copies in flight: wait for the last stages' loads
      if (*abort_flag) {
        for (int i = max(0, nt - ST); i < nt; ++i)
          for (uint32_t k = 0; k < (1u << 20) && !mbar_try_wait(&full[i % ST], (i / ST) & 1); ++k) {
          }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && nt > 0) {
      constexpr uint32_t IS = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t IP = idesc_bf16_f32(128, D, true);
      const uint32_t q_base = smem_u32(sQ), kv_base = smem_u32(sKV), p_base = smem_u32(sP);
      bool ok = mbar_wait(qbar, 0, abort_flag);
      tc_fence_after();
      auto issue_s = [&](int i) -> bool {
        const int st = i % ST;
        if (!mbar_wait(&full[st], (i / ST) & 1, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kb = kv_base + st * C::STAGE_BYTES;
        const int buf = i & 1;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const uint32_t d_t = tmem + NM * D + (buf * NM + m) * 64;
#pragma unroll
          for (int k = 0; k < D / 16; ++k) {
            const int h = k >> 2, kk = k & 3;
            const uint64_t ad =
                sdesc_sw128(q_base + (m * C::HALVES + h) * 16384 + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kb + h * 8192 + kk * 32, 16, 1024);
            mma_f16_ss(d_t, ad, bd, IS, k > 0 ? 1u : 0u);
          }
        }
        mma_commit(&s_full[buf]);
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int i = 0; ok && i < nt; ++i) {
        if (i + 1 < nt && !issue_s(i + 1)) break;
        const int buf = i & 1;
        if (!mbar_wait(&p_ready[buf], (i >> 1) & 1, abort_flag)) break;
        tc_fence_after();
        const int st = i % ST;
        const uint32_t vb = kv_base + st * C::STAGE_BYTES + C::KT_BYTES;
        const int pbuf = PB == 2 ? buf : 0;
#pragma unroll
        for (int m = 0; m < NM; ++m) {
          const uint32_t d_t = tmem + m * D;
          const uint32_t pb = p_base + (pbuf * NM + m) * C::P_TILE;
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t ad = sdesc_sw128(pb + k * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(vb + k * 2048, 8192, 1024);
            mma_f16_ss(d_t, ad, bd, IP, (i > 0 || k > 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[st]);
        mma_commit(&pv_done[pbuf]);
      }
      if (*abort_flag) {  // give issued MMAs time to finish before TMEM is freed
        for (uint32_t k = 0; k < (1u << 16); ++k) __nanosleep(1000);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int m = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int r = m * 128 + row;
    const bool active = r < R;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = NM * D;
    const float c2 = static_cast<float>(s.scale * 1.4426950408889634);
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = nt > 0;
    // completion index of pv_done[x] for tile t is t / PB (PB buffers share tiles)
    auto wait_pv = [&](int t) -> bool {
      const bool w = mbar_wait(&pv_done[PB == 2 ? (t & 1) : 0], (PB == 2 ? (t >> 1) : t) & 1,
                               abort_flag);
      return __all_sync(0xffffffffu, w);
    };
    for (int i = 0; ok && i < nt; ++i) {
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (i >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[64];
      {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sv[32]);
        tmem_ld32(tmem + lane_base + s_col + (buf * NM + m) * 64, lo);
        tmem_ld32(tmem + lane_base + s_col + (buf * NM + m) * 64 + 32, hi);
        tmem_ld_wait();
      }
      const int valid = t_valid[i];
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const float x = (active && c < valid) ? __uint_as_float(sv[c]) * c2 : -INFINITY;
        sv[c] = __float_as_uint(x);
        tmax = fmaxf(tmax, x);
      }
      const float m_new = fmaxf(m_run, tmax);
      const bool grow = m_new > m_run + 8.0f;
      const bool live = grow && m_run != -INFINITY;  // an accumulator to rescale
      if (__any_sync(0xffffffffu, live)) {
        ok = wait_pv(i - 1);  // O holds every P V before tile i
        if (!ok) break;
        tc_fence_after();
        const float alpha = live ? exp2f(m_run - m_new) : 1.0f;
#pragma unroll 1
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_base + m * D + cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
          tmem_st32(tmem + lane_base + m * D + cc, o);
        }
        tmem_st_wait();
      }
      if (grow) {
        l_run = (m_run == -INFINITY) ? 0.0f : l_run * exp2f(m_run - m_new);
        m_run = m_new;
      }
      uint32_t packed[32];
      float psum = 0.0f;
#pragma unroll
      for (int c = 0; c < 64; c += 2) {
        const float x0 = __uint_as_float(sv[c]), x1 = __uint_as_float(sv[c + 1]);
        const float p0 = (m_run == -INFINITY) ? 0.0f : ex2_approx(x0 - m_run);
        const float p1 = (m_run == -INFINITY) ? 0.0f : ex2_approx(x1 - m_run);
        psum += p0 + p1;
        packed[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_run += psum;
      // the P buffer is free once the P V that last read it is done
      if (i >= PB) {
        ok = wait_pv(i - PB);
        if (!ok) break;
      }
      uint8_t* prow = sP + ((PB == 2 ? buf : 0) * NM + m) * C::P_TILE + row * 128;
#pragma unroll
      for (int ch = 0; ch < 8; ++ch) {
        *reinterpret_cast<uint4*>(prow + ((ch ^ (row & 7)) << 4)) =
            make_uint4(packed[4 * ch], packed[4 * ch + 1], packed[4 * ch + 2], packed[4 * ch + 3]);
      }
      if (m == 0 && valid < 64) {
        // rows past the valid keys may hold anything (even NaN): zero V there
        uint8_t* sV = sKV + (i % ST) * C::STAGE_BYTES + C::KT_BYTES;
        const int per_row = C::HALVES * 8;
        const int nz = (64 - valid) * per_row;
        for (int e = row; e < nz; e += 128) {
          const int rr = valid + e / per_row, rem = e % per_row;
          *reinterpret_cast<uint4*>(sV + (rem >> 3) * 8192 + rr * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[buf]);
    }
    // epilogue: unnormalised partial O, running max (natural log) and sum
    Partials part = partials_of(a.ws, s, n_split);
    const size_t prow = ((size_t)bg * n_split + sp) * R + r;
    if (ok) ok = wait_pv(nt - 1);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_base + m * D + cc, o);
        tmem_ld_wait();
        if (active) {
          float4* dst = reinterpret_cast<float4*>(part.o + prow * D + cc);
#pragma unroll
          for (int k = 0; k < 8; ++k)
            dst[k] = make_float4(__uint_as_float(o[4 * k]), __uint_as_float(o[4 * k + 1]),
                                 __uint_as_float(o[4 * k + 2]), __uint_as_float(o[4 * k + 3]));
        }
      }
    }
    if (active) {
      const bool any = ok && m_run != -INFINITY;
      part.ml[prow] = make_float2(any ? m_run * 0.69314718055994531f : -INFINITY,
                                  any ? l_run : 0.0f);
    }
  }
  if (threadIdx.x == 0 && *abort_flag) flag_error(a.err, ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------- host side
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
  static EncodeTiled fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiled>(p);
  });
  return fn;
}

}  // namespace

// bf16 rows of `inner` elements, boxes of 64 x box_rows, 128-byte swizzle.
bool tc_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiled fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// decode block K/V: [bg][L_q][d], boxes of 64 x 64 x 1 (rows past L_q read 0)
bool map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t L_q, uint64_t n_bg) {
  EncodeTiled fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, L_q, n_bg};
  cuuint64_t strides[2] = {inner * 2, L_q * inner * 2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int tc_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

namespace {

// Splits per (b, g): minimise waves x (tiles per CTA + fixed cost), one CTA
// per SM resident.
int tc_splits(int bgs, int max_tiles, int sms) {
  int best = 1;
  double best_cost = 1e30;
  for (int n = 1; n <= kMaxSplits && n <= max_tiles; ++n) {
    const int tps = (max_tiles + n - 1) / n;
    if (tps > kTcMaxTiles) continue;
    const long long ctas = (long long)bgs * n;
    const long long waves = (ctas + sms - 1) / sms;
    const double cost = (double)waves * (tps + 6.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = n;
    }
  }
  return best;
}

}  // namespace

cudaError_t launch_combine(const AttnArgs& a, int n_split, cudaStream_t st);

template <int D, int NM, int ST, int PB>
static cudaError_t run_tc(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  using C = TcCfg<D, NM, ST, PB>;
  const Shape& s = a.s;
  CUtensorMap mq, mk, mv, mkd, mvd;
  const uint64_t pool_rows = (uint64_t)s.n_slots * s.H_kv * 64;
  const uint64_t q_rows = (uint64_t)s.batch * s.H * s.L_q;
  const uint64_t n_bg = (uint64_t)s.batch * s.H_kv;
  if (!tc_map_2d(&mq, a.Q, D, q_rows, 128) || !tc_map_2d(&mk, a.Kp, D, pool_rows, 64) ||
      !tc_map_2d(&mv, a.Vp, D, pool_rows, 64) || !map_3d(&mkd, a.Kd, D, s.L_q, n_bg) ||
      !map_3d(&mvd, a.Vd, D, s.L_q, n_bg))
    return cudaErrorInvalidValue;
  const int n_split = tc_splits((int)n_bg, max_tiles, tc_sm_count());
  const int tps = (max_tiles + n_split - 1) / n_split;
  auto kern = attn_tc_kernel<D, NM, ST, PB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  kern<<<dim3(n_split, (unsigned)n_bg), C::THREADS, C::SMEM, st>>>(mq, mk, mv, mkd, mvd, a,
                                                                   n_split, tps);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_combine(a, n_split, st);
}

// Whether the tensor-core kernel takes this call (bf16, block or dense keys,
// at most two M-tiles of query rows, pool addressable by 32-bit TMA rows).
bool attn_tc_supported(const AttnArgs& a) {
  const Shape& s = a.s;
  return s.dtype == 0 && a.mode != kGather && s.G * s.L_q <= 256 &&
         (uint64_t)s.n_slots * s.H_kv * 64 < (1ull << 31) &&
         (uint64_t)s.batch * s.H * s.L_q < (1ull << 31);
}

cudaError_t launch_attn_tc(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  const Shape& s = a.s;
  const int nm = (s.G * s.L_q + 127) / 128;
  if (s.d == 128)
    return nm == 1 ? run_tc<128, 1, 4, 2>(a, max_tiles, st) : run_tc<128, 2, 3, 1>(a, max_tiles, st);
  return nm == 1 ? run_tc<64, 1, 6, 2>(a, max_tiles, st) : run_tc<64, 2, 4, 2>(a, max_tiles, st);
}

}  // namespace dl
