// (a4) Attention-sink mass on the sm_100a tensor cores (bf16 inputs).
//
// Focus-dLLM abstract: sinks are the highly influential attention columns,
// identified once and reused by deeper layers.  mass[b][t] = sum over every
// head h and predicted row i of exp(scale q_hi . k_t - LSE_hi), where LSE_hi
// is the row's log-sum-exp over the whole context plus the decode block.
//
// Pass 1 (the LSEs) is the tensor-core attention kernel in dense mode, in
// its LSE-only form where it has one (when the key-major kernel takes the
// shape: no V, no P V, no O), otherwise with V taken equal to K; it returns
// the natural-log LSE of every decode row.
//
// Pass 2 (this file) computes S^T = K Q^T with the keys as the MMA's M
// dimension: 128 keys (two pages) on the 128 TMEM lanes and the predicted
// rows of one KV group's heads as N (padded to a multiple of 16).  Thread t
// of the epilogue owns key t, so its mass is a sum over its own TMEM row --
// no cross-thread reduction.  One CTA owns a run of page pairs of one
// sequence and loops over the KV groups (outer) and its page pairs (inner),
// accumulating each key's mass in shared memory in group order, then writes
// it.  Roles: warp 0 = TMA producer, warp 1 = MMA issuer, warps 2-3 = gather
// the predicted Q rows (and their LSEs) of the next group, every lane with
// up to eight 16-byte loads in flight, warps 4-7 = epilogue.  Every wait is
// bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "sm100.cuh"
#include "launch.cuh"

namespace dl {

using namespace sm100;

constexpr int kMassMaxStages = 6;
constexpr int kMassMaxPairs = 64;  // page pairs per CTA

struct MassArgs {
  Shape s;
  const void* Q;          // [b][H][L_q][d]
  const int32_t* q_idx;   // [b][L_q]
  const int32_t* q_cnt;   // [b]
  const int32_t* page_table;
  const float* lse;       // natural log, [b][H][L_q]
  float* mass;            // [b][L_ctx]
  int n_pad;              // N of the MMA: G*L_q rounded up to 32
  int pairs_per_cta;
  int stages;             // K tiles in flight (2..6, as shared memory allows)
  unsigned* err;
};

template <int D>
struct MassCfg {
  static constexpr int HALVES = D / 64;
  static constexpr int KT_BYTES = HALVES * 128 * 128;  // [half][128 keys][128 B]
  __host__ __device__ static size_t q_bytes(int n_pad) { return (size_t)HALVES * n_pad * 128; }
  static size_t smem(int n_pad, int pairs, int stages) {
    return 1024 + 2 * q_bytes(n_pad) + (size_t)stages * KT_BYTES + 2 * 256 * 4 +
           (size_t)pairs * 128 * 4 + 64 * 8 + 64 + 256 * 4;
  }
};

template <int D>
__global__ void __launch_bounds__(256, 1)
sink_mass_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const MassArgs a) {
  using C = MassCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const Shape& s = a.s;
  const int n_pad = a.n_pad;
  const size_t QB = C::q_bytes(n_pad);
  uint8_t* sQ = smem;                               // [2][half][n_pad][128 B]
  uint8_t* sK = sQ + 2 * QB;                        // [stages][half][128][128 B]
  float* s_lse2 = reinterpret_cast<float*>(sK + a.stages * C::KT_BYTES);  // [2][256]
  float* s_mass = s_lse2 + 2 * 256;                 // [pairs*128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(s_mass + a.pairs_per_cta * 128);
  uint64_t* full = bars;                            // [stages]
  uint64_t* empty = full + kMassMaxStages;          // [stages]
  uint64_t* q_full = empty + kMassMaxStages;        // [2]  (32 arrivals)
  uint64_t* q_empty = q_full + 2;                   // [2]  (MMA commit + 128 epilogue)
  uint64_t* s_full = q_empty + 2;                   // [2]
  uint64_t* s_free = s_full + 2;                    // [2]  (128 epilogue)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s_free + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_qidx = reinterpret_cast<int*>(bars + 64) + 16;  // [L_q <= 256] predicted rows

  const int b = blockIdx.y;
  const int n_ctx_pages = (s.L_ctx + 63) / 64;
  const int n_pairs_all = (n_ctx_pages + 1) / 2;
  const int pp0 = blockIdx.x * a.pairs_per_cta;
  const int np = max(0, min(pp0 + a.pairs_per_cta, n_pairs_all) - pp0);
  const int n_tiles = np * s.H_kv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t tmem_cols = 2 * n_pad <= 32 ? 32 : 2 * n_pad <= 64 ? 64 : 2 * n_pad <= 128 ? 128
                             : 2 * n_pad <= 256 ? 256 : 512;
  // tensor memory first; the successor may be scheduled only after that
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
    pdl_trigger();
  }
  pdl_wait();
  const int nq = min(max(a.q_cnt[b], 0), s.L_q);
  const int Rg = nq * s.G;  // real rows per group

  if (threadIdx.x == 0) {
    for (int i = 0; i < a.stages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 64);
      mbar_init(&q_empty[i], 1 + 128);
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int e = threadIdx.x; e < np * 128; e += blockDim.x) s_mass[e] = 0.0f;
  for (int i = threadIdx.x; i < nq; i += blockDim.x) s_qidx[i] = a.q_idx[(size_t)b * s.L_q + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (n_tiles > 0 && warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int t = 0; t < n_tiles; ++t) {
        const int g = t / np, pp = t % np;
        const int st = t % a.stages;
        if (t >= a.stages && !mbar_wait(&empty[st], ((t / a.stages) - 1) & 1, abort_flag))
          break;
        int y[2], nload = 0;
        for (int q = 0; q < 2; ++q) {
          const int page = (pp0 + pp) * 2 + q;
          y[q] = -1;
          if (page < n_ctx_pages) {
            const int slot = a.page_table[(size_t)b * s.n_pages + page];
            if (slot >= 0 && slot < s.n_slots) {
              y[q] = (slot * s.H_kv + g) * 64;
              ++nload;
            } else {
              flag_error(a.err, ERR_BAD_INDEX);
            }
          }
        }
        if (nload == 0) {
          mbar_arrive(&full[st]);
          continue;
        }
        mbar_arrive_expect_tx(&full[st], nload * C::HALVES * 8192);
        uint8_t* dst = sK + st * C::KT_BYTES;
        for (int q = 0; q < 2; ++q) {
          if (y[q] < 0) continue;
          for (int h = 0; h < C::HALVES; ++h)
            tma_load_2d(dst + h * 16384 + q * 8192, &tm_k, h * 64, y[q], &full[st]);
        }
      }
    }
  } else if (n_tiles > 0 && warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, n_pad, false);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
      bool ok = true;
      for (int t = 0; ok && t < n_tiles; ++t) {
        const int g = t / np, pp = t % np;
        const int qb = g & 1, st = t % a.stages, buf = t & 1;
        if (pp == 0 && !(ok = mbar_wait(&q_full[qb], (g >> 1) & 1, abort_flag))) break;
        if (!(ok = mbar_wait(&full[st], (t / a.stages) & 1, abort_flag))) break;
        if (t >= 2 && !(ok = mbar_wait(&s_free[buf], ((t >> 1) - 1) & 1, abort_flag))) break;
        tc_fence_after();
        const uint32_t d_t = tmem + buf * n_pad;
#pragma unroll
        for (int k = 0; k < D / 16; ++k) {
          const int h = k >> 2, kk = k & 3;
          const uint64_t ad = sdesc_sw128(k_base + st * C::KT_BYTES + h * 16384 + kk * 32, 16, 1024);
          const uint64_t bd =
              sdesc_sw128(q_base + (uint32_t)(qb * QB + h * n_pad * 128) + kk * 32, 16, 1024);
          mma_f16_ss(d_t, ad, bd, idesc, k > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[buf]);
        mma_commit(&empty[st]);
        if (pp == np - 1) mma_commit(&q_empty[qb]);
      }
      if (*abort_flag)
        for (uint32_t k = 0; k < (1u << 16); ++k) __nanosleep(1000);
    }
  } else if (n_tiles > 0 && (warp == 2 || warp == 3)) {
    // ------------------------------------------------------------ Q gather
    constexpr int per_row = C::HALVES * 8;  // 16-byte chunks
    constexpr int IN_FLIGHT = 8;
    const float log2e = 1.4426950408889634f;
    const int gt = threadIdx.x - 64;  // 0..63
    const int total = n_pad * per_row;
    for (int g = 0; g < s.H_kv; ++g) {
      const int qb = g & 1;
      if (g >= 2) {
        const bool w = mbar_wait(&q_empty[qb], ((g >> 1) - 1) & 1, abort_flag);
        if (!__all_sync(0xffffffffu, w)) break;
      }
      uint8_t* dst = sQ + qb * QB;
      for (int e0 = 0; e0 < total; e0 += 64 * IN_FLIGHT) {
        uint4 v[IN_FLIGHT];
#pragma unroll
        for (int u = 0; u < IN_FLIGHT; ++u) {  // every load issued before any store
          const int e = e0 + u * 64 + gt;
          const int n = e / per_row, rem = e % per_row;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (e < total && n < Rg) {
            const int h = g * s.G + n / nq;
            const int i = s_qidx[n % nq];
            if (i >= 0 && i < s.L_q) {
              const __nv_bfloat16* src = reinterpret_cast<const __nv_bfloat16*>(a.Q) +
                                         (((size_t)b * s.H + h) * s.L_q + i) * D + rem * 8;
              v[u] = __ldg(reinterpret_cast<const uint4*>(src));
            }
          }
        }
#pragma unroll
        for (int u = 0; u < IN_FLIGHT; ++u) {
          const int e = e0 + u * 64 + gt;
          if (e >= total) continue;
          const int n = e / per_row, rem = e % per_row;
          const int h_half = rem >> 3, ch = rem & 7;
          *reinterpret_cast<uint4*>(dst + h_half * n_pad * 128 + n * 128 + ((ch ^ (n & 7)) << 4)) =
              v[u];
        }
      }
      for (int n = gt; n < n_pad; n += 64) {
        float l2 = INFINITY;  // padded rows contribute exp2(-inf) = 0
        if (n < Rg) {
          const int h = g * s.G + n / nq;
          const int i = s_qidx[n % nq];
          if (i >= 0 && i < s.L_q) l2 = a.lse[((size_t)b * s.H + h) * s.L_q + i] * log2e;
        }
        s_lse2[qb * 256 + n] = l2;
      }
      fence_proxy_async_smem();
      mbar_arrive(&q_full[qb]);
    }
  } else if (n_tiles > 0 && warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int key = quad * 32 + lane;  // TMEM lane = key within the page pair
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const float c2 = static_cast<float>(s.scale * 1.4426950408889634);
    bool ok = true;
    for (int t = 0; ok && t < n_tiles; ++t) {
      const int g = t / np, pp = t % np;
      const int qb = g & 1, buf = t & 1;
      if (pp == 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(&q_full[qb], (g >> 1) & 1, abort_flag));
        if (!ok) break;
      }
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (t >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      float acc = 0.0f;
      const float* l2 = s_lse2 + qb * 256;
      for (int c0 = 0; c0 < n_pad; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + lane_base + buf * n_pad + c0, v);
        tmem_ld_wait();
#pragma unroll
        for (int k = 0; k < 32; ++k)
          if (c0 + k < Rg) acc += ex2_approx(__uint_as_float(v[k]) * c2 - l2[c0 + k]);
      }
      tc_fence_before();
      mbar_arrive(&s_free[buf]);
      if (pp == np - 1) mbar_arrive(&q_empty[qb]);
      s_mass[pp * 128 + key] += acc;
    }
  }
  if (threadIdx.x == 0 && *abort_flag) flag_error(a.err, ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  // write the masses of this CTA's keys (page slots that were skipped read 0)
  for (int e = threadIdx.x; e < np * 128; e += blockDim.x) {
    const long long tpos = (long long)(pp0 * 2) * 64 + e;
    if (tpos < s.L_ctx) {
      const int page = (int)(tpos / 64);
      const int slot = a.page_table[(size_t)b * s.n_pages + page];
      a.mass[(size_t)b * s.L_ctx + tpos] = (slot >= 0 && slot < s.n_slots) ? s_mass[e] : 0.0f;
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Shared with attn_tc.cu: tensor maps and the SM count.
bool tc_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);
int tc_sm_count();

static int mass_n_pad(const Shape& s) { return ((s.G * s.L_q + 31) / 32) * 32; }

// Page pairs per CTA (about one CTA per SM over the batch) and K stages.
static void mass_plan(const Shape& s, int* pairs, int* stages, size_t* smem) {
  const int n_pairs = ((s.L_ctx + 63) / 64 + 1) / 2;
  int target = tc_sm_count() / s.batch;
  target = target < 1 ? 1 : target;
  int per = (n_pairs + target - 1) / target;
  per = per < 1 ? 1 : (per > kMassMaxPairs ? kMassMaxPairs : per);
  const int n_pad = mass_n_pad(s);
  int st = kMassMaxStages;
  for (; st > 2; --st) {
    const size_t need = s.d == 128 ? MassCfg<128>::smem(n_pad, per, st)
                                   : MassCfg<64>::smem(n_pad, per, st);
    if (need <= 232448) break;
  }
  *pairs = per;
  *stages = st;
  *smem = s.d == 128 ? MassCfg<128>::smem(n_pad, per, st) : MassCfg<64>::smem(n_pad, per, st);
}

cudaError_t launch_sink_mass_tc(const Shape& s, const void* Q, const int32_t* q_idx,
                                const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                                const float* lse, float* mass, unsigned* err, cudaStream_t st) {
  MassArgs a;
  a.s = s; a.Q = Q; a.q_idx = q_idx; a.q_cnt = q_cnt; a.page_table = page_table; a.lse = lse;
  a.mass = mass; a.err = err;
  a.n_pad = mass_n_pad(s);
  size_t smem = 0;
  mass_plan(s, &a.pairs_per_cta, &a.stages, &smem);
  if (smem > 232448) return cudaErrorInvalidValue;
  const int n_pairs = ((s.L_ctx + 63) / 64 + 1) / 2;
  const int n_cta = (n_pairs + a.pairs_per_cta - 1) / a.pairs_per_cta;
  CUtensorMap mk;
  if (!tc_map_2d(&mk, Kp, s.d, (uint64_t)s.n_slots * s.H_kv * 64, 64))
    return cudaErrorInvalidValue;
  cudaError_t e;
  if (s.d == 128) {
    e = cudaFuncSetAttribute(sink_mass_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    DL_LAUNCH(sink_mass_tc_kernel<128>, dim3(n_cta, s.batch), 256, smem, st, mk, a);
  } else {
    e = cudaFuncSetAttribute(sink_mass_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    DL_LAUNCH(sink_mass_tc_kernel<64>, dim3(n_cta, s.batch), 256, smem, st, mk, a);
  }
  return cudaGetLastError();
}

}  // namespace dl
