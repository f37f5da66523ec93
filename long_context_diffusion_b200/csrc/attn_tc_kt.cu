// (a6) Block-sparse bidirectional attention on the sm_100a tensor cores,
// keys on the MMA's M side ("key-major"), for head dim 128 and at most 32
// query rows per KV group.
//
// Focus-dLLM abstract / summary: every decode-block query attends to the
// selected (sink-aware) context blocks and to the decode block itself, with
// no causal mask; shallow layers attend to every block.
//
// With a 32-token decode block and one query head per KV head, the rows of a
// KV group are far fewer than the 128 of an MMA tile.  This kernel therefore
// computes the transposed products, so that the 128-wide side of every MMA
// is a dimension that really has 128 entries:
//   S^T [128 keys x 32 rows] = K_step [128 keys x d] . Q^T      (A = K, B = Q)
//   O^T [d x 32 rows]       += V_step^T [d x 128 keys] . P^T   (A = V^T, B = P^T)
// A step is two 64-key pages (one when a segment's run is odd).  S^T and O^T
// live in TMEM (32 columns each, two buffers of each); P^T goes to shared
// memory in the 128-byte-swizzled layout of an MN-major B operand.
//
// Softmax (4 warps, thread = TMEM lane = key of the step for S^T, model
// dimension for O^T): every thread keeps the same reference maximum per
// query row, m_ref[q].  A step whose scores all stay below m_ref + 8 (log2
// units) uses it as is: p = 2^(s - m_ref) <= 256, so P (bf16), l and O (fp32)
// stay in range.  Otherwise (always on a segment's first step) the four
// warps take the step's maximum per row (a transposing butterfly over the
// lanes, then shared memory), raise m_ref, and rescale O^T's columns and
// their own partial sums.  Each thread sums p over its own keys; the sums
// over the 128 lanes are taken once per segment, in the epilogue.  This is
// the online softmax of flash attention with the row maximum replaced by a
// shared reference that is only ever raised: the result is the same
// normalised sum.
//
// Roles: warp 0 one thread: TMA of Q (per segment) and of the K ring;
// warp 2 one thread: the V ring; warp 1 one thread: S^T MMAs; warp 3 one
// thread: O^T MMAs; warps 4..7: softmax.  Work is split over the SMs in tile
// slots exactly as in attn_tc.cu; partials go to the same combine kernel.
// (Merging inside this kernel, by the CTA whose partial completes a (b, g),
// measured slower: the merges land on the last CTAs, at the tail.)
// Every wait is bounded and the softmax warps exchange through mbarriers (no
// named barriers), so a role that gives up cannot leave another waiting.
// With O == nullptr only the row LSEs are produced (the first pass of the
// sink search): the V ring, the O^T MMAs and all O work are skipped.  (Also
// skipping the rows that are not predicted measured no faster: the pass is
// not bound by its exponentials.)
#include <mutex>

#include "sm100.cuh"
#include "tc_common.cuh"
#include "launch.cuh"

namespace dl {

using namespace sm100;

namespace kt {

constexpr int D = 128;
constexpr int NQ = 32;                     // query rows (MMA N)
constexpr int QB = 2;                      // Q buffers (alternating segments)
constexpr int Q_BYTES = 2 * NQ * 128;      // [d-half][32 rows][128 B]
constexpr int KS_BYTES = 2 * 128 * 128;    // [d-half][128 keys][128 B]
constexpr int PT_BYTES = 128 * 128;        // [128 keys][128 B] (64 B used)
constexpr int MAX_STEPS = kTcMaxTiles / 2 + kMaxSegs;
constexpr int THREADS = 256;
constexpr uint32_t TMEM_COLS = 128;  // S^T [2][32] at 0, O^T [2][32] at 64
constexpr uint32_t S_COL = 0, O_COL = 64;

// Shared-memory layout.  Attention: a K ring of three two-page stages and a V
// ring of two (a third V stage measured slower), two P^T tiles.  LSE-only
// (the first pass of the sink search): no V, no P^T, so six K stages.
template <bool LSE>
struct Layout {
  static constexpr int STK = LSE ? 6 : 3;
  static constexpr int STV = LSE ? 0 : 2;
  static constexpr int NPT = LSE ? 0 : 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + QB * Q_BYTES;
  static constexpr int V_OFF = K_OFF + STK * KS_BYTES;
  static constexpr int PT_OFF = V_OFF + STV * KS_BYTES;
  static constexpr int RED_OFF = PT_OFF + NPT * PT_BYTES;   // float [4][32] maxima, [4][32] sums
  static constexpr int FLAG_OFF = RED_OFF + 2 * 4 * NQ * 4;  // int [2][4] rescale votes
  static constexpr int BAR_OFF = FLAG_OFF + 2 * 4 * 4;
  // full_k, empty_k [STK]; full_v, empty_v [STV]; q_full, q_free, s_full,
  // p_ready, pv_done, o_free, xbar [2]; mxbar, lbar
  static constexpr int N_BARS = 2 * STK + 2 * STV + 7 * 2 + 2;
  static constexpr int MISC_OFF = (BAR_OFF + N_BARS * 8 + 15) / 16 * 16;
  static constexpr int STEP_OFF = MISC_OFF + 32;                  // int4 [MAX_STEPS]
  static constexpr int SEG_OFF = STEP_OFF + MAX_STEPS * 16;       // int4 [kMaxSegs]
  static constexpr int MARK_OFF = SEG_OFF + kMaxSegs * 16;        // int2 [kMaxSegs]
  static constexpr int SEGHI_OFF = MARK_OFF + kMaxSegs * 8;       // int [kMaxSegs]
  static constexpr int NCTX_OFF = SEGHI_OFF + kMaxSegs * 4;       // int [kMaxSegs]
  static constexpr int SMEM = NCTX_OFF + kMaxSegs * 4 + 1024;     // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(BAR_OFF % 16 == 0 && STEP_OFF % 16 == 0 && SEG_OFF % 16 == 0, "alignment");
};

// After the call, lane L holds op over the 32 lanes of v[L] (v is clobbered):
// a butterfly in which each level keeps half of the entries and trades the
// other half with the partner lane.
template <bool MAX>
__device__ __forceinline__ float xreduce32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

// step entry: (y of page 0, y of page 1, info0 | seg << 16, info1), info =
// valid keys (0..64) | decode flag << 15
__device__ __forceinline__ int step_seg(const int4& e) { return e.z >> 16; }
__device__ __forceinline__ int page_valid(int info) { return info & 0x7F; }
__device__ __forceinline__ bool page_dec(int info) { return (info >> 15) & 1; }

}  // namespace kt

template <bool LSE>
__global__ void __launch_bounds__(kt::THREADS, 1)
attn_tc_kt_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v,
                  const __grid_constant__ CUtensorMap tm_kd,
                  const __grid_constant__ CUtensorMap tm_vd, const AttnArgs a, const TcPlan plan) {
  using namespace kt;
  using Lk = Layout<LSE>;
  constexpr int STK = Lk::STK, STV = Lk::STV;
  constexpr int STVd = STV > 0 ? STV : 1;  // divisor in the (LSE-unreachable) V paths
  constexpr int Q_OFF = Lk::Q_OFF, K_OFF = Lk::K_OFF, V_OFF = Lk::V_OFF, PT_OFF = Lk::PT_OFF;
  constexpr int RED_OFF = Lk::RED_OFF, FLAG_OFF = Lk::FLAG_OFF, BAR_OFF = Lk::BAR_OFF;
  constexpr int MISC_OFF = Lk::MISC_OFF, STEP_OFF = Lk::STEP_OFF, SEG_OFF = Lk::SEG_OFF;
  constexpr int MARK_OFF = Lk::MARK_OFF, SEGHI_OFF = Lk::SEGHI_OFF, NCTX_OFF = Lk::NCTX_OFF;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + Q_OFF;
  uint8_t* sK = smem + K_OFF;
  uint8_t* sV = smem + V_OFF;
  uint8_t* sPT = smem + PT_OFF;
  float* s_max = reinterpret_cast<float*>(smem + RED_OFF);  // [4][32]
  float* s_sum = s_max + 4 * NQ;                            // [4][32]
  int* s_vote = reinterpret_cast<int*>(smem + FLAG_OFF);    // [2][4]
  uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint64_t* empty_k = full_k + STK;
  uint64_t* full_v = empty_k + STK;
  uint64_t* empty_v = full_v + STV;
  uint64_t* q_full = empty_v + STV;  // [2] Q of a segment landed
  uint64_t* q_free = q_full + 2;    // [2] every S^T of a segment done
  uint64_t* s_full = q_free + 2;    // [2] S^T buffer written
  uint64_t* p_ready = s_full + 2;   // [2] P^T written (and O^T rescaled)
  uint64_t* pv_done = p_ready + 2;  // [2] O^T += V^T P^T of that parity done
  uint64_t* o_free = pv_done + 2;   // [2] segment's O^T read out
  uint64_t* xbar = o_free + 2;      // [2] rescale vote, per step parity
  uint64_t* mxbar = xbar + 2;       // step maxima exchanged
  uint64_t* lbar = mxbar + 1;       // segment sums exchanged
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + MISC_OFF + 4);
  int* s_nstep = reinterpret_cast<int*>(smem + MISC_OFF + 8);
  int* s_nseg = s_nstep + 1;
  int* s_nmark = s_nstep + 2;
  int4* steps = reinterpret_cast<int4*>(smem + STEP_OFF);
  int4* seg = reinterpret_cast<int4*>(smem + SEG_OFF);    // (bg, slot, first step, lo tile)
  int2* mark = reinterpret_cast<int2*>(smem + MARK_OFF);  // (bg, slot) of empty runs
  int* seg_hi = reinterpret_cast<int*>(smem + SEGHI_OFF);  // end tile (exclusive)
  int* s_nctx = reinterpret_cast<int*>(smem + NCTX_OFF);   // context tiles of each (b, g) in range

  const Shape& s = a.s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool lse_only = LSE;  // row LSEs only: no V, no P V, no O
  // tensor memory first; the successor may be scheduled only after that
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
    pdl_trigger();
  }
  pdl_wait();
  const int R = s.G * s.L_q;
  const int n_dec = (s.L_q + 63) / 64;
  const long long U = (long long)s.batch * s.H_kv * plan.S;
  const long long u0 = (long long)blockIdx.x * U / gridDim.x;
  const long long u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
  Partials part = partials_of(a.ws, s, plan.nslot);

  // the (b, g) pairs this CTA's slots touch, their tile counts in parallel
  const int bg_lo = u1 > u0 ? (int)(u0 / plan.S) : 0;
  const int nb = u1 > u0 ? (int)((u1 - 1) / plan.S) - bg_lo + 1 : 0;  // <= kMaxSegs (plan)
  if (threadIdx.x < nb) s_nctx[threadIdx.x] = ctx_tile_count(a, bg_lo + threadIdx.x);
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2 * (STK + STV); ++i) mbar_init(&full_k[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], 128);
      mbar_init(&pv_done[i], 1);
      mbar_init(&o_free[i], 128);
      mbar_init(&xbar[i], 4);
    }
    mbar_init(mxbar, 4);
    mbar_init(lbar, 4);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // the V ring starts zeroed: the keys of a missing second page are masked
  // (p = 0), and 0 * (stale but finite) V = 0
  for (int e = threadIdx.x; e < STV * KS_BYTES / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(sV)[e] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();  // before TMA writes the same bytes
  __syncthreads();
  if (threadIdx.x == 0) {
    int nseg = 0, nmark = 0, nstep = 0;
    for (int i = 0; i < nb; ++i) {
      const int bg = bg_lo + i;
      const long long base = (long long)bg * plan.S;
      const int lo = (int)max(u0 - base, 0ll);
      const int hi = (int)min(u1 - base, (long long)plan.S);
      const int thi = min(hi, s_nctx[i] + n_dec);
      const int slot = (int)blockIdx.x - tc_owner(base, U, gridDim.x);
      if (thi > lo) {
        seg[nseg] = make_int4(bg, slot, nstep, lo);
        seg_hi[nseg] = thi;
        ++nseg;
        nstep += (thi - lo + 1) / 2;
      } else {
        mark[nmark++] = make_int2(bg, slot);
      }
    }
    *s_nstep = nstep;
    *s_nseg = nseg;
    *s_nmark = nmark;
  }
  __syncthreads();
  const int nst = *s_nstep, nseg = *s_nseg, nmark = *s_nmark;
  for (int e = threadIdx.x; e < nmark * R; e += blockDim.x) {
    const int2 mk = mark[e / R];
    part.ml[((size_t)mk.x * plan.nslot + mk.y) * R + e % R] = make_float2(-INFINITY, 0.0f);
  }
  // step table, every entry in parallel: step t of segment k holds tiles
  // lo + 2(t - first) and (if below the segment's end) the next one
  for (int t = threadIdx.x; t < nst; t += blockDim.x) {
    int k = 0;
    while (k + 1 < nseg && seg[k + 1].z <= t) ++k;
    const int bg = seg[k].x;
    const int n_ctx = s_nctx[bg - bg_lo];
    const int tile = seg[k].w + 2 * (t - seg[k].z);
    const int2 p0 = tc_tile_info(a, bg, tile, n_ctx);
    const int2 p1 = tile + 1 < seg_hi[k] ? tc_tile_info(a, bg, tile + 1, n_ctx) : make_int2(0, 0);
    steps[t] = make_int4(p0.x, p1.x, p0.y | (k << 16), p1.y);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto first_of = [&](int j) { return j == 0 || step_seg(steps[j - 1]) != step_seg(steps[j]); };
  auto last_of = [&](int j) { return j == nst - 1 || step_seg(steps[j + 1]) != step_seg(steps[j]); };

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    const bool is_k = warp == 0;
    uint64_t* full = is_k ? full_k : full_v;
    uint64_t* empty = is_k ? empty_k : empty_v;
    uint8_t* ring = is_k ? sK : sV;
    const CUtensorMap* map = is_k ? &tm_k : &tm_v;
    const CUtensorMap* map_dec = is_k ? &tm_kd : &tm_vd;
    const int ST = is_k ? STK : STVd;
    if (lane == 0 && nst > 0 && (is_k || !lse_only)) {
      prefetch_tmap(map);
      prefetch_tmap(map_dec);
      int next_q = 0;
      bool ok = true;
      for (int j = 0; ok && j < nst; ++j) {
        const int4 e = steps[j];
        const int k = step_seg(e);
        while (is_k && ok && next_q < nseg && next_q <= k) {
          const int qb = next_q & 1;
          if (next_q >= QB &&
              !(ok = mbar_wait(&q_free[qb], ((next_q - QB) >> 1) & 1, abort_flag)))
            break;
          const int bg = seg[next_q].x;
          const int b = bg / s.H_kv, g = bg % s.H_kv;
          const int q_row0 = (b * s.H + g * s.G) * s.L_q;
          mbar_arrive_expect_tx(&q_full[qb], Q_BYTES);
          for (int h = 0; h < 2; ++h)
            tma_load_2d(sQ + qb * Q_BYTES + h * (NQ * 128), &tm_q, h * 64, q_row0, &q_full[qb]);
          ++next_q;
        }
        if (!ok) break;
        const int st = j % ST;
        if (j >= ST && !(ok = mbar_wait(&empty[st], ((j / ST) - 1) & 1, abort_flag))) break;
        uint8_t* dst = ring + st * KS_BYTES;
        const int info[2] = {e.z & 0xFFFF, e.w};
        const int ys[2] = {e.x, e.y};
        const uint32_t bytes = (page_valid(info[0]) > 0 ? 16384u : 0u) +
                               (page_valid(info[1]) > 0 ? 16384u : 0u);
        if (bytes == 0) {
          mbar_arrive(&full[st]);
          continue;
        }
        mbar_arrive_expect_tx(&full[st], bytes);
        for (int p = 0; p < 2; ++p) {
          if (page_valid(info[p]) == 0) continue;
          for (int h = 0; h < 2; ++h) {
            if (!page_dec(info[p]))
              tma_load_2d(dst + h * 16384 + p * 8192, map, h * 64, ys[p], &full[st]);
            else
              tma_load_3d(dst + h * 16384 + p * 8192, map_dec, h * 64, ys[p],
                          seg[k].x, &full[st]);
          }
        }
      }
      if (*abort_flag) {  // do not leave with copies in flight
        for (int j = max(0, nst - ST); j < nst; ++j)
          for (uint32_t t = 0; t < (1u << 20) && !mbar_try_wait(&full[j % ST], (j / ST) & 1); ++t) {
          }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    if (lane == 0 && nst > 0 && (warp == 1 || !lse_only)) {
      // K and Q K-major (LBO 16, SBO 1024 B); V^T and P^T MN-major (LBO =
      // the 64-column half, SBO = 1024 B per 8 keys)
      const uint64_t q_desc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(smem_u32(sK), 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(smem_u32(sV), 16384, 1024);
      const uint64_t p_desc0 = sdesc_sw128(smem_u32(sPT), 1024, 1024);
      bool ok = true;
      if (warp == 1) {
        constexpr uint32_t IS = idesc_bf16_f32_ab(128, NQ, false, false);
        for (int j = 0; ok && j < nst; ++j) {
          const int k = step_seg(steps[j]);
          const int qb = k & 1;
          if (first_of(j) && !(ok = mbar_wait(&q_full[qb], (k >> 1) & 1, abort_flag))) break;
          const int buf = j & 1;
          // the S^T buffer is free once the softmax of step j-2 has read it
          if (j >= 2 && !(ok = mbar_wait(&p_ready[buf], ((j - 2) >> 1) & 1, abort_flag))) break;
          const int st = j % STK;
          if (!(ok = mbar_wait(&full_k[st], (j / STK) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t ad0 = k_desc0 + (uint64_t)((st * KS_BYTES) >> 4);
          const uint64_t bd0 = q_desc0 + (uint64_t)((qb * Q_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int h = kk >> 2, k4 = kk & 3;
            mma_f16_ss(tmem + S_COL + buf * NQ, ad0 + (uint64_t)((h * 16384 + k4 * 32) >> 4),
                       bd0 + (uint64_t)((h * NQ * 128 + k4 * 32) >> 4), IS, kk > 0 ? 1u : 0u);
          }
          mma_commit(&s_full[buf]);
          mma_commit(&empty_k[st]);
          if (last_of(j)) mma_commit(&q_free[qb]);
        }
      } else {
        constexpr uint32_t IP = idesc_bf16_f32_ab(128, NQ, true, true);
        for (int j = 0; ok && j < nst; ++j) {
          const int k = step_seg(steps[j]);
          const int buf = j & 1;
          if (!(ok = mbar_wait(&p_ready[buf], (j >> 1) & 1, abort_flag))) break;
          const bool first = first_of(j);
          const int ob = k & 1;
          if (first && k >= 2 && !(ok = mbar_wait(&o_free[ob], ((k - 2) >> 1) & 1, abort_flag)))
            break;
          const int st = j % STVd;
          if (!(ok = mbar_wait(&full_v[st], (j / STVd) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t ad0 = v_desc0 + (uint64_t)((st * KS_BYTES) >> 4);
          const uint64_t bd0 = p_desc0 + (uint64_t)((buf * PT_BYTES) >> 4);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_f16_ss(tmem + O_COL + ob * NQ, ad0 + (uint64_t)((kk * 2048) >> 4),
                       bd0 + (uint64_t)((kk * 2048) >> 4), IP, (!first || kk > 0) ? 1u : 0u);
          mma_commit(&empty_v[st]);
          mma_commit(&pv_done[buf]);
        }
      }
      if (*abort_flag) {  // give issued MMAs time to finish before TMEM is freed
        for (uint32_t t = 0; t < (1u << 16); ++t) __nanosleep(1000);
      }
    }
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int quad = warp & 3;
    const int key = quad * 32 + lane;  // TMEM lane: key of the step / model dimension
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const float c2 = static_cast<float>(s.scale * 1.4426950408889634);
    float m_ref[NQ], l_sum[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      m_ref[q] = -INFINITY;
      l_sum[q] = 0.0f;
    }
    float m_mine = -INFINITY;  // m_ref[lane], kept as a scalar for the epilogue
    int n_resc = 0, n_segdone = 0;
    bool ok = nst > 0;
    auto wait_all = [&](uint64_t* bar, uint32_t parity) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag));
    };
    // end of segment k: the row sums over the 128 lanes, (max, sum) of each
    // row to the partial, and a fresh reference for the next segment
    auto segment_sums = [&](int k) -> bool {
      s_sum[quad * NQ + lane] = xreduce32<false>(l_sum, lane);
      __syncwarp();
      if (lane == 0) mbar_arrive(lbar);
      if (!wait_all(lbar, n_segdone & 1)) return false;
      ++n_segdone;
      if (quad == 0 && lane < R) {
        const size_t prow0 = ((size_t)seg[k].x * plan.nslot + seg[k].y) * R;
        const float lt = s_sum[lane] + s_sum[NQ + lane] + s_sum[2 * NQ + lane] + s_sum[3 * NQ + lane];
        part.ml[prow0 + lane] = make_float2(
            m_mine == -INFINITY ? -INFINITY : m_mine * 0.69314718055994531f,
            m_mine == -INFINITY ? 0.0f : lt);
      }
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        m_ref[q] = -INFINITY;
        l_sum[q] = 0.0f;
      }
      m_mine = -INFINITY;
      return true;
    };
    for (int j = 0; ok && j < nst; ++j) {
      const int4 e = steps[j];
      const int k = step_seg(e);
      const int ob = k & 1;
      const bool first = first_of(j);
      const bool last = last_of(j);
      const int buf = j & 1;
      const int st = j % STVd;
      const int pinfo = (key < 64) ? (e.z & 0xFFFF) : e.w;
      const int pvalid = page_valid(pinfo);
      const bool kvalid = (key & 63) < pvalid;
      if (!(ok = wait_all(&s_full[buf], (j >> 1) & 1))) break;
      tc_fence_after();
      uint32_t sv[NQ];
      tmem_ld<NQ>(tmem + lane_base + S_COL + buf * NQ, sv);
      tmem_ld_wait();
      float x[NQ];
      bool need = false;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        x[q] = (kvalid && q < R) ? __uint_as_float(sv[q]) * c2 : -INFINITY;
        need |= x[q] > m_ref[q] + 8.0f;
      }
      // vote: does any thread of the four warps need a larger reference?
      const unsigned bal = __ballot_sync(0xffffffffu, need);
      if (lane == 0) s_vote[buf * 4 + quad] = bal != 0u;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[buf]);
      if (!(ok = wait_all(&xbar[buf], (j >> 1) & 1))) break;
      const bool any = s_vote[buf * 4] | s_vote[buf * 4 + 1] | s_vote[buf * 4 + 2] |
                       s_vote[buf * 4 + 3];
      if (any) {
        float v[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) v[q] = x[q];
        s_max[quad * NQ + lane] = xreduce32<true>(v, lane);
        __syncwarp();
        if (lane == 0) mbar_arrive(mxbar);
        if (!(ok = wait_all(mxbar, n_resc & 1))) break;
        ++n_resc;
        float alpha[NQ];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const float tmax = fmaxf(fmaxf(s_max[q], s_max[NQ + q]),
                                   fmaxf(s_max[2 * NQ + q], s_max[3 * NQ + q]));
          const float m_new = fmaxf(m_ref[q], tmax);
          alpha[q] = m_ref[q] == -INFINITY ? 0.0f : exp2f(m_ref[q] - m_new);
          l_sum[q] *= alpha[q];
          m_ref[q] = m_new;
        }
        m_mine = fmaxf(m_mine, fmaxf(fmaxf(s_max[lane], s_max[NQ + lane]),
                                     fmaxf(s_max[2 * NQ + lane], s_max[3 * NQ + lane])));
        if (!first && !lse_only) {
          // O^T holds every step before j: rescale this thread's row
          if (!(ok = wait_all(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1))) break;
          tc_fence_after();
          uint32_t o[NQ];
          tmem_ld<NQ>(tmem + lane_base + O_COL + ob * NQ, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < NQ; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha[q]);
          tmem_st<NQ>(tmem + lane_base + O_COL + ob * NQ, o);
          tmem_st_wait();
        }
      }
      uint32_t pk[NQ / 2];
#pragma unroll
      for (int q = 0; q < NQ; q += 2) {
        const float p0 = (x[q] == -INFINITY || m_ref[q] == -INFINITY) ? 0.0f : ex2_approx(x[q] - m_ref[q]);
        const float p1 = (x[q + 1] == -INFINITY || m_ref[q + 1] == -INFINITY)
                             ? 0.0f : ex2_approx(x[q + 1] - m_ref[q + 1]);
        l_sum[q] += p0;
        l_sum[q + 1] += p1;
        pk[q >> 1] = pack_bf16x2(p0, p1);
      }
      if (lse_only) {  // the row sums are all that is kept
        tc_fence_before();
        mbar_arrive(&p_ready[buf]);
        if (last && !(ok = segment_sums(k))) break;
        continue;
      }
      // the P^T buffer is free once the O^T MMAs of step j-2 are done
      if (j >= 2 && !(ok = wait_all(&pv_done[buf], ((j - 2) >> 1) & 1))) break;
      uint8_t* prow = sPT + buf * PT_BYTES + (key >> 3) * 1024 + (key & 7) * 128;
#pragma unroll
      for (int c = 0; c < NQ / 8; ++c)
        *reinterpret_cast<uint4*>(prow + ((c ^ (key & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      if (!kvalid && pvalid > 0) {
        // a loaded page's rows past its valid keys may hold anything (even
        // NaN): zero this key's V row once it has landed
        ok = mbar_wait(&full_v[st], (j / STVd) & 1, abort_flag);
        if (ok) {
          uint8_t* vr = sV + st * KS_BYTES + key * 128;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int c = 0; c < 8; ++c)
              *reinterpret_cast<uint4*>(vr + h * 16384 + c * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      if (!(ok = __all_sync(0xffffffffu, ok))) break;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[buf]);
      if (!last) continue;
      // ---- segment epilogue: O^T columns (rows of O), reference max, sum
      if (!(ok = wait_all(&pv_done[buf], (j >> 1) & 1))) break;
      tc_fence_after();
      const int bg = seg[k].x;
      const size_t prow0 = ((size_t)bg * plan.nslot + seg[k].y) * R;
      uint32_t o[NQ];
      tmem_ld<NQ>(tmem + lane_base + O_COL + ob * NQ, o);
      tmem_ld_wait();
#pragma unroll
      for (int q = 0; q < NQ; ++q)
        if (q < R) part.o[(prow0 + q) * D + key] = __uint_as_float(o[q]);
      tc_fence_before();
      mbar_arrive(&o_free[ob]);
      if (!(ok = segment_sums(k))) break;
    }
  }
  if (threadIdx.x == 0 && *abort_flag) flag_error(a.err, ERR_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Whether the key-major kernel takes this call: bf16, head dim 128, block or
// dense keys, at most 32 query rows per KV group.
bool attn_tc_kt_supported(const AttnArgs& a) {
  const Shape& s = a.s;
  return s.dtype == 0 && s.d == 128 && a.mode != kGather && s.G * s.L_q <= kt::NQ &&
         (uint64_t)s.n_slots * s.H_kv * 64 < (1ull << 31) &&
         (uint64_t)s.batch * s.H * s.L_q < (1ull << 31);
}

cudaError_t launch_attn_tc_kt(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  const Shape& s = a.s;
  CUtensorMap mq, mk, mv, mkd, mvd;
  const uint64_t pool_rows = (uint64_t)s.n_slots * s.H_kv * 64;
  const uint64_t q_rows = (uint64_t)s.batch * s.H * s.L_q;
  const uint64_t n_bg = (uint64_t)s.batch * s.H_kv;
  if (!tc_map_2d(&mq, a.Q, kt::D, q_rows, kt::NQ) ||
      !tc_map_2d(&mk, a.Kp, kt::D, pool_rows, 64) || !tc_map_2d(&mv, a.Vp, kt::D, pool_rows, 64) ||
      !tc_map_3d(&mkd, a.Kd, kt::D, s.L_q, n_bg) || !tc_map_3d(&mvd, a.Vd, kt::D, s.L_q, n_bg))
    return cudaErrorInvalidValue;
  const TcLaunch L = tc_plan((int)n_bg, max_tiles, tc_sm_count());
  if (L.plan.nslot > kMaxSplits) return cudaErrorInvalidValue;  // workspace bound
  cudaError_t e;
  if (a.O == nullptr) {  // the row LSEs only
    constexpr int smem = kt::Layout<true>::SMEM;
    if ((e = cudaFuncSetAttribute(attn_tc_kt_kernel<true>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    DL_LAUNCH(attn_tc_kt_kernel<true>, L.grid, kt::THREADS, smem, st, mq, mk, mv, mkd, mvd, a,
              L.plan);
  } else {
    constexpr int smem = kt::Layout<false>::SMEM;
    if ((e = cudaFuncSetAttribute(attn_tc_kt_kernel<false>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    DL_LAUNCH(attn_tc_kt_kernel<false>, L.grid, kt::THREADS, smem, st, mq, mk, mv, mkd, mvd, a,
              L.plan);
  }
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_combine(a, L.plan.nslot, st, L.plan.S, L.grid);
}

}  // namespace dl
