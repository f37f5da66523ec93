// (a6) Block-sparse bidirectional attention on the sm_100a tensor cores.
//
// Focus-dLLM abstract / summary: every decode-block query attends to the
// selected (sink-aware) context blocks and to the decode block itself, with
// no causal mask; shallow layers attend to every block.
//
// One CTA per (split, b, g).  Its tiles are 64-key pages: the selected
// context blocks (through the page table) and then the decode block.  Roles:
//   warp 0, one thread : TMA producer of Q (per segment) and of the K ring;
//   warp 2, one thread : TMA producer of the V ring (128-byte swizzle; the
//                        pool is a 2-D tensor map of 64-row pages, so a
//                        gathered block is just a coordinate; a K slot is
//                        freed when its S is done, a V slot when its P V is);
//   warp 1, one thread : tcgen05.mma issuer of S = Q K^T into TMEM (two
//                        buffers; a buffer is reused once the softmax of the
//                        tile two back has read it);
//   warp 3, one thread : tcgen05.mma issuer of O += P V into TMEM (each
//                        issuer has its own chain of waits, so the two
//                        streams of MMAs overlap);
//   warps 4.. (4 per M-tile of 128 rows): softmax -- one thread per TMEM
//                        lane.  With at most 32 (64) query rows, the M-tile
//                        holds 4 (2) replicas of them, one per lane quadrant
//                        (pair), so that all four SM sub-partitions work:
//                        replica c takes columns [c*64/REP, (c+1)*64/REP) of
//                        each tile, the row maximum is exchanged through
//                        shared memory, and each replica writes its P columns
//                        into every replica block, so every replica's O row
//                        is complete; replica c rescales and writes out only
//                        its share of O's columns.  Each thread keeps a running
//                        max (lazy rescale: O and l are rescaled only when the
//                        max grows by more than 2^8) and sum, writes P (bf16)
//                        to shared memory in the MMA's K-major swizzled
//                        layout, and at the end writes its partial (O, m, l).
// Gathered tokens (the chunked prefix: arbitrary cached positions): a tile is
// 64 consecutive entries of the (b, g)'s position list.  The pool's tensor
// maps then have one-row boxes and the whole producer warp loads the tile's
// rows with TMA row gathers (four rows per instruction, lane = four rows of
// one 64-column half) into the same swizzled layout, every lane's loads
// completing on the tile's full barrier.  Each lane resolves two rows'
// positions through the page table; rows past the tile's valid keys, or with
// a bad position, take the row past the pool, which TMA fills with zeros (so
// a NaN in an unused pool row never reaches P V).  Decode tiles keep their
// tiled TMA path.
// The G*L_q query rows of a KV group are padded to M-tiles of 128 rows (the
// path is HBM-bound: padding costs tensor time, not bytes).  Partials of the
// splits of one (b, g) are merged by the combine kernel of attn_simt.cu.
//
// Every wait is bounded: a role that gives up raises the shared abort flag
// and the device error word (ERR_TIMEOUT) and leaves its loop; the CTA then
// frees its TMEM and returns.
#include <cstdlib>
#include <mutex>

#include "sm100.cuh"
#include "score_common.cuh"
#include "tc_common.cuh"
#include "launch.cuh"

namespace dl {

using namespace sm100;

// Four rows y0..y3 of a 2-D tensor map whose box is one row high, columns
// [x, x + box width), to four consecutive box rows at dst (the map's swizzle
// applied); rows past the tensor are filled with zeros.
__device__ __forceinline__ void tma_gather4_2d(void* dst, const CUtensorMap* map, int x, int y0,
                                               int y1, int y2, int y3, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y0), "r"(y1),
      "r"(y2), "r"(y3)
      : "memory");
}

// D head dim, NM M-tiles of 128 rows, REP replicas of the query rows in an
// M-tile (4: at most 32 rows, 2: at most 64, 1 otherwise), ST K/V stages, QB
// Q buffers and OB O accumulators (2 = the next segment starts while the
// previous one is written out).
template <int D, int NM, int REP, int ST, int QB, int OB>
struct TcCfg {
  static constexpr int PB = 2;                             // P buffers
  static constexpr int HALVES = D / 64;                    // 128-byte column chunks
  static constexpr int Q_TILE = NM * HALVES * 128 * 128;   // [m][half][128 rows][128 B]
  static constexpr int KT_BYTES = HALVES * 64 * 128;       // [half][64 rows][128 B]
  static constexpr int RING_BYTES = ST * KT_BYTES;         // one ring of K (or V) tiles
  static constexpr int P_TILE = 128 * 128;                 // [128 rows][64 keys bf16]
  static constexpr int RB = 128 / REP;                     // rows per replica block
  static constexpr int NC = 64 / REP;                      // S columns per softmax thread
  static constexpr int OC = D / REP;                       // O columns per softmax thread
  static constexpr int SOFTMAX_THREADS = 128 * NM;
  static constexpr int KV_OFF = QB * Q_TILE;
  static constexpr int P_OFF = KV_OFF + 2 * RING_BYTES;    // K ring, then V ring
  static constexpr int RED_OFF = P_OFF + PB * NM * P_TILE;
  static constexpr int RED_BYTES = 3 * 128 * 4;            // tile maxima x2, final sums
  static constexpr int BAR_OFF = RED_OFF + RED_BYTES;
  // full_k, empty_k, full_v, empty_v [ST]; q_full, q_free [2]; s_full,
  // p_ready [2]; pv_done [2]; o_free [2]; xbar [2][NM][4]; lbar [NM][4]
  static constexpr int N_BARS = 4 * ST + 2 + 2 + 2 + 2 + 2 + 2 + 3 * NM * 4;
  static constexpr int MISC_OFF = (BAR_OFF + N_BARS * 8 + 15) / 16 * 16;
  static constexpr int TILE_OFF = MISC_OFF + 16;                   // int2 [kTcMaxTiles]
  static constexpr int SEG_OFF = TILE_OFF + kTcMaxTiles * 8;       // int4 [kMaxSegs]
  static constexpr int SEGLO_OFF = SEG_OFF + kMaxSegs * 16;        // int [kMaxSegs]
  static constexpr int MARK_OFF = SEGLO_OFF + kMaxSegs * 4;        // int2 [kMaxSegs]
  static constexpr int ROWS_OFF = MARK_OFF + kMaxSegs * 8;         // int [ROWS_CAP]
  static constexpr int ROWS_CAP = 64 * 64;  // gathered rows resolved up front (64 tiles)
  static_assert(BAR_OFF % 16 == 0 && TILE_OFF % 16 == 0 && SEG_OFF % 16 == 0, "alignment");
  static constexpr int SMEM = ROWS_OFF + ROWS_CAP * 4 + 1024;      // + alignment slack
  static constexpr int THREADS = 128 + SOFTMAX_THREADS;
  static constexpr uint32_t TMEM_NEED = OB * NM * D + 2 * NM * 64;
  static constexpr uint32_t TMEM_COLS = TMEM_NEED <= 128 ? 128 : TMEM_NEED <= 256 ? 256 : 512;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(TMEM_NEED <= 512, "tensor memory budget");
  static_assert(NC >= 16 && OC >= 16, "column split");
  static_assert(REP == 1 || NM == 1, "replicas only within one M-tile");
};

template <int D, int NM, int REP, int ST, int QB, int OB>
__global__ void __launch_bounds__(128 + 128 * NM, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kd,
               const __grid_constant__ CUtensorMap tm_vd, const AttnArgs a, const TcPlan plan) {
  using C = TcCfg<D, NM, REP, ST, QB, OB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sK = smem + C::KV_OFF;               // K ring [ST][KT_BYTES]
  uint8_t* sV = sK + C::RING_BYTES;              // V ring [ST][KT_BYTES]
  uint8_t* sP = smem + C::P_OFF;
  float* s_red = reinterpret_cast<float*>(smem + C::RED_OFF);  // [2][RB][REP]
  float* s_lsum = s_red + 2 * 128;                             // [RB][REP]
  // K and V travel in separate rings: a K slot is free once its S = Q K^T is
  // done, a V slot once its P V is done, so neither waits for the softmax
  uint64_t* full_k = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  uint64_t* empty_k = full_k + ST;
  uint64_t* full_v = empty_k + ST;
  uint64_t* empty_v = full_v + ST;
  uint64_t* q_full = empty_v + ST;   // [2] Q of a segment landed
  uint64_t* q_free = q_full + 2;     // [2] every S of a segment done (Q reusable)
  uint64_t* s_full = q_free + 2;     // [2] S buffer written
  uint64_t* p_ready = s_full + 2;    // [2] P written, O rescaled
  uint64_t* pv_done = p_ready + 2;   // [2] P V of the tiles of that parity done
  uint64_t* o_free = pv_done + 2;    // [2] segment's O read out
  uint64_t* xbar = o_free + 2;       // [2][NM][4] tile-max exchange
  uint64_t* lbar = xbar + 2 * NM * 4;  // [NM][4] final-sum exchange
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::MISC_OFF + 4);
  int* s_nt = reinterpret_cast<int*>(smem + C::MISC_OFF + 8);
  int* s_nseg = s_nt + 1;
  int2* t_info = reinterpret_cast<int2*>(smem + C::TILE_OFF);  // (y, valid | seg << 16)
  int4* seg = reinterpret_cast<int4*>(smem + C::SEG_OFF);      // (bg, slot, first, n)
  int* seg_lo = reinterpret_cast<int*>(smem + C::SEGLO_OFF);   // first tile index in (b, g)
  int2* mark = reinterpret_cast<int2*>(smem + C::MARK_OFF);    // (bg, slot) of empty runs
  int* s_rows = reinterpret_cast<int*>(smem + C::ROWS_OFF);    // pool row of each gathered key
  int* s_nmark = s_nt + 2;

  const Shape& s = a.s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // tensor memory first; the successor may be scheduled only after that
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
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

  if (threadIdx.x == 0) {
    for (int i = 0; i < 4 * ST; ++i) mbar_init(&full_k[i], 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_free[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_ready[i], C::SOFTMAX_THREADS);
      mbar_init(&o_free[i], C::SOFTMAX_THREADS);
      mbar_init(&pv_done[i], 1);
    }
    for (int i = 0; i < 3 * NM * 4; ++i) mbar_init(&xbar[i], 128);
    *abort_flag = 0;
    fence_mbar_init();
    // runs of (b, g) in this CTA's slots: segments (with tiles) and markers
    int nseg = 0, nmark = 0, ntile = 0;
    if (u1 > u0) {
      for (int bg = (int)(u0 / plan.S); bg <= (int)((u1 - 1) / plan.S); ++bg) {
        const long long base = (long long)bg * plan.S;
        const int lo = (int)max(u0 - base, 0ll);
        const int hi = (int)min(u1 - base, (long long)plan.S);
        const int n_tiles = ctx_tile_count(a, bg) + n_dec;
        const int thi = min(hi, n_tiles);
        const int slot = (int)blockIdx.x - tc_owner(base, U, gridDim.x);
        if (thi > lo) {
          seg[nseg] = make_int4(bg, slot, ntile, thi - lo);
          seg_lo[nseg] = lo;
          ++nseg;
          ntile += thi - lo;
        } else {
          mark[nmark++] = make_int2(bg, slot);
        }
      }
    }
    *s_nt = ntile;
    *s_nseg = nseg;
    *s_nmark = nmark;
  }
  __syncthreads();
  const int nt = *s_nt, nseg = *s_nseg, nmark = *s_nmark;
  for (int e = threadIdx.x; e < nmark * R; e += blockDim.x) {
    const int2 mk = mark[e / R];
    part.ml[((size_t)mk.x * plan.nslot + mk.y) * R + e % R] = make_float2(-INFINITY, 0.0f);
  }
  // tile table: TMA row coordinate, valid keys, segment
  for (int k = 0; k < nseg; ++k) {
    const int bg = seg[k].x;
    const int n_ctx = ctx_tile_count(a, bg);
    const int lo = seg_lo[k];
    for (int t = threadIdx.x; t < seg[k].w; t += blockDim.x) {
      int2 ti;
      if (a.mode == kGather && lo + t < n_ctx) {  // rows are resolved by the producer
        const int c = min(max(a.cnt[bg], 0), a.max_idx);
        ti = make_int2(0, min(64, c - (lo + t) * 64));
      } else {
        ti = tc_tile_info(a, bg, lo + t, n_ctx);
      }
      t_info[seg[k].z + t] = make_int2(ti.x, ti.y | (k << 16));
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  auto tile_seg = [&](int i) { return t_info[i].y >> 16; };
  auto tile_valid = [&](int i) { return t_info[i].y & 0x7F; };
  auto tile_dec = [&](int i) { return (t_info[i].y >> 15) & 1; };
  // gathered keys: each row's pool row (through its position and the page
  // table), resolved by every thread at once so that the producers only copy
  const bool rows_staged = a.mode == kGather && nt * 64 <= C::ROWS_CAP;
  if (rows_staged) {
    for (int e = threadIdx.x; e < nt * 64; e += blockDim.x) {
      const int i = e >> 6, r = e & 63;
      int row = -1;
      if (!tile_dec(i) && r < tile_valid(i)) {
        const int k = tile_seg(i);
        const int bg = seg[k].x;
        const int b = bg / s.H_kv, g = bg % s.H_kv;
        const int pos = a.idx[(size_t)bg * a.max_idx + (seg_lo[k] + i - seg[k].z) * 64 + r];
        const int slot =
            pos >= 0 && pos < s.L_ctx ? a.page_table[(size_t)b * s.n_pages + pos / 64] : -1;
        if (slot >= 0 && slot < s.n_slots)
          row = (slot * s.H_kv + g) * 64 + pos % 64;
        else
          flag_error(a.err, ERR_BAD_INDEX);  // the key is left zero
      }
      s_rows[e] = row;
    }
    __syncthreads();
  }

  if (warp == 0 || warp == 2) {
    // ------------------------------------------------------------ producers
    // warp 0: Q of every segment and the K ring; warp 2: the V ring
    const bool is_k = warp == 0;
    uint64_t* full = is_k ? full_k : full_v;
    uint64_t* empty = is_k ? empty_k : empty_v;
    uint8_t* ring = is_k ? sK : sV;
    const CUtensorMap* map = is_k ? &tm_k : &tm_v;
    const CUtensorMap* map_dec = is_k ? &tm_kd : &tm_vd;
    if (a.mode == kGather && nt > 0) {
      // ---- gathered rows: TMA row gathers issued by the whole warp
      if (lane == 0) {
        prefetch_tmap(map);
        prefetch_tmap(map_dec);
      }
      const int oob_row = s.n_slots * s.H_kv * 64;  // past the pool: zero fill
      auto load_q = [&](int k) -> bool {
        const int qb = QB == 2 ? (k & 1) : 0;
        bool w = true;
        if (k >= QB) {  // the buffer's previous segment must be done with it
          const int prev = k - QB;
          if (lane == 0)
            w = mbar_wait(&q_free[qb], (QB == 2 ? (prev >> 1) : prev) & 1, abort_flag);
          w = __shfl_sync(0xffffffffu, w, 0);
        }
        if (w && lane == 0) {
          const int bg = seg[k].x;
          const int b = bg / s.H_kv, g = bg % s.H_kv;
          const int q_row0 = (b * s.H + g * s.G) * s.L_q;
          mbar_arrive_expect_tx(&q_full[qb], C::Q_TILE);
          for (int m = 0; m < NM; ++m)
            for (int h = 0; h < C::HALVES; ++h)
              for (int c = 0; c < REP; ++c)
                tma_load_2d(sQ + qb * C::Q_TILE + (m * C::HALVES + h) * 16384 + c * C::RB * 128,
                            &tm_q, h * 64, q_row0 + m * 128, &q_full[qb]);
        }
        return w;
      };
      if (is_k && lane == 0) prefetch_tmap(&tm_q);
      int next_q = 0;
      bool ok = true;
      for (int i = 0; ok && i < nt; ++i) {
        const int k = tile_seg(i);
        while (is_k && ok && next_q < nseg && next_q <= k) {
          ok = load_q(next_q);
          ++next_q;
        }
        if (!ok) break;
        const int st = i % ST;
        if (i >= ST) {
          bool w = true;
          if (lane == 0) w = mbar_wait(&empty[st], ((i / ST) - 1) & 1, abort_flag);
          if (!(ok = __shfl_sync(0xffffffffu, w, 0))) break;
        }
        uint8_t* dst = ring + st * C::KT_BYTES;
        const int valid = tile_valid(i);
        if (valid > 0 && !tile_dec(i)) {
          const int bg = seg[k].x;
          const int b = bg / s.H_kv, g = bg % s.H_kv;
          const int tile = seg_lo[k] + (i - seg[k].z);  // tile of the (b, g)'s list
          // lane owns rows lane and lane + 32 (their pool rows resolved here)
          int own[2] = {oob_row, oob_row};
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            const int r = lane + 32 * rr;
            if (rows_staged) {
              const int row = s_rows[i * 64 + r];
              if (row >= 0) own[rr] = row;
            } else if (r < valid) {
              const int pos = a.idx[(size_t)bg * a.max_idx + tile * 64 + r];
              const int slot = pos >= 0 && pos < s.L_ctx
                                   ? a.page_table[(size_t)b * s.n_pages + pos / 64] : -1;
              if (slot >= 0 && slot < s.n_slots)
                own[rr] = (slot * s.H_kv + g) * 64 + pos % 64;
              else
                flag_error(a.err, ERR_BAD_INDEX);  // the key is left zero
            }
          }
          if (lane == 0) mbar_arrive_expect_tx(&full[st], C::KT_BYTES);
          __syncwarp();
          // lane: rows 4 q4 .. 4 q4 + 3 of column half h
          const int q4 = (lane & 15) * 4, h = lane >> 4;
          int y[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int r = q4 + j;
            const int lo = __shfl_sync(0xffffffffu, own[0], r & 31);
            const int hi = __shfl_sync(0xffffffffu, own[1], r & 31);
            y[j] = r < 32 ? lo : hi;
          }
          if (h < C::HALVES)
            tma_gather4_2d(dst + h * 8192 + q4 * 128, map, h * 64, y[0], y[1], y[2], y[3],
                           &full[st]);
        } else if (valid > 0) {
          if (lane == 0) {
            mbar_arrive_expect_tx(&full[st], C::KT_BYTES);
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_3d(dst + h * 8192, map_dec, h * 64, t_info[i].x, seg[k].x, &full[st]);
          }
        } else if (lane == 0) {
          mbar_arrive(&full[st]);
        }
      }
      if (*abort_flag && lane == 0) {  // do not leave with loads in flight
        for (int i = max(0, nt - ST); i < nt; ++i)
          for (uint32_t t = 0; t < (1u << 20) && !mbar_try_wait(&full[i % ST], (i / ST) & 1); ++t) {
          }
      }
    } else if (lane == 0 && nt > 0) {
      prefetch_tmap(map);
      prefetch_tmap(map_dec);
      auto load_q = [&](int k) -> bool {
        const int qb = QB == 2 ? (k & 1) : 0;
        if (k >= QB) {  // the buffer's previous segment must be done with it
          const int prev = k - QB;
          if (!mbar_wait(&q_free[qb], (QB == 2 ? (prev >> 1) : prev) & 1, abort_flag))
            return false;
        }
        const int bg = seg[k].x;
        const int b = bg / s.H_kv, g = bg % s.H_kv;
        const int q_row0 = (b * s.H + g * s.G) * s.L_q;
        mbar_arrive_expect_tx(&q_full[qb], C::Q_TILE);
        for (int m = 0; m < NM; ++m)
          for (int h = 0; h < C::HALVES; ++h)
            for (int c = 0; c < REP; ++c)  // replica c at rows [c*RB, (c+1)*RB)
              tma_load_2d(sQ + qb * C::Q_TILE + (m * C::HALVES + h) * 16384 + c * C::RB * 128,
                          &tm_q, h * 64, q_row0 + m * 128, &q_full[qb]);
        return true;
      };
      int next_q = 0;  // next segment whose Q is to be loaded
      bool ok = true;
      for (int i = 0; ok && i < nt; ++i) {
        const int k = tile_seg(i);
        // a segment's Q is loaded with its first K tile
        while (is_k && ok && next_q < nseg && next_q <= k) {
          ok = load_q(next_q);
          ++next_q;
        }
        if (!ok) break;
        const int st = i % ST;
        if (i >= ST && !mbar_wait(&empty[st], ((i / ST) - 1) & 1, abort_flag)) break;
        uint8_t* dst = ring + st * C::KT_BYTES;
        if (tile_valid(i) > 0) {
          mbar_arrive_expect_tx(&full[st], C::KT_BYTES);
          if (!tile_dec(i)) {
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_2d(dst + h * 8192, map, h * 64, t_info[i].x, &full[st]);
          } else {
            const int bg = seg[k].x;
            for (int h = 0; h < C::HALVES; ++h)
              tma_load_3d(dst + h * 8192, map_dec, h * 64, t_info[i].x, bg, &full[st]);
          }
        } else {
          mbar_arrive(&full[st]);  // nothing to load: the tile is fully masked
        }
      }
      if (*abort_flag) {  // do not leave with copies in flight
        for (int i = max(0, nt - ST); i < nt; ++i)
          for (uint32_t t = 0; t < (1u << 20) && !mbar_try_wait(&full[i % ST], (i / ST) & 1); ++t) {
          }
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ------------------------------------------------------------ MMA issuers
    // warp 1 issues S = Q K^T, warp 3 issues O += P V: two single-thread
    // issue chains, each with its own waits, so neither waits on the other
    if (lane == 0 && nt > 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      const uint32_t p_base = smem_u32(sP);
      // base descriptors (128-byte swizzle): Q and K K-major (LBO 16, SBO
      // 1024 B), P K-major, V MN-major (LBO = the 64-column half, 8 KB); the
      // descriptor of an offset address differs by the address field only
      const uint64_t q_desc0 = sdesc_sw128(q_base, 16, 1024);
      const uint64_t k_desc0 = sdesc_sw128(k_base, 16, 1024);
      const uint64_t p_desc0 = sdesc_sw128(p_base, 16, 1024);
      const uint64_t v_desc0 = sdesc_sw128(v_base, 8192, 1024);
      bool ok = true;
      auto is_first = [&](int i) { return i == 0 || tile_seg(i - 1) != tile_seg(i); };
      auto is_last = [&](int i) { return i == nt - 1 || tile_seg(i + 1) != tile_seg(i); };
      if (warp == 1) {
        constexpr uint32_t IS = idesc_bf16_f32(128, 64, false);
        for (int i = 0; ok && i < nt; ++i) {
          const int k = tile_seg(i);
          const int qb = QB == 2 ? (k & 1) : 0;
          if (is_first(i) &&
              !(ok = mbar_wait(&q_full[qb], (QB == 2 ? (k >> 1) : k) & 1, abort_flag)))
            break;
          const int buf = i & 1;
          // the S buffer is free once the softmax of tile i-2 has read it
          if (i >= 2 && !(ok = mbar_wait(&p_ready[buf], ((i - 2) >> 1) & 1, abort_flag))) break;
          const int st = i % ST;
          if (!(ok = mbar_wait(&full_k[st], (i / ST) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t ad0 = q_desc0 + (uint64_t)((qb * C::Q_TILE) >> 4);
          const uint64_t bd0 = k_desc0 + (uint64_t)((st * C::KT_BYTES) >> 4);
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const uint32_t d_t = tmem + OB * NM * D + (buf * NM + m) * 64;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int h = kk >> 2, k4 = kk & 3;
              mma_f16_ss(d_t, ad0 + (uint64_t)(((m * C::HALVES + h) * 16384 + k4 * 32) >> 4),
                         bd0 + (uint64_t)((h * 8192 + k4 * 32) >> 4), IS, kk > 0 ? 1u : 0u);
            }
          }
          mma_commit(&s_full[buf]);
          mma_commit(&empty_k[st]);  // K is no longer needed once S is done
          if (is_last(i)) mma_commit(&q_free[qb]);  // only S reads Q
        }
      } else {
        constexpr uint32_t IP = idesc_bf16_f32(128, D, true);
        for (int i = 0; ok && i < nt; ++i) {
          const int k = tile_seg(i);
          const int buf = i & 1;
          if (!(ok = mbar_wait(&p_ready[buf], (i >> 1) & 1, abort_flag))) break;
          const bool first = is_first(i);
          const int ob = OB == 2 ? (k & 1) : 0;
          if (first && k >= OB &&
              !(ok = mbar_wait(&o_free[ob], (OB == 2 ? ((k - OB) >> 1) : (k - OB)) & 1, abort_flag)))
            break;
          const int st = i % ST;
          if (!(ok = mbar_wait(&full_v[st], (i / ST) & 1, abort_flag))) break;
          tc_fence_after();
          const uint64_t vd0 = v_desc0 + (uint64_t)((st * C::KT_BYTES) >> 4);
#pragma unroll
          for (int m = 0; m < NM; ++m) {
            const uint32_t d_t = tmem + (ob * NM + m) * D;
            const uint64_t pd0 = p_desc0 + (uint64_t)(((buf * NM + m) * C::P_TILE) >> 4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_f16_ss(d_t, pd0 + (uint64_t)((kk * 32) >> 4),
                         vd0 + (uint64_t)((kk * 2048) >> 4), IP, (!first || kk > 0) ? 1u : 0u);
          }
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
    // thread -> TMEM lane `row` of M-tile m; replica `rp` of query row `qr`
    const int m = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int rp = row / C::RB;
    const int qr = row % C::RB;
    const int r = m * 128 + qr;
    const bool active = r < R;
    const int col0 = rp * C::NC;
    const int ocol0 = rp * C::OC;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t s_col = OB * NM * D;
    const float c2 = static_cast<float>(s.scale * 1.4426950408889634);
    float m_run = -INFINITY, l_run = 0.0f;
    bool ok = nt > 0;
    // pv_done[t & 1] completes once per tile of that parity: tile t is its
    // completion t >> 1
    auto wait_pv = [&](int t) -> bool {
      return __all_sync(0xffffffffu, mbar_wait(&pv_done[t & 1], (t >> 1) & 1, abort_flag));
    };
    for (int i = 0; ok && i < nt; ++i) {
      const int k = tile_seg(i);
      const int ob = OB == 2 ? (k & 1) : 0;
      const uint32_t o_col = (ob * NM + m) * D;
      const bool first = i == 0 || tile_seg(i - 1) != k;
      const bool last = i == nt - 1 || tile_seg(i + 1) != k;
      if (first) {
        m_run = -INFINITY;
        l_run = 0.0f;
      }
      const int buf = i & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&s_full[buf], (i >> 1) & 1, abort_flag));
      if (!ok) break;
      tc_fence_after();
      uint32_t sv[C::NC];
      tmem_ld<C::NC>(tmem + lane_base + s_col + (buf * NM + m) * 64 + col0, sv);
      tmem_ld_wait();
      const int valid = tile_valid(i);
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < C::NC; ++c) {
        const float x = (active && col0 + c < valid) ? __uint_as_float(sv[c]) * c2 : -INFINITY;
        sv[c] = __float_as_uint(x);
        tmax = fmaxf(tmax, x);
      }
      if constexpr (REP > 1) {
        // the row's maximum over the whole tile: exchange between replicas
        float* red = s_red + buf * 128 + qr * REP;
        red[rp] = tmax;
        mbar_arrive(&xbar[buf]);
        ok = __all_sync(0xffffffffu, mbar_wait(&xbar[buf], (i >> 1) & 1, abort_flag));
        if (!ok) break;
#pragma unroll
        for (int q = 0; q < REP; ++q) tmax = fmaxf(tmax, red[q]);
      }
      const float m_new = fmaxf(m_run, tmax);
      const bool grow = m_new > m_run + 8.0f;
      const bool live = grow && m_run != -INFINITY;  // an accumulator to rescale
      if (__any_sync(0xffffffffu, live)) {
        ok = wait_pv(i - 1);  // O holds every P V before tile i
        if (!ok) break;
        tc_fence_after();
        const float alpha = live ? exp2f(m_run - m_new) : 1.0f;
        constexpr int CH = C::OC < 32 ? C::OC : 32;
#pragma unroll 1
        for (int cc = 0; cc < C::OC; cc += CH) {
          uint32_t o[CH];
          tmem_ld<CH>(tmem + lane_base + o_col + ocol0 + cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int q = 0; q < CH; ++q) o[q] = __float_as_uint(__uint_as_float(o[q]) * alpha);
          tmem_st<CH>(tmem + lane_base + o_col + ocol0 + cc, o);
        }
        tmem_st_wait();
      }
      if (grow) {
        l_run = (m_run == -INFINITY) ? 0.0f : l_run * exp2f(m_run - m_new);
        m_run = m_new;
      }
      uint32_t packed[C::NC / 2];
      float psum = 0.0f;
#pragma unroll
      for (int c = 0; c < C::NC; c += 2) {
        const float x0 = __uint_as_float(sv[c]), x1 = __uint_as_float(sv[c + 1]);
        const float p0 = (m_run == -INFINITY) ? 0.0f : ex2_approx(x0 - m_run);
        const float p1 = (m_run == -INFINITY) ? 0.0f : ex2_approx(x1 - m_run);
        psum += p0 + p1;
        packed[c >> 1] = pack_bf16x2(p0, p1);
      }
      l_run += psum;
      // the P buffer is free once the P V that last read it (tile i-2) is done
      if (i >= 2) {
        ok = wait_pv(i - 2);
        if (!ok) break;
      }
      // this replica's columns, into the P row of every replica block
#pragma unroll
      for (int blk = 0; blk < REP; ++blk) {
        const int prow_idx = blk * C::RB + qr;
        uint8_t* prow = sP + (buf * NM + m) * C::P_TILE + prow_idx * 128;
#pragma unroll
        for (int q = 0; q < C::NC / 8; ++q) {
          const int ch = col0 / 8 + q;
          *reinterpret_cast<uint4*>(prow + ((ch ^ (prow_idx & 7)) << 4)) =
              make_uint4(packed[4 * q], packed[4 * q + 1], packed[4 * q + 2], packed[4 * q + 3]);
        }
      }
      if (m == 0 && valid < 64 && (a.mode != kGather || tile_dec(i))) {
        // rows past the valid keys may hold anything (even NaN): zero V there
        // once it has landed (gathered tiles are zero-filled by their copies)
        ok = __all_sync(0xffffffffu, mbar_wait(&full_v[i % ST], (i / ST) & 1, abort_flag));
        if (!ok) break;
        uint8_t* sVt = sV + (i % ST) * C::KT_BYTES;
        const int per_row = C::HALVES * 8;
        const int nz = (64 - valid) * per_row;
        for (int e = row; e < nz; e += 128) {
          const int rr = valid + e / per_row, rem = e % per_row;
          *reinterpret_cast<uint4*>(sVt + (rem >> 3) * 8192 + rr * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_ready[buf]);
      if (!last) continue;
      // ---- segment epilogue: unnormalised partial O, running max and sum
      ok = wait_pv(i);
      if (!ok) break;
      tc_fence_after();
      const int bg = seg[k].x;
      const size_t prow_i = ((size_t)bg * plan.nslot + seg[k].y) * R + r;
      constexpr int CH = C::OC < 32 ? C::OC : 32;
#pragma unroll 1
      for (int cc = 0; cc < C::OC; cc += CH) {
        uint32_t o[CH];
        tmem_ld<CH>(tmem + lane_base + o_col + ocol0 + cc, o);
        tmem_ld_wait();
        if (active) {
          float4* dst = reinterpret_cast<float4*>(part.o + prow_i * D + ocol0 + cc);
#pragma unroll
          for (int q = 0; q < CH / 4; ++q)
            dst[q] = make_float4(__uint_as_float(o[4 * q]), __uint_as_float(o[4 * q + 1]),
                                 __uint_as_float(o[4 * q + 2]), __uint_as_float(o[4 * q + 3]));
        }
      }
      tc_fence_before();
      mbar_arrive(&o_free[ob]);
      float l_tot = l_run;
      if constexpr (REP > 1) {
        float* ls = s_lsum + qr * REP;
        ls[rp] = l_run;
        mbar_arrive(lbar);
        ok = __all_sync(0xffffffffu, mbar_wait(lbar, k & 1, abort_flag));
        if (!ok) break;
        l_tot = 0.0f;
#pragma unroll
        for (int q = 0; q < REP; ++q) l_tot += ls[q];
        // the sums are read before the next segment writes them: the next
        // write follows at least one tile-maximum exchange of every replica
      }
      if (active && rp == 0)
        part.ml[prow_i] = make_float2(m_run == -INFINITY ? -INFINITY : m_run * 0.69314718055994531f,
                                      m_run == -INFINITY ? 0.0f : l_tot);
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

bool tc_map_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t L_q, uint64_t n_bg) {
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

// int8 planes of `inner` bytes x rows, stacked `planes` deep; boxes of
// inner x box_rows x 1, 128-byte swizzle (inner must be 128).
bool tc_map_i8_3d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows,
                  uint64_t planes, uint32_t box_rows) {
  EncodeTiled fn = encoder();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, planes};
  cuuint64_t strides[2] = {inner, rows * inner};
  cuuint32_t box[3] = {static_cast<cuuint32_t>(inner), box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// Work split of the persistent kernel: one CTA per SM (more when the tile
// table of a CTA would overflow), S = the largest tile count of a (b, g).
TcLaunch tc_plan(int n_bg, int max_tiles, int sms) {
  TcLaunch L;
  L.plan.S = max_tiles;
  const long long U = (long long)n_bg * max_tiles;
  long long grid = U < sms ? U : sms;
  // partial slots per (b, g) stay within the workspace's kMaxSplits
  const long long cap = (long long)n_bg * (kMaxSplits - 2);
  grid = grid < cap ? grid : cap;
  // a CTA's tile table and its (b, g) runs must fit in shared memory
  if ((U + grid - 1) / grid > kTcMaxTiles) grid = (U + kTcMaxTiles - 1) / kTcMaxTiles;
  const long long per_seg = (long long)(kMaxSegs - 1) * max_tiles;
  if ((U + grid - 1) / grid > per_seg) grid = (U + per_seg - 1) / per_seg;
  L.grid = (int)grid;
  // CTAs that share one (b, g): those owning its first and last slots
  int nslot = 1;
  for (int bg = 0; bg < n_bg; ++bg) {
    const int n = tc_owner((long long)bg * max_tiles + max_tiles - 1, U, L.grid) -
                  tc_owner((long long)bg * max_tiles, U, L.grid) + 1;
    nslot = n > nslot ? n : nslot;
  }
  L.plan.nslot = nslot;
  return L;
}


template <int D, int NM, int REP, int ST, int QB, int OB>
static cudaError_t run_tc(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  using C = TcCfg<D, NM, REP, ST, QB, OB>;
  const Shape& s = a.s;
  CUtensorMap mq, mk, mv, mkd, mvd;
  const uint64_t pool_rows = (uint64_t)s.n_slots * s.H_kv * 64;
  const uint64_t q_rows = (uint64_t)s.batch * s.H * s.L_q;
  const uint64_t n_bg = (uint64_t)s.batch * s.H_kv;
  // gathered keys: one-row boxes for the row gathers; else 64-key pages
  const uint32_t pool_box = a.mode == kGather ? 1 : 64;
  if (!tc_map_2d(&mq, a.Q, D, q_rows, C::RB) || !tc_map_2d(&mk, a.Kp, D, pool_rows, pool_box) ||
      !tc_map_2d(&mv, a.Vp, D, pool_rows, pool_box) || !tc_map_3d(&mkd, a.Kd, D, s.L_q, n_bg) ||
      !tc_map_3d(&mvd, a.Vd, D, s.L_q, n_bg))
    return cudaErrorInvalidValue;
  const TcLaunch L = tc_plan((int)n_bg, max_tiles, tc_sm_count());
  if (L.plan.nslot > kMaxSplits) return cudaErrorInvalidValue;  // workspace bound
  auto kern = attn_tc_kernel<D, NM, REP, ST, QB, OB>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  DL_LAUNCH(kern, L.grid, C::THREADS, C::SMEM, st, mq, mk, mv, mkd, mvd, a, L.plan);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_combine(a, L.plan.nslot, st, L.plan.S, L.grid);
}

// Whether the tensor-core kernel takes this call (bf16, block or dense keys,
// at most two M-tiles of query rows, pool addressable by 32-bit TMA rows).
bool attn_tc_supported(const AttnArgs& a) {
  const Shape& s = a.s;
  return s.dtype == 0 && (a.mode != kGather || !(kernel_flags() & DL_FLAG_GATHER_SIMT)) && s.G * s.L_q <= 256 &&
         (uint64_t)s.n_slots * s.H_kv * 64 < (1ull << 31) &&
         (uint64_t)s.batch * s.H * s.L_q < (1ull << 31);
}

bool attn_tc_kt_supported(const AttnArgs& a);
cudaError_t launch_attn_tc_kt(const AttnArgs& a, int max_tiles, cudaStream_t st);

cudaError_t launch_attn_tc(const AttnArgs& a, int max_tiles, cudaStream_t st) {
  if (attn_tc_kt_supported(a)) return launch_attn_tc_kt(a, max_tiles, st);
  const Shape& s = a.s;
  const int R = s.G * s.L_q;
  if (s.d == 128) {
    if (R > 128) return run_tc<128, 2, 1, 2, 1, 1>(a, max_tiles, st);
    if (R > 64) return run_tc<128, 1, 1, 4, 1, 2>(a, max_tiles, st);
    if (R > 32) return run_tc<128, 1, 2, 4, 1, 2>(a, max_tiles, st);
    return run_tc<128, 1, 4, 4, 1, 2>(a, max_tiles, st);
  }
  if (R > 128) return run_tc<64, 2, 1, 4, 1, 2>(a, max_tiles, st);
  if (R > 64) return run_tc<64, 1, 1, 6, 1, 2>(a, max_tiles, st);
  if (R > 32) return run_tc<64, 1, 2, 6, 1, 2>(a, max_tiles, st);
  return run_tc<64, 1, 4, 6, 1, 2>(a, max_tiles, st);
}

}  // namespace dl
