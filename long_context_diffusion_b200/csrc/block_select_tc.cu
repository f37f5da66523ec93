// (a3 + a5) Block scores and sink-aware top-K selection with the logits
// taken exactly on the int8 tensor cores; one CTA per (b, g).
//
// Focus-dLLM (research.elamur.ai summary): the predicted queries score every
// KV block against the block's mean key, the most relevant blocks are kept,
// and (abstract) the attention sinks are always kept:
//   l[r][u] = scale * q_r . Kbar_u,   score[u] = sum_r softmax_u(l[r][.]).
//
// The selection is an integer result decided by real numbers, so it must be
// the one the exact scores give.  This kernel computes the dot products
// q_r . Kbar_u as integers: the pooled keys arrive as five base-128 digit
// planes with one exponent per key (kdigits.cuh, written by dl_pool_keys /
// dl_cache_write) and the query rows are cut into four digit planes here.
// One tcgen05.mma kind::i8 (s8 x s8 products, s32 sums, exact) multiplies a
// key digit plane t (M = 128 keys) with the four query planes stacked on N
// (4 x NQ rows), into tensor-memory columns starting at t * NQ: the product
// of query plane s lands at column (s + t) * NQ + row, i.e. every digit pair
// of one weight level c = s + t accumulates in the same 32-bit column.  Five
// key planes x four 32-byte k-steps = 20 MMAs per tile of 128 keys; every
// digit pair is kept.  The eight level sums of a (row, key) are combined and
// scaled in fp64, exponentiated and summed into the scores in fp64.
//
// What is not exact, and bounded (per row r, with E_max the largest key
// exponent field, NK the largest count of truncated key values, nq_r the
// row's count of truncated query values):
//   truncated query values                    <= nq_r 2^(E_r+E_max-280)
//   truncated key values                      <= NK 2^(E_r+E_max-287)
//   fp64 rounding of the combination          <= 2^(E_r+E_max-320) + 2^-49 B_r
// times scale, where B_r = scale ||q_r||_1 2^(E_max-126) bounds |l[r][u]|.
// With every logit of row r within delta_r of the exact one, every
// softmax_u(l[r][.]) is within a factor exp(+-2 delta_r), so each score is
// within a relative E = 2.5 max_r delta_r + 1e-12 (the constant covers the
// fp64 exponentials, sums and the oracle's own rounding).  The top-K set is
// certain when the K-th and (K+1)-th scores satisfy s_K (1 - E) > s_K+1 (1 + E);
// otherwise (near-ties, or |l| possibly above 700) the CTA recomputes its
// (b, g) with the fp64 kernel of block_select_common.cuh.  The exponentials
// are taken without subtracting the row maximum: |l| <= B_r <= 700 keeps
// exp(l) finite and normal, and the softmax does not depend on the shift.
//
// Roles (512 threads, 16 warps): thread 448 (warp 14, lane 0) streams the
// key digit planes by TMA through a ring of ten 16 KB stages (128 keys x
// 128 bytes, one plane each); thread 480 (warp 15, lane 0) copies the
// group's decode rows, issues the MMAs and commits them, tile by tile, into
// two alternating sets of accumulator columns.  Warpgroup w < MT drains row
// block w (query rows 8w .. 8w+7) of every tile: thread = key, the eight
// level columns read from tensor memory, combined into fp64 logits, the
// columns zeroed for the tile after next, and the exponentials kept in
// registers.  With the issuing threads in warpgroup 3, at most three row
// blocks (24 query rows) are drained; larger groups take the fp64 kernel.
// After the scores, all 16 warps run the selection (one key per thread).
// All waits are bounded; a role that gives up sets the abort flag and the
// error word (ERR_TIMEOUT), the CTA waits (bounded) for its loads and MMAs
// in flight, frees its tensor memory and writes nothing.  The decision to
// keep the fast result or recompute in fp64 is taken by one thread and
// broadcast through shared memory, so every thread takes the same branch.
#include <cudaTypedefs.h>

#include "block_select_common.cuh"
#include "fexp64.cuh"
#include "kdigits.cuh"
#include "launch.cuh"
#include "sm100.cuh"
#include "tc_common.cuh"

namespace dl {

namespace bstc {
constexpr int kThreads = bs::kThreads;                   // 512: one key per thread
constexpr int kTileKeys = 128;                           // keys per MMA tile (M)
constexpr int kPlaneBytes = kTileKeys * 128;             // one digit plane of a tile: 16 KB
constexpr int kStages = 10;                              // planes in flight per CTA
constexpr int kLevels = kKeyDigits + kQueryDigits - 1;   // digit-pair weight levels: 8
constexpr int kTmemCols = 512;
constexpr int kQOff = kStages * kPlaneBytes;             // query digit planes after the ring
constexpr int kQRawRows = 64;                            // decode rows prefetched whole
constexpr int kCtl = 480;                                // MMA-issuing thread (warp 15, lane 0)
constexpr int kProd = 448;                               // TMA-issuing thread (warp 14, lane 0)
template <int NQ>
struct Layout {
  static constexpr int QPLANE = NQ * 128;
  static constexpr int TILE_COLS = kLevels * NQ;         // tensor-memory columns of one tile
  static constexpr int NB = kQueryDigits * NQ;           // MMA N: the query planes stacked
  static constexpr int QRAW_OFF = kQOff + kQueryDigits * QPLANE;
  static constexpr int BYTES = QRAW_OFF + kQRawRows * 256;
  static constexpr int FP64_BYTES = bs::Smem<__nv_bfloat16, 128>::BYTES;
  static constexpr int SMEM = (BYTES > FP64_BYTES ? BYTES : FP64_BYTES) + 1024;  // + alignment
  static_assert(2 * TILE_COLS <= kTmemCols, "two tiles of accumulators");
};
}  // namespace bstc

// Rows of 16 doubles per lane -> lane l gets the sum over the warp of row
// (l & 15) (a transposing butterfly: 15 exchanges, then one across halves).
__device__ __forceinline__ double warp_rows_sum16(double (&v)[16], int lane) {
#pragma unroll
  for (int w = 8; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const double send = upper ? v[i] : v[i + w];
      const double keep = upper ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, w);
    }
  }
  return v[0] + __shfl_xor_sync(0xffffffffu, v[0], 16);
}

// 2^k as a double, for k in the normal range [-1022, 1023] (every use here:
// exponent fields lie in [1, 254]).
__device__ __forceinline__ double pow2i(int k) {
  return __longlong_as_double((long long)(k + 1023) << 52);
}

// Radix select over one key per thread (kThreads threads): the key of rank
// `take` (1-based) among the keys, ties broken by the thread index.  Keys
// are desc_key() of the scores (smaller = better); units that must not be
// taken carry ~0 and take is at most the number of other units.  The
// leading bits all candidate keys share are skipped (block min and max);
// then MSB first, 8 bits per pass: a histogram of the next byte among the
// keys that share the prefix fixed so far, and the byte at which the count
// reaches the rank; it stops early once the rank falls in a bin of one key.
// *k_star gets the key of that rank, *rem_out how many keys equal to it
// are within the first `take` (the lowest threads among the equal ones).
struct RadixScratch {
  int hist[256];
  int digit, rem, count;
  unsigned long long kmin[bs::kWarps], kmax[bs::kWarps], found;
};
__device__ __forceinline__ void radix_kth(uint64_t key, bool cand, int take, RadixScratch& rs,
                                          uint64_t* k_star, int* rem_out) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  unsigned long long mn = cand ? key : ~0ull, mx = cand ? key : 0ull;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
    const unsigned long long c = __shfl_xor_sync(0xffffffffu, mx, o);
    mn = a < mn ? a : mn;
    mx = c > mx ? c : mx;
  }
  if (lane == 0) {
    rs.kmin[warp] = mn;
    rs.kmax[warp] = mx;
  }
  __syncthreads();
  if (warp == 0) {  // the 16 warps' extremes, by shuffles
    mn = lane < bs::kWarps ? rs.kmin[lane] : ~0ull;
    mx = lane < bs::kWarps ? rs.kmax[lane] : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long a = __shfl_xor_sync(0xffffffffu, mn, o);
      const unsigned long long c = __shfl_xor_sync(0xffffffffu, mx, o);
      mn = a < mn ? a : mn;
      mx = c > mx ? c : mx;
    }
    if (lane == 0) {
      rs.kmin[0] = mn;
      rs.kmax[0] = mx;
    }
  }
  __syncthreads();
  mn = rs.kmin[0];
  mx = rs.kmax[0];
  // bytes above the first one where the smallest and largest candidate differ
  const int lead = mn == mx ? 64 : __clzll((long long)(mn ^ mx));
  const int first_shift = mn == mx ? -8 : 56 - (lead / 8) * 8;
  const uint64_t hi_mask = first_shift >= 56 ? 0ull : (~0ull << (first_shift + 8));
  uint64_t prefix = mn & hi_mask, fixed = hi_mask;
  int rem = take;
  for (int shift = first_shift; shift >= 0; shift -= 8) {
    if (tid < 256) rs.hist[tid] = 0;
    __syncthreads();
    const bool in = (key & fixed) == prefix;
    const unsigned dg = (unsigned)(key >> shift) & 255u;
    if (in) atomicAdd(&rs.hist[dg], 1);
    __syncthreads();
    if (warp == 0) {
      int c[8], loc = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = rs.hist[lane * 8 + j];
        loc += c[j];
      }
      int incl = loc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const int excl = incl - loc;
      if (excl < rem && incl >= rem) {
        int cum = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (cum + c[j] >= rem) {
            rs.digit = lane * 8 + j;
            rs.rem = rem - cum;
            rs.count = c[j];
            break;
          }
          cum += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= (uint64_t)rs.digit << shift;
    fixed |= (uint64_t)255 << shift;
    rem = rs.rem;
    if (rs.count == 1) {  // one key left with this prefix: it is the one
      if (in && dg == (unsigned)rs.digit) rs.found = key;
      __syncthreads();
      prefix = rs.found;
      break;
    }
  }
  *k_star = prefix;
  *rem_out = rem;
}

// Exclusive prefix count of `flag` over the CTA in thread order (kThreads
// threads), and the total: ballots per warp, the 16 warp counts scanned by
// warp 0 with shuffles.
__device__ __forceinline__ int cta_prefix_count(bool flag, int* s_cnt, int* total) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) s_cnt[warp] = __popc(bal);
  __syncthreads();
  if (warp == 0) {
    const int c = lane < bs::kWarps ? s_cnt[lane] : 0;
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane < bs::kWarps) s_cnt[32 + lane] = incl - c;
    if (lane == 31) s_cnt[64] = incl;
  }
  __syncthreads();
  *total = s_cnt[64];
  return s_cnt[32 + warp] + __popc(bal & ((1u << lane) - 1u));
}

// Counters of the int8 kernel: CTAs that kept their fast result, CTAs that
// fell back to fp64 (read and cleared by dl_read_counters).
__device__ unsigned long long g_select_counts[2];

template <int NQ, int MT>
__global__ void __launch_bounds__(bstc::kThreads, 1)
block_select_tc_kernel(const __grid_constant__ CUtensorMap kdig_map,
                       const __nv_bfloat16* __restrict__ Q, const int32_t* __restrict__ q_idx,
                       const int32_t* __restrict__ q_cnt, const float* __restrict__ Kbar,
                       const int32_t* __restrict__ Kexp, Shape s, int n_units,
                       double* __restrict__ score, int unit_size, int topK,
                       const int32_t* __restrict__ sink_pos, int n_sinks,
                       int32_t* __restrict__ blk_idx, int32_t* __restrict__ blk_cnt, int max_sel,
                       unsigned* err) {
  using namespace sm100;
  using namespace bstc;
  using L = Layout<NQ>;
  constexpr int NR = 8 * MT;  // query rows of the launch (<= NQ)
  // row block w is drained by warpgroup w; warpgroup 3 holds the issuing
  // threads and never drains, so at most three row blocks
  static_assert(NR <= NQ && NQ <= 32 && MT <= 3, "rows");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = smem;                // ring of kStages key digit planes [128 keys][128 B], swizzled
  uint8_t* sQ = smem + kQOff;        // [4 planes][NQ rows][128 B], swizzled
  uint8_t* sQraw = smem + L::QRAW_OFF;  // the group's decode rows, bf16 [G*L_q][128]
  __shared__ uint64_t full[kStages], empty[kStages], mma_done[4], tmem_free[2], qfull;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag, s_issued_tma, s_issued_mma;
  __shared__ int s_rowE[32], s_rowNq[32];
  __shared__ float s_rowL1[32];
  __shared__ int s_Emax, s_NK;
  __shared__ double s_red[bs::kWarps][32];
  __shared__ double s_iZ[32];
  __shared__ double s_E;
  __shared__ int s_keep_fast;
  __shared__ int s_qpos[256], s_qcnt;
  __shared__ double s_exp_tab[64];
  __shared__ uint8_t s_sink[bs::kMaxUnits];
  __shared__ int s_ke[bs::kMaxUnits];  // exponent field of every key (at least 1)
  __shared__ int s_cnt[72];
  __shared__ unsigned long long s_min[bs::kWarps];
  __shared__ RadixScratch s_rad;
  volatile int* abort_v = &abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bg = blockIdx.x, b = bg / s.H_kv, g = bg % s.H_kv;
  const int nt = (n_units + kTileKeys - 1) / kTileKeys;  // <= 4
  const int tl = nt - 1;                                 // the last tile
  const int J = nt * kKeyDigits;                         // digit planes to stream
  const bool q_whole = s.G * s.L_q <= kQRawRows;         // decode rows prefetched whole
  auto plane_load = [&](int j) {  // producer thread only
    const int st = j % kStages;
    mbar_arrive_expect_tx(&full[st], kPlaneBytes);
    tma_load_3d(sK + st * kPlaneBytes, &kdig_map, 0, (j / kKeyDigits) * kTileKeys,
                bg * kKeyDigits + j % kKeyDigits, &full[st]);
  };

  pdl_wait();
  // The small loads are issued first (into registers; a barrier does not
  // wait for them), so that they enter the memory queues ahead of the key
  // digit stream, which starts right after the barrier.  The control thread
  // sets up the barriers and copies the group's decode rows.
  if (tid == kCtl) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 4; ++i) mbar_init(&mma_done[i], 1);
    mbar_init(&tmem_free[0], 128 * MT);  // the draining warpgroups
    mbar_init(&tmem_free[1], 128 * MT);
    mbar_init(&qfull, 1);
    abort_flag = 0;
    s_Emax = 1;
    s_NK = 0;
    s_issued_tma = 0;
    s_issued_mma = 0;
    fence_mbar_init();
    prefetch_tmap(&kdig_map);
    if (q_whole) {
      const uint32_t bytes = (uint32_t)(s.G * s.L_q * 256);
      mbar_arrive_expect_tx(&qfull, bytes);
      bulk_load(sQraw, Q + ((size_t)b * s.H + (size_t)g * s.G) * s.L_q * 128, bytes, &qfull);
    }
  }
  const int key = tid;
  const bool key_ok = key < n_units;
  const int ke = key_ok ? __ldg(Kexp + (size_t)bg * n_units + key) : 0;
  int qcnt = 0;
  if (warp == 1) {
    for (int i = lane; i < s.L_q; i += 32) s_qpos[i] = q_idx ? q_idx[(size_t)b * s.L_q + i] : i;
    if (lane == 0) qcnt = q_idx ? q_cnt[b] : s.L_q;
  }
  const int sp0 = (warp == 2 && lane < n_sinks) ? sink_pos[(size_t)b * n_sinks + lane] : -1;
  const double tabv = tid < 64 ? kPow2Frac64[tid] : 0.0;
  s_sink[tid] = 0;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, kTmemCols);
    tmem_relinquish();
    pdl_trigger();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  if (tid == kProd) {  // the key digit stream: the first kStages planes
    const int n0 = J < kStages ? J : kStages;
    for (int j = 0; j < n0; ++j) plane_load(j);
    s_issued_tma = n0;
  }
  if (warp == 1 && lane == 0) s_qcnt = qcnt;
  if (tid < 64) s_exp_tab[tid] = tabv;
  if (warp == 2 && lane < n_sinks && sp0 >= 0) {  // sink units (kept whatever their score)
    const long long u = sp0 / unit_size;
    if (u < n_units) s_sink[u] = 1;
    else flag_error(err, ERR_BAD_INDEX);
  }
  for (int q = 32 + tid; q < n_sinks; q += kThreads) {  // more than 32 sinks: plain loads
    const int pos = sink_pos[(size_t)b * n_sinks + q];
    if (pos >= 0) {
      const long long u = pos / unit_size;
      if (u < n_units) s_sink[u] = 1;
      else flag_error(err, ERR_BAD_INDEX);
    }
  }

  // every digit-pair MMA accumulates: the two tiles' columns start at zero
  // (warps 0-7 for both buffers, each its 32 lanes; later rows are zeroed
  // by the warps that drain them)
  auto zero_cols = [&](int buf) {  // this warp's 32 lanes of one tile buffer
    uint32_t z[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) z[i] = 0u;
    const uint32_t base = tmem + ((uint32_t)((warp & 3) * 32) << 16) + buf * L::TILE_COLS;
#pragma unroll
    for (int c = 0; c < L::TILE_COLS; c += 32) tmem_st32(base + c, z);
    tmem_st_wait();
  };
  if (warp < 8) zero_cols(warp >> 2);

  // key exponents: block maxima for the bound
  int Eu = 1;
  {
    int em = 1, nk = 0;
    if (key_ok) {
      Eu = max(ke & 255, 1);
      em = Eu;
      nk = (ke >> 8) & 255;
    }
    s_ke[tid] = Eu;
    em = __reduce_max_sync(0xffffffffu, em);
    nk = __reduce_max_sync(0xffffffffu, nk);
    if (lane == 0) {
      atomicMax(&s_Emax, em);
      atomicMax(&s_NK, nk);
    }
  }
  __syncthreads();  // s_qpos, s_qcnt, s_exp_tab, s_sink
  int nq = min(max(s_qcnt, 0), s.L_q);
  if (nq * s.G > NR) {  // more rows than the caller's bound: reported, rows cut
    if (tid == 0) flag_error(err, ERR_BAD_INDEX);
    nq = NR / s.G;
  }
  const int R = nq * s.G;  // <= NR

  // ---- query rows -> four digit planes (row r = tid / 16, dims 8p .. 8p+7)
  {
    const int r = tid >> 4, p = tid & 15;
    uint4 raw = make_uint4(0u, 0u, 0u, 0u);
    bool have = false;
    int hrow = 0;
    if (r < R) {
      const int i = s_qpos[r % nq];
      if (i >= 0 && i < s.L_q) {
        have = true;
        hrow = (r / nq) * s.L_q + i;  // row of the group's block [G][L_q]
      } else if (p == 0) {
        flag_error(err, ERR_BAD_INDEX);
      }
    }
    if (q_whole) {
      if (!__all_sync(0xffffffffu, mbar_wait(&qfull, 0, abort_v))) have = false;
      if (have) raw = *reinterpret_cast<const uint4*>(sQraw + hrow * 256 + 16 * p);
    } else if (have) {
      raw = __ldg(reinterpret_cast<const uint4*>(
          Q + (((size_t)b * s.H + (size_t)g * s.G) * s.L_q + hrow) * 128 + 8 * p));
    }
    uint32_t hv[8];
    hv[0] = raw.x & 0xFFFFu; hv[1] = raw.x >> 16; hv[2] = raw.y & 0xFFFFu; hv[3] = raw.y >> 16;
    hv[4] = raw.z & 0xFFFFu; hv[5] = raw.z >> 16; hv[6] = raw.w & 0xFFFFu; hv[7] = raw.w >> 16;
    int E = 1;
    float l1 = 0.0f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      E = max(E, exp_field_bf16(hv[k]));
      l1 += fabsf(__uint_as_float(hv[k] << 16));
    }
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
      E = max(E, __shfl_xor_sync(0xffffffffu, E, o));
      l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    }
    int dg[8][kQueryDigits];
    int nin = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) nin += query_digits(hv[k], E, dg[k]) ? 1 : 0;
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) nin += __shfl_xor_sync(0xffffffffu, nin, o);
    if (r < NQ) {
#pragma unroll
      for (int pl = 0; pl < kQueryDigits; ++pl) {
        uint8_t* dst = sQ + pl * L::QPLANE + r * 128 + (((p >> 1) ^ (r & 7)) << 4) + ((p & 1) << 3);
        *reinterpret_cast<uint2*>(dst) =
            make_uint2(pack4_i8(dg[0][pl], dg[1][pl], dg[2][pl], dg[3][pl]),
                       pack4_i8(dg[4][pl], dg[5][pl], dg[6][pl], dg[7][pl]));
      }
    }
    if (p == 0) {
      s_rowE[r] = E;
      s_rowNq[r] = nin;
      s_rowL1[r] = l1 * 1.0001f;  // fp32 sum of 128 magnitudes, rounded up generously
    }
  }
  fence_proxy_async_smem();  // the query digits are read by the tensor cores
  tc_fence_before();         // and the zeroed columns are written to
  __syncthreads();

  // ---- MMAs (thread kCtl): digit plane j = (tile t, key plane tk) times
  // the stacked query planes into tile t's columns tk*NQ .. tk*NQ + 4*NQ,
  // four k-steps of 32 bytes.  Refills (thread kProd): the ring stage of
  // plane j gets plane j + kStages once plane j's MMAs are done.
  if (tid == kCtl) {
    constexpr uint32_t IDESC = idesc_s8_s32(kTileKeys, L::NB);
    const uint64_t kdesc0 = sdesc_sw128(smem_u32(sK), 16, 1024);
    const uint64_t qdesc0 = sdesc_sw128(smem_u32(sQ), 16, 1024);
    bool ok = true;
    int j = 0;
    for (; ok && j < J; ++j) {
      const int t = j / kKeyDigits, tk = j % kKeyDigits, st = j % kStages;
      if (!(ok = mbar_wait(&full[st], (j / kStages) & 1, abort_v))) break;
      if (tk == 0 && t >= 2 &&
          !(ok = mbar_wait(&tmem_free[t & 1], ((t - 2) >> 1) & 1, abort_v)))
        break;
      tc_fence_after();
      const uint32_t dcol = tmem + (t & 1) * L::TILE_COLS + tk * NQ;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_i8_ss(dcol, kdesc0 + (uint64_t)((st * kPlaneBytes + kk * 32) >> 4),
                  qdesc0 + (uint64_t)((kk * 32) >> 4), IDESC, 1u);
      mma_commit(&empty[st]);
      if (tk == kKeyDigits - 1) mma_commit(&mma_done[t]);
    }
    s_issued_mma = j;
    if (!ok) flag_error(err, ERR_TIMEOUT);
  } else if (tid == kProd) {
    bool ok = true;
    int j = 0;
    for (; ok && j + kStages < J; ++j) {
      const int st = j % kStages;
      if (!(ok = mbar_wait(&empty[st], (j / kStages) & 1, abort_v))) break;
      plane_load(j + kStages);
    }
    s_issued_tma = (J < kStages ? J : kStages) + j;
    if (!ok) flag_error(err, ERR_TIMEOUT);
  }
  __syncwarp();

  // ---- drains: every tile by every warpgroup w < MT, row block w (rows
  // 8w .. 8w+7), thread = key 128 t + (threadIdx.x & 127).  Level sums ->
  // fp64 logits -> softmax numerators p = exp(l) without a shift (|l| <= B_r;
  // if B_r <= 700 fails below, the fp64 kernel redoes the (b, g)); the p
  // values stay in registers (one row block of four keys) and each warp adds
  // its partial row sums to s_red[warp][row].
  const int wg = warp >> 2;
  const double sc = s.scale;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  double pv[4][8];  // [tile][row of the block]
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int i = 0; i < 8; ++i) pv[t][i] = 0.0;
  double zr[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) zr[i] = 0.0;
  const bool drains = wg < MT;
  const int row0 = wg * 8;
  int erow[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) erow[i] = s_rowE[(row0 + i) & 31];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    if (t < nt) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&mma_done[t], 0, abort_v));
      const int tkey = t * kTileKeys + (tid & 127);
      const bool kok = tkey < n_units;
      if (ok && drains) {
        const int et = kok ? s_ke[tkey] : 1;
        tc_fence_after();
        const uint32_t base = tmem + lane_base + (t & 1) * L::TILE_COLS + row0;
        // V = h0 2^42 + h1 2^28 + h2 2^14 + h3, h_k = A_2k * 128 + A_2k+1 (int32),
        // the eight levels read in two halves
        double l[8];
        {
          uint32_t a[4][8];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld8(base + c * NQ, a[c]);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int h0 = (int)a[0][i] * 128 + (int)a[1][i];
            const int h1 = (int)a[2][i] * 128 + (int)a[3][i];
            l[i] = fma((double)h1, 0x1p28, (double)h0 * 0x1p42);
          }
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld8(base + (4 + c) * NQ, a[c]);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int h2 = (int)a[0][i] * 128 + (int)a[1][i];
            const int h3 = (int)a[2][i] * 128 + (int)a[3][i];
            const double v = fma((double)h2, 0x1p14, l[i]) + (double)h3;
            l[i] = v * (sc * pow2i(erow[i] + et - 315));
          }
        }
        if (t + 2 < nt) {  // tile t + 2 accumulates in these columns: zero them
          uint32_t z[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) z[i] = 0u;
#pragma unroll
          for (int c = 0; c < kLevels; ++c) tmem_st8(base + c * NQ, z);
          tmem_st_wait();
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const double pe = exp_fp64(l[i], s_exp_tab);
          pv[t][i] = (kok && row0 + i < R) ? pe : 0.0;
          zr[i] += pv[t][i];
        }
      }
      tc_fence_before();
      if (drains && t + 2 < nt) mbar_arrive(&tmem_free[t & 1]);  // read and zeroed
    }
  }
  // this warp's partial row sums: the 8 rows of its block over its 32 keys
  if (drains) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      double v = zr[i];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      zr[i] = v;
    }
    if (lane < 8) {
      double v = zr[0];
#pragma unroll
      for (int i = 1; i < 8; ++i) v = lane == i ? zr[i] : v;
      s_red[warp][row0 + lane] = v;
    }
  }
  tc_fence_before();
  __syncthreads();
  // every load and MMA issued has completed unless a wait gave up; then wait
  // (bounded) for what is in flight before the tensor memory is freed
  if (*abort_v) {
    if (tid == kCtl) {  // bounded waits that ignore the abort flag
      for (int j = 0; j < s_issued_tma; ++j)
        for (uint32_t i = 0;
             i < kWaitLimit && !mbar_try_wait(&full[j % kStages], (j / kStages) & 1); ++i) {
        }
      for (int j = 0; j < s_issued_mma; ++j)
        for (uint32_t i = 0;
             i < kWaitLimit && !mbar_try_wait(&empty[j % kStages], (j / kStages) & 1); ++i) {
        }
      if (q_whole)
        for (uint32_t i = 0; i < kWaitLimit && !mbar_try_wait(&qfull, 0); ++i) {
        }
      flag_error(err, ERR_TIMEOUT);
    }
    __syncthreads();
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (*abort_v) return;

  // ---- Z_r (sum of the four warps of the row's block) and the bound of the
  // logit errors
  if (tid < 32) {
    const int r = tid, w0 = (r >> 3) * 4;
    const double z = (r < 8 * MT) ? (s_red[w0][r] + s_red[w0 + 1][r]) + (s_red[w0 + 2][r] + s_red[w0 + 3][r]) : 0.0;
    s_iZ[r] = (r < R && z > 0.0) ? 1.0 / z : 0.0;
  } else if (warp == 9) {
    const int Emax = s_Emax, NK = s_NK;
    double dmax = 0.0, bmax = 0.0;
    if (lane < R) {
      const int er = s_rowE[lane];
      const double b_r = sc * (double)s_rowL1[lane] * pow2i(Emax - 126) * 1.001;
      const double d_r = sc * ((double)s_rowNq[lane] * pow2i(er + Emax - 280) +
                               (double)NK * pow2i(er + Emax - 287) + pow2i(er + Emax - 320)) +
                         0x1p-49 * b_r;
      dmax = d_r;
      bmax = b_r;
    }
    dmax = warp_max_d(dmax);
    bmax = warp_max_d(bmax);
    if (lane == 0) {
      s_E = 2.5 * dmax + 1e-12;             // relative bound of every score
      s_keep_fast = bmax <= 700.0 ? 1 : 0;  // exp(l) stays finite and normal
    }
  }
  __syncthreads();
  // scores: each warpgroup's row-block partial of its four keys, then the
  // sum over the row blocks (the ring is free: every MMA is done)
  double* sPart = reinterpret_cast<double*>(sK);  // [MT][512]
  if (drains) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      double a0 = 0.0;
#pragma unroll
      for (int i = 0; i < 8; ++i) a0 = fma(pv[t][i], s_iZ[row0 + i], a0);
      sPart[wg * 512 + t * kTileKeys + (tid & 127)] = a0;
    }
  }
  __syncthreads();
  double my = 0.0;
  for (int w = 0; w < MT; ++w) my += sPart[w * 512 + tid];
  const double E = s_E;
  const bool bounded = s_keep_fast != 0;

  // ---- selection (radix select of the topK non-sink units) and its certificate
  const bool is_sink = key_ok && s_sink[tid];
  const int n_sb = __syncthreads_count(is_sink);
  const int n_cand = n_units - n_sb;
  const int take = topK < n_cand ? topK : n_cand;
  const uint64_t mykey = (key_ok && !is_sink) ? desc_key(my) : ~0ull;
  bool sel = false;
  bool fast = bounded || R == 0;
  if (take >= 1) {
    uint64_t kstar;
    int rem;
    radix_kth(mykey, key_ok && !is_sink, take, s_rad, &kstar, &rem);
    // the keys equal to k* are taken in thread order, rem of them
    const int n_eq = __syncthreads_count(mykey == kstar);
    if (n_eq == 1) {
      sel = mykey <= kstar;
    } else {
      int tot = 0;
      const int eq_before = cta_prefix_count(mykey == kstar, s_cnt, &tot);
      sel = mykey < kstar || (mykey == kstar && eq_before < rem);
    }
    if (take < n_cand && R > 0) {
      // the best key not taken: the next equal one, or the smallest above k*
      unsigned long long above = mykey > kstar ? mykey : ~0ull;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long v = __shfl_xor_sync(0xffffffffu, above, o);
        above = v < above ? v : above;
      }
      if (lane == 0) s_min[warp] = above;
      __syncthreads();
      if (tid == 0) {  // one thread decides, for every thread
        unsigned long long next = n_eq > rem ? kstar : ~0ull;
        for (int w = 0; w < bs::kWarps; ++w) next = s_min[w] < next ? s_min[w] : next;
        const double s_k = score_of_desc_key(kstar), s_k1 = score_of_desc_key(next);
        s_keep_fast = (fast && s_k * (1.0 - E) > s_k1 * (1.0 + E)) ? 1 : 0;
      }
      __syncthreads();
      fast = s_keep_fast != 0;
    }
  }
  if (R == 0) fast = true;  // no rows: every score is exactly 0 on both sides
  if (fast) {
    if (key_ok) score[(size_t)bg * n_units + key] = my;
    const bool keep = key_ok && (sel || is_sink);
    int total = 0;
    const int pos = cta_prefix_count(keep, s_cnt, &total);
    int32_t* out = blk_idx + (size_t)bg * max_sel;
    if (keep && pos < max_sel) out[pos] = key;
    for (int e = total + tid; e < max_sel; e += kThreads) out[e] = -1;
    if (tid == 0) {
      blk_cnt[bg] = total < max_sel ? total : max_sel;
      atomicAdd(&g_select_counts[0], 1ull);
    }
  } else {
    __syncthreads();  // everyone is past the scratch before it is reused
    block_select_fp64<__nv_bfloat16, 128, MT>(Q, q_idx, q_cnt, Kbar, s, n_units, score,
                                               unit_size, topK, sink_pos, n_sinks, blk_idx,
                                               blk_cnt, max_sel, err, smem);
    if (tid == 0) atomicAdd(&g_select_counts[1], 1ull);
  }
}

// Whether the int8 kernel takes this call.
bool block_select_tc_supported(const Shape& s, int rows, int n_units) {
  return s.dtype == 0 && s.d == 128 && rows <= 24 && n_units <= bs::kMaxUnits &&
         !(kernel_flags() & DL_FLAG_SCORE_FP64);
}

cudaError_t launch_block_select_tc(const Shape& s, const void* Q, const int32_t* q_idx,
                                   const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                                   const int32_t* Kexp, int n_units, double* score,
                                   int unit_size, int topK, const int32_t* sink_pos,
                                   int n_sinks, int32_t* blk_idx, int32_t* blk_cnt, int max_sel,
                                   int rows, unsigned* err, cudaStream_t st) {
  if (s.G * s.L_q <= bstc::kQRawRows &&
      (reinterpret_cast<uintptr_t>(Q) & 15u) != 0)  // the whole-block copy needs 16 B
    return cudaErrorInvalidValue;
  CUtensorMap map;
  if (!tc_map_i8_3d(&map, Kdig, 128, (uint64_t)n_units, (uint64_t)s.batch * s.H_kv * kKeyDigits,
                    bstc::kTileKeys))
    return cudaErrorInvalidValue;
  cudaError_t e;
#define DL_BSTC(NQ_, MT_)                                                                      \
  {                                                                                           \
    auto k = block_select_tc_kernel<NQ_, MT_>;                                                \
    constexpr int smem = bstc::Layout<NQ_>::SMEM;                                             \
    if ((e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=   \
        cudaSuccess)                                                                          \
      return e;                                                                               \
    DL_LAUNCH(k, s.batch * s.H_kv, bstc::kThreads, smem, st, map,                             \
              reinterpret_cast<const __nv_bfloat16*>(Q), q_idx, q_cnt, Kbar, Kexp, s, n_units, \
              score, unit_size, topK, sink_pos, n_sinks, blk_idx, blk_cnt, max_sel, err);     \
  }
  switch ((rows + 7) / 8) {
    case 0:
    case 1: DL_BSTC(16, 1) break;
    case 2: DL_BSTC(16, 2) break;
    default: DL_BSTC(32, 3) break;
  }
#undef DL_BSTC
  return cudaGetLastError();
}

// Reads and clears the counters (host side of dl_read_counters).
cudaError_t read_select_counts(unsigned long long* fast, unsigned long long* fallback) {
  unsigned long long v[2] = {0, 0};
  cudaError_t e = cudaMemcpyFromSymbol(v, g_select_counts, sizeof(v));
  if (e != cudaSuccess) return e;
  const unsigned long long z[2] = {0, 0};
  e = cudaMemcpyToSymbol(g_select_counts, z, sizeof(z));
  if (fast) *fast = v[0];
  if (fallback) *fallback = v[1];
  return e;
}

}  // namespace dl
