// (a7) Intra-chunk token selection on the sm_100a tensor cores (bf16, d 128).
//
// Prefilling-dLLM abstract: the prefix is split into chunks cached once; the
// top-K chunks are kept with intra-chunk token sparsity, and the BOS token
// prepended to each chunk acts as an attention anchor.  For one selected
// chunk of one KV group, every decode query row r of the group gives
// p_rt = softmax over the chunk's content tokens t of scale q_r . k_t, the
// token's mass is tau_t = sum_r p_rt, and the top-T tokens by (mass
// descending, position ascending) are kept with the chunk's BOS.
//
// Items are (b, g, selected chunk); a persistent CTA takes items c, c + grid,
// ...  The chunk starts on a page boundary, so its first 1024 positions (the
// BOS and content tokens 1..1023) are eight tiles of two 64-key pages; a
// content token at position 1024 (a chunk of 1024 content tokens) is scored
// on the CUDA cores.  Keys are the MMA's M side: S^T [128 keys x N rows] =
// K_tile . Q^T for each tile, all eight tiles resident in TMEM at once (8 x N
// <= 512 columns).  With thread = TMEM lane = key of a tile: pass 1 takes each
// row's maximum, tile by tile as the MMAs finish (warps 4-7, one per lane
// quadrant, while the rest still streams), then reduces it; then with 8
// warps, four tiles each, pass 2 the exponentials 2^(x - max) (written back
// over S^T) and each row's sum, and pass 3 each key's mass, the sum over rows
// of its exponentials divided by the row sums.  The top-T cut is a radix
// select on the masses' bit patterns (non-negative floats order as integers)
// with the tied entries at the cut taken in position order; the kept tokens
// are written in ascending position order.
//
// Roles: warp 8 one thread: TMA of each item's query rows (contiguous rows of
// Q: the G heads' L_q positions) and of its K tiles (a ring of four), running
// ahead of the other warps: once an item's MMAs are done it loads the next
// item's rows and up to four of its tiles while the passes of the current
// item still run (the next MMAs must wait for them: S^T fills the TMEM).
// (Measured: a six-stage ring, the item's page slots loaded ahead of the issue
// loop, or that loop unrolled, made the step slower.)
// Warps 0-7, per item: warp 1 one thread: the MMAs (each tile committed to a
// barrier of its own); warps 2-3: the score of the token past the tiles;
// warps 4-7: pass 1; then all eight the passes and the selection, with a
// barrier of their own (the producer never takes it).  Every wait is bounded.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"
#include "kdigits.cuh"
#include "sm100.cuh"
#include "launch.cuh"

namespace dl {

using namespace sm100;

namespace ts {

constexpr int D = 128;
constexpr int MAX_TILES = 8;              // 8 tiles x 128 keys = 1024 positions
constexpr int STAGES = 4;
constexpr int KT_BYTES = 2 * 128 * 128;   // [d-half][128 keys][128 B]
constexpr int EP_THREADS = 256;            // warps 0-7: MMAs, last token, passes, selection
constexpr int THREADS = EP_THREADS + 32;   // + warp 8: the TMA producer
constexpr int MAXC = 1024;                // content tokens per chunk

template <int N>
struct Layout {
  static constexpr int Q_BYTES = 2 * N * 128;           // [d-half][N rows][128 B]
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + Q_BYTES;
  static constexpr int RED_OFF = K_OFF + STAGES * KT_BYTES;  // float [8 warps][N]
  static constexpr int ROW_OFF = RED_OFF + 8 * N * 4;       // float [4][N]: M, 1/Z, x_left, e_left
  static constexpr int TAU_OFF = ROW_OFF + 4 * N * 4;       // uint32 [MAXC] mass keys
  static constexpr int HIST_OFF = TAU_OFF + MAXC * 4;       // int [256]
  static constexpr int SCAN_OFF = HIST_OFF + 256 * 4;       // int [40]
  static constexpr int FLAG_OFF = SCAN_OFF + 40 * 4;        // int [8] flags (see the kernel)
  static constexpr int BAR_OFF = (FLAG_OFF + 8 * 4 + 15) / 16 * 16;
  // full, empty [STAGES]; q_full; s_done; tile_done [MAX_TILES]
  static constexpr int N_BARS = 2 * STAGES + 2 + MAX_TILES;
  static constexpr int MISC_OFF = BAR_OFF + N_BARS * 8;      // tmem slot, abort flag
  static constexpr int SMEM = MISC_OFF + 16 + 1024;          // + alignment slack
  static_assert(SMEM <= 232448, "shared memory budget");
};

// Barrier of the item warps (0-7); the producer warp never takes it.
__device__ __forceinline__ void ep_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Lane L ends with op over the 32 lanes of v[L] (v is clobbered): a butterfly
// in which each level keeps half of the entries and trades the other half.
template <bool MAX>
__device__ __forceinline__ float xreduce32(float* v, int lane) {
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

// Exclusive prefix sum of v over the item warps (256 threads); *total = the sum.
__device__ __forceinline__ int block_exclusive_sum(int v, int* s_scan, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += n;
  }
  ep_sync();
  if (lane == 31) s_scan[warp] = inc;
  ep_sync();
  int before = 0, all = 0;
  for (int w = 0; w < EP_THREADS / 32; ++w) {
    const int t = s_scan[w];
    before += w < warp ? t : 0;
    all += t;
  }
  *total = all;
  return before + inc - v;
}

// fp64 recheck of one chunk's undecided cut (certified cut, see the kernel):
// the LSE of every row over the chunk's usable content tokens, then the mass
// of every candidate (s_key[i] - 1 >= thr as fp32 bits), and keep[i] = the
// candidate is among the T largest fp64 masses (ties to the lower position).
// scratch: >= R * D + R + MAXC doubles (the K ring, free after streaming).
// Every thread of the item warps calls it.
__device__ __noinline__ void token_recheck_fp64(
    const Shape& s, const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ Kp,
    const int32_t* __restrict__ page_table, int b, int g, long long base, int n, int T,
    double thr, const uint32_t* s_key, double* scratch, uint8_t* keep_bits) {
  constexpr int RG = 16;  // rows per LSE pass
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = s.G * s.L_q;
  double* q64 = scratch;              // [R][D]
  double* lse = q64 + R * D;          // [R]
  double* tau = lse + R;              // [MAXC]: fp64 mass of each candidate, -1 otherwise
  __shared__ double s_m[EP_THREADS / 32][RG], s_z[EP_THREADS / 32][RG];
  for (int e = tid; e < R * D; e += EP_THREADS) {
    const int r = e / D, c = e % D;
    const int h = g * s.G + r / s.L_q, i = r % s.L_q;
    q64[e] = (double)__bfloat162float(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + c]);
  }
  ep_sync();
  auto usable = [&](int i) {  // content index i <-> offset i + 1
    return i < n && s_key[i] != 0u;
  };
  auto key_src = [&](int i) {
    const long long pos = base + 1 + i;
    const int slot = page_table[(size_t)b * s.n_pages + pos / 64];
    return Kp + (((size_t)slot * s.H_kv + g) * 64 + pos % 64) * D;
  };
  // fp64 logits of rows r0 .. r0+nr-1 against key i (dimension order)
  auto logits = [&](const __nv_bfloat16* k, int r0, int nr, double(&acc)[RG]) {
#pragma unroll
    for (int j = 0; j < RG; ++j) acc[j] = 0.0;
    for (int c = 0; c < D; c += 8) {
      float kv[8];
      Vec16<__nv_bfloat16>::load(k + c, kv);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        if (j < nr) {
          const double* q = q64 + (r0 + j) * D + c;
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[j] = fma(q[e], (double)kv[e], acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < RG; ++j) acc[j] *= s.scale;
  };
  // row LSEs over the usable content tokens
  for (int r0 = 0; r0 < R; r0 += RG) {
    const int nr = min(RG, R - r0);
    double m[RG], z[RG];
#pragma unroll
    for (int j = 0; j < RG; ++j) {
      m[j] = -INFINITY;
      z[j] = 0.0;
    }
    for (int i = tid; i < n; i += EP_THREADS) {
      if (!usable(i)) continue;
      double l[RG];
      logits(key_src(i), r0, nr, l);
#pragma unroll
      for (int j = 0; j < RG; ++j) {
        if (j >= nr) continue;
        if (l[j] > m[j]) {
          z[j] = z[j] * exp(m[j] - l[j]) + 1.0;
          m[j] = l[j];
        } else {
          z[j] += exp(l[j] - m[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < RG; ++j) {  // merge over the warp, then over the warps
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double om = __shfl_xor_sync(0xffffffffu, m[j], o);
        const double oz = __shfl_xor_sync(0xffffffffu, z[j], o);
        const double mm = fmax(m[j], om);
        z[j] = (m[j] == -INFINITY ? 0.0 : z[j] * exp(m[j] - mm)) +
               (om == -INFINITY ? 0.0 : oz * exp(om - mm));
        m[j] = mm;
      }
      if (lane == 0) {
        s_m[warp][j] = m[j];
        s_z[warp][j] = z[j];
      }
    }
    ep_sync();
    if (tid < nr) {
      double mm = -INFINITY;
      for (int w = 0; w < EP_THREADS / 32; ++w) mm = fmax(mm, s_m[w][tid]);
      double zz = 0.0;
      for (int w = 0; w < EP_THREADS / 32; ++w)
        if (s_m[w][tid] != -INFINITY) zz += s_z[w][tid] * exp(s_m[w][tid] - mm);
      lse[r0 + tid] = mm + log(zz);
    }
    ep_sync();
  }
  // candidates' fp64 masses, summed over the rows in order
  for (int i = tid; i < MAXC; i += EP_THREADS) {
    double t = -1.0;
    if (usable(i) && (double)__uint_as_float(s_key[i] - 1u) >= thr) {
      const __nv_bfloat16* k = key_src(i);
      t = 0.0;
      for (int r0 = 0; r0 < R; r0 += RG) {
        const int nr = min(RG, R - r0);
        double l[RG];
        logits(k, r0, nr, l);
#pragma unroll
        for (int j = 0; j < RG; ++j)
          if (j < nr) t += exp(l[j] - lse[r0 + j]);
      }
    }
    tau[i] = t;
  }
  ep_sync();
  // keep: a candidate with fewer than T better ones (mass desc, position asc)
  for (int i = tid; i < MAXC; i += EP_THREADS) {
    bool kp = false;
    const double ti = tau[i];
    if (ti >= 0.0) {
      int better = 0;
      for (int j = 0; j < MAXC; ++j) {
        const double tj = tau[j];
        better += (tj > ti || (tj == ti && j < i)) ? 1 : 0;
      }
      kp = better < T;
    }
    keep_bits[i] = kp ? 1 : 0;
  }
  ep_sync();
}

}  // namespace ts

template <int N>
__global__ void __launch_bounds__(ts::THREADS, 1)
token_select_tc_kernel(const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_q, Shape s,
                       const __nv_bfloat16* __restrict__ Q, const __nv_bfloat16* __restrict__ Kp,
                       const int32_t* __restrict__ page_table,
                       const int32_t* __restrict__ chunk_idx, int n_sel, int stride, int content,
                       int topT, const int32_t* __restrict__ Kexp, int n_chunks,
                       int32_t* __restrict__ tok_pos, int32_t* __restrict__ tok_cnt,
                       unsigned* err) {
  using namespace ts;
  using L = Layout<N>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem + L::Q_OFF;
  uint8_t* sK = smem + L::K_OFF;
  float* s_red = reinterpret_cast<float*>(smem + L::RED_OFF);   // [8][N]
  float* s_M = reinterpret_cast<float*>(smem + L::ROW_OFF);     // [N] row maxima (log2 units)
  float* s_iZ = s_M + N;                                        // [N] 1 / row sums
  float* s_xl = s_iZ + N;                                       // [N] score of the last token
  float* s_el = s_xl + N;                                       // [N] its exponential
  uint32_t* s_key = reinterpret_cast<uint32_t*>(smem + L::TAU_OFF);  // [content] mass keys
  int* s_hist = reinterpret_cast<int*>(smem + L::HIST_OFF);
  int* s_scan = reinterpret_cast<int*>(smem + L::SCAN_OFF);
  int* s_flag = reinterpret_cast<int*>(smem + L::FLAG_OFF);     // see below
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* empty = full + STAGES;
  uint64_t* q_full = empty + STAGES;
  uint64_t* s_done = q_full + 1;
  uint64_t* tile_done = s_done + 1;  // [MAX_TILES]: the tile's S^T is in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  // s_flag: [0] the last token's page is valid; [1 + p] the passes run (item
  // parity p); [3 + p] stop after the item (parity p).  One thread writes each
  // before a barrier and every thread reads it after, so that branches around
  // the barriers are uniform although the producer may raise the abort flag
  // at any time.

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(s_done, 1);
    for (int i = 0; i < MAX_TILES; ++i) mbar_init(&tile_done[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int n_bg = s.batch * s.H_kv;
  const int n_items = n_bg * n_sel;
  const int R = s.G * s.L_q;
  const int per = topT + 1;
  const int last_o = min(content, MAXC - 1);  // last position offset in the tiles
  const int n_tv = last_o / 128 + 1;          // MMA tiles of a usable chunk
  const float c2 = (float)(s.scale * 1.4426950408889634);
  // item = (b, g, selected chunk); its chunk start, or -1 if the chunk index
  // is out of range (the chunk then has no tiles)
  auto chunk_base = [&](int item) -> long long {
    const int c = chunk_idx[(size_t)(item / n_sel) * n_sel + item % n_sel];
    const long long base = (long long)c * stride;
    return (c >= 0 && base + content < (long long)s.L_ctx) ? base : -1ll;
  };

  if (warp == 8) {
    // ---------------------------------------------------------- TMA producer
    // Per item: the previous item's MMAs done (they read sQ), then the
    // group's query rows, then the K tiles through the ring.  The ring's
    // stages are freed by the MMAs, which wait for the previous item's passes
    // (its S^T is in TMEM), so up to STAGES tiles of the next item load while
    // those passes run.
    if (lane == 0) {
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_q);
      uint32_t tp = 0;  // tiles issued so far
      int k = 0;        // items with tiles so far
      bool ok = true;
      for (int item = blockIdx.x; ok && item < n_items; item += gridDim.x) {
        const long long base = chunk_base(item);
        if (base < 0) continue;
        const int bg = item / n_sel, b = bg / s.H_kv, g = bg % s.H_kv;
        const int page0 = (int)(base / 64);
        if (k > 0 && !(ok = mbar_wait(s_done, (k - 1) & 1, abort_flag))) break;
        // the R rows of the group are rows (b H + g G) L_q .. + R - 1 of Q;
        // rows past R (another group's or the zero fill past the end) only
        // fill S^T columns that every pass masks
        const int row0 = (b * s.H + g * s.G) * s.L_q;
        mbar_arrive_expect_tx(q_full, 2 * N * 128);
        for (int h = 0; h < 2; ++h) tma_load_2d(sQ + h * N * 128, &tm_q, h * 64, row0, q_full);
        for (int t = 0; t < n_tv; ++t, ++tp) {
          const int st = tp % STAGES;
          if (tp >= STAGES && !(ok = mbar_wait(&empty[st], ((tp / STAGES) - 1) & 1, abort_flag)))
            break;
          int y[2], nload = 0;
          for (int p = 0; p < 2; ++p) {
            const int lp = 2 * t + p;  // page of the chunk
            y[p] = -1;
            if (lp * 64 <= last_o) {
              const int sl = page_table[(size_t)b * s.n_pages + page0 + lp];
              if (sl >= 0 && sl < s.n_slots) {
                y[p] = (sl * s.H_kv + g) * 64;
                ++nload;
              } else {
                flag_error(err, ERR_BAD_INDEX);
              }
            }
          }
          if (nload == 0) {
            mbar_arrive(&full[st]);
            continue;
          }
          mbar_arrive_expect_tx(&full[st], nload * 16384);
          uint8_t* dst = sK + st * KT_BYTES;
          for (int p = 0; p < 2; ++p) {
            if (y[p] < 0) continue;
            for (int h = 0; h < 2; ++h)
              tma_load_2d(dst + h * 16384 + p * 8192, &tm_k, h * 64, y[p], &full[st]);
          }
        }
        ++k;
      }
      if (*abort_flag) {  // do not leave with copies in flight
        const uint32_t t0 = tp > (uint32_t)STAGES ? tp - STAGES : 0u;
        for (uint32_t t = t0; t < tp; ++t)
          for (uint32_t i = 0; i < (1u << 20) && !mbar_try_wait(&full[t % STAGES], (t / STAGES) & 1); ++i) {
          }
        for (uint32_t i = 0; i < (1u << 20) && k > 0 && !mbar_try_wait(q_full, (k - 1) & 1); ++i) {
        }
      }
    }
  } else {
    // ---------------------------------------------------------- items
    const int quad = warp & 3;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int k = 0;  // items with tiles so far (the barriers' phases)
    int it = 0;
    for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
      const int sel = item % n_sel, bg = item / n_sel;
      const int b = bg / s.H_kv, g = bg % s.H_kv;
      const int par = it & 1;
      int32_t* out = tok_pos + ((size_t)bg * n_sel + sel) * per;
      const long long cb = chunk_base(item);
      const bool chunk_ok = cb >= 0;
      const long long base = chunk_ok ? cb : 0;
      const int n_t = chunk_ok ? n_tv : 0;
      const bool has_left = chunk_ok && content >= MAXC;  // the token at offset 1024
      const int page0 = (int)(base / 64);
      // page validity of the chunk's first 16 pages (as the producer decides it)
      bool pok = false;
      if (chunk_ok && lane < 2 * MAX_TILES && lane * 64 <= last_o) {
        const int slot = page_table[(size_t)b * s.n_pages + page0 + lane];
        pok = slot >= 0 && slot < s.n_slots;
      }
      const uint32_t pvm = __ballot_sync(0xffffffffu, pok);
      auto key_ok = [&](int o) {  // offset o from the chunk start holds a usable content token
        return o >= 1 && o <= last_o && ((pvm >> (o >> 6)) & 1u);
      };
      float m[N];  // pass 1: this thread's maxima of each row (warps 4-7)
#pragma unroll
      for (int r = 0; r < N; ++r) m[r] = -INFINITY;

      if (warp == 1) {
        // -------------------------------------------------------- MMA issuer
        if (n_t > 0 && lane == 0) {
          constexpr uint32_t idesc = idesc_bf16_f32(128, N, false);
          const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK);
          bool ok = mbar_wait(q_full, k & 1, abort_flag);
          for (int t = 0; ok && t < n_t; ++t) {
            const uint32_t tt = (uint32_t)k * n_tv + t;  // ring position
            const int st = tt % STAGES;
            if (!(ok = mbar_wait(&full[st], (tt / STAGES) & 1, abort_flag))) break;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const int h = kk >> 2, k4 = kk & 3;
              const uint64_t ad = sdesc_sw128(k_base + st * KT_BYTES + h * 16384 + k4 * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(q_base + h * N * 128 + k4 * 32, 16, 1024);
              mma_f16_ss(tmem + t * N, ad, bd, idesc, kk > 0 ? 1u : 0u);
            }
            mma_commit(&empty[st]);
            mma_commit(&tile_done[t]);
          }
          if (ok) mma_commit(s_done);
        }
      } else if (warp == 2 || warp == 3) {
        // -------------------------------------------------------- last token
        const int r = threadIdx.x - 64;
        float x = -INFINITY;
        if (has_left) {
          const long long pos = base + MAXC;
          const int slot = page_table[(size_t)b * s.n_pages + pos / 64];
          const bool slot_ok = slot >= 0 && slot < s.n_slots;
          if (r == 0) {
            s_flag[0] = slot_ok ? 1 : 0;
            if (!slot_ok) flag_error(err, ERR_BAD_INDEX);
          }
          if (slot_ok && r < R && r < N) {
            const int h = g * s.G + r / s.L_q, i = r % s.L_q;
            const __nv_bfloat16* qr = Q + (((size_t)b * s.H + h) * s.L_q + i) * D;
            const __nv_bfloat16* kr = Kp + (((size_t)slot * s.H_kv + g) * 64 + pos % 64) * D;
            float acc = 0.0f;
            for (int x0 = 0; x0 < D; x0 += 8) {
              float qv[8], kv[8];
              Vec16<__nv_bfloat16>::load(qr + x0, qv);
              Vec16<__nv_bfloat16>::load(kr + x0, kv);
#pragma unroll
              for (int kx = 0; kx < 8; ++kx) acc = fmaf(qv[kx], kv[kx], acc);
            }
            x = acc * c2;
          }
        }
        if (r < N) s_xl[r] = x;
      } else if (n_t > 0 && warp >= 4) {
        // -------------------------------------------------------- pass 1
        for (int t = 0; t < n_t; ++t) {
          bool w = true;
          if (lane == 0) w = mbar_wait(&tile_done[t], k & 1, abort_flag);
          if (!__shfl_sync(0xffffffffu, w, 0)) break;
          tc_fence_after();
          const int o = t * 128 + quad * 32 + lane;
          const bool kv = key_ok(o);
#pragma unroll
          for (int c0 = 0; c0 < N; c0 += 32) {  // 32 columns at a time (registers)
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + t * N + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int r = 0; r < 32; ++r)
              m[c0 + r] =
                  fmaxf(m[c0 + r], (kv && c0 + r < R) ? __uint_as_float(v[r]) * c2 : -INFINITY);
          }
        }
      }
      // ------------------------------------------------------------ epilogue
      // every warp: TMEM lanes of its quadrant, four of the tiles
      if (threadIdx.x == 128) {
        bool ok = true;
        if (n_t > 0 && !mbar_wait(s_done, k & 1, abort_flag)) {
          *abort_flag = 1;
          ok = false;
        }
        s_flag[1 + par] = (n_t > 0 && ok && !*abort_flag) ? 1 : 0;
      }
      tc_fence_before();
      ep_sync();
      tc_fence_after();
      const bool run = s_flag[1 + par] != 0;
      if (n_t > 0) ++k;
      if (run && warp >= 4) {  // pass 1, the reduction over the lanes of each warp
#pragma unroll
        for (int r0 = 0; r0 < N; r0 += 32)
          s_red[(warp - 4) * N + r0 + lane] = xreduce32<true>(m + r0, lane);
      }
      ep_sync();
      if (run && threadIdx.x < N) {
        const int r = threadIdx.x;
        float mx = s_xl[r];
        for (int w = 0; w < 4; ++w) mx = fmaxf(mx, s_red[w * N + r]);
        s_M[r] = mx;
      }
      ep_sync();
      if (run) {
        // pass 2: exponentials (written back over S^T) and row sums
        float z[N];
#pragma unroll
        for (int r = 0; r < N; ++r) z[r] = 0.0f;
        for (int j = warp >> 2; j < n_t; j += 2) {
          const int o = j * 128 + quad * 32 + lane;
          const bool kv = key_ok(o);
#pragma unroll
          for (int c0 = 0; c0 < N; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + j * N + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int r = 0; r < 32; ++r) {
              const float mr = s_M[c0 + r];
              const float e = (kv && c0 + r < R && mr != -INFINITY)
                                  ? ex2_approx(__uint_as_float(v[r]) * c2 - mr) : 0.0f;
              z[c0 + r] += e;
              v[r] = __float_as_uint(e);
            }
            tmem_st32(tmem + lane_base + j * N + c0, v);
          }
        }
        tmem_st_wait();
#pragma unroll
        for (int r0 = 0; r0 < N; r0 += 32) s_red[warp * N + r0 + lane] = xreduce32<false>(z + r0, lane);
      }
      tc_fence_before();
      ep_sync();
      tc_fence_after();
      if (run && threadIdx.x < N) {
        const int r = threadIdx.x;
        const float mr = s_M[r];
        const float el = (s_xl[r] != -INFINITY && mr != -INFINITY) ? ex2_approx(s_xl[r] - mr) : 0.0f;
        float zt = el;
        for (int w = 0; w < 8; ++w) zt += s_red[w * N + r];
        s_el[r] = el;
        s_iZ[r] = zt > 0.0f ? 1.0f / zt : 0.0f;
      }
      ep_sync();
      // pass 3: masses, as order-preserving keys (0 = unusable token)
      if (run) {
        for (int j = warp >> 2; j < n_t; j += 2) {
          const int o = j * 128 + quad * 32 + lane;
          float tau = 0.0f;
#pragma unroll
          for (int c0 = 0; c0 < N; c0 += 32) {
            uint32_t v[32];
            tmem_ld32(tmem + lane_base + j * N + c0, v);
            tmem_ld_wait();
#pragma unroll
            for (int r = 0; r < 32; ++r) tau = fmaf(__uint_as_float(v[r]), s_iZ[c0 + r], tau);
          }
          if (o >= 1 && o <= last_o) s_key[o - 1] = key_ok(o) ? __float_as_uint(tau) + 1u : 0u;
        }
        if (has_left && threadIdx.x == 0) {
          float tau = 0.0f;
          for (int r = 0; r < N; ++r) tau = fmaf(s_el[r], s_iZ[r], tau);
          s_key[MAXC - 1] = s_flag[0] ? __float_as_uint(tau) + 1u : 0u;
        }
      }
      // the next item's MMAs may overwrite S^T once every thread is past here
      tc_fence_before();
      ep_sync();
      tc_fence_after();
      if (!chunk_ok || !run) {
        if (threadIdx.x == 0 && !chunk_ok) flag_error(err, ERR_BAD_INDEX);
        for (int e = threadIdx.x; e < per; e += EP_THREADS) out[e] = -1;
        if (threadIdx.x == 0 && sel == 0) tok_cnt[bg] = n_sel * per;
      } else {
        // top-T by (key desc, position asc): radix select of the T-th largest key
        const int n = content;
        const int T = min(topT, n);
        uint32_t prefix = 0u, mask = 0u;
        int k_rem = T;
        for (int pass = 0; pass < 4 && T > 0; ++pass) {
          const int shift = 24 - 8 * pass;
          s_hist[threadIdx.x] = 0;  // 256 bins, 256 threads
          ep_sync();
          for (int i = threadIdx.x; i < n; i += EP_THREADS) {
            const uint32_t v = s_key[i];
            if ((v & mask) == prefix) atomicAdd(&s_hist[(v >> shift) & 255u], 1);
          }
          ep_sync();
          if (warp == 0) {
            int cnt[8], tot = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              cnt[q] = s_hist[lane * 8 + q];
              tot += cnt[q];
            }
            int above = tot;  // elements in this lane's bins and every higher lane's
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
              const int x = __shfl_down_sync(0xffffffffu, above, o);
              if (lane + o < 32) above += x;
            }
            int run_cnt = above - tot;  // elements in higher lanes' bins
            for (int q = 7; q >= 0; --q) {
              if (run_cnt < k_rem && run_cnt + cnt[q] >= k_rem) {
                s_scan[32] = lane * 8 + q;
                s_scan[33] = run_cnt;
              }
              run_cnt += cnt[q];
            }
          }
          ep_sync();
          prefix |= static_cast<uint32_t>(s_scan[32]) << shift;
          mask |= 255u << shift;
          k_rem -= s_scan[33];
          ep_sync();
        }
        // Certified cut (with the chunk's exponent word): the fp32 masses are
        // within a relative eps of the exact ones (the bound of the sink search,
        // sinks_cert.cu: logits d 2^-23 ||q|| ||k|| scale, the exponentials and
        // sums on top).  Tokens below thr = v_T (1 - eps) / (1 + eps) are not in
        // the top T; if more than T reach thr, the CTA recomputes those in fp64.
        __shared__ int s_cnt_thr;
        __shared__ float s_qmax;
        __shared__ double s_thr;
        bool recheck = false;
        if (Kexp != nullptr && T > 0 && T < n) {
          if (warp == 0) {  // largest row norm of the group (rounded up)
            float qm = 0.0f;
            for (int r = lane; r < R; r += 32) {
              const int h = g * s.G + r / s.L_q, i = r % s.L_q;
              const __nv_bfloat16* qr = Q + (((size_t)b * s.H + h) * s.L_q + i) * D;
              float sq = 0.0f;
              for (int c2i = 0; c2i < D; ++c2i) {
                const float v = __bfloat162float(qr[c2i]);
                sq = __fmaf_rn(v, v, sq);
              }
              qm = fmaxf(qm, __fsqrt_ru(sq * (1.0f + 0x1p-14f)));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, o));
            if (lane == 0) {
              s_qmax = qm;
              s_cnt_thr = 0;
              const int c = (int)(base / stride);
              const double kn = (double)key_norm_of(Kexp[(size_t)bg * n_chunks + c]);
              const double delta = s.scale * (double)qm * kn * (1.0 + 0x1p-20) * (D + 2) * 0x1p-23;
              const double eps = 4.0 * delta + ((double)n / 32.0 + R + 512.0) * 0x1p-24 + 0x1p-20;
              const double vT = (double)__uint_as_float(prefix - 1u);
              s_thr = vT * (1.0 - eps) / (1.0 + eps);
            }
          }
          ep_sync();
          int cnt = 0;
          for (int i = threadIdx.x; i < n; i += EP_THREADS)
            cnt += (s_key[i] != 0u && (double)__uint_as_float(s_key[i] - 1u) >= s_thr) ? 1 : 0;
          atomicAdd(&s_cnt_thr, cnt);
          ep_sync();
          recheck = s_cnt_thr != T;
        }
        uint8_t* keep_bits = reinterpret_cast<uint8_t*>(s_hist);  // 1024 flags over hist + scan
        if (recheck) {
          ts::token_recheck_fp64(s, Q, Kp, page_table, b, g, base, n, T, s_thr, s_key,
                                 reinterpret_cast<double*>(sK), keep_bits);
        }
        // keep: above the cut, or at it among the first k_rem in position order
        constexpr int PER_T = MAXC / EP_THREADS;  // positions per thread, contiguous
        const int i0 = threadIdx.x * PER_T;
        int n_eq = 0;
#pragma unroll
        for (int q = 0; q < PER_T; ++q) {
          const int i = i0 + q;
          n_eq += (T > 0 && i < n && s_key[i] == prefix) ? 1 : 0;
        }
        int tot_eq = 0;
        int eq_before = block_exclusive_sum(n_eq, s_scan, &tot_eq);
        bool keep[PER_T];
        int n_keep = 0;
#pragma unroll
        for (int q = 0; q < PER_T; ++q) {
          const int i = i0 + q;
          bool kp = false;
          if (recheck) {
            kp = i < n && keep_bits[i] != 0;
          } else if (T > 0 && i < n) {
            const uint32_t v = s_key[i];
            if (v > prefix) {
              kp = true;
            } else if (v == prefix) {
              kp = eq_before < k_rem;
              ++eq_before;
            }
          }
          keep[q] = kp;
          n_keep += kp ? 1 : 0;
        }
        int total = 0;
        const int p0 = block_exclusive_sum(n_keep, s_scan, &total);
        int p = p0;
#pragma unroll
        for (int q = 0; q < PER_T; ++q)
          if (keep[q]) out[1 + p++] = (int)(base + 1 + i0 + q);
        if (threadIdx.x == 0) {
          out[0] = (int)base;
          if (sel == 0) tok_cnt[bg] = n_sel * per;
        }
        for (int e = 1 + total + threadIdx.x; e < per; e += EP_THREADS) out[e] = -1;
      }
      // end of the item: the scratch above is reused by the next one
      if (threadIdx.x == 0) s_flag[3 + par] = *abort_flag;
      ep_sync();
      if (s_flag[3 + par]) break;
    }
    if (threadIdx.x == 0 && *abort_flag) flag_error(err, ERR_TIMEOUT);
    if (warp == 1 && lane == 0 && *abort_flag)  // issued MMAs finish before TMEM is freed
      for (uint32_t kx = 0; kx < (1u << 16); ++kx) __nanosleep(1000);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

bool tc_map_2d(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);
int tc_sm_count();

// Whether the tensor-core kernel takes this call: bf16, head dim 128, 64-token
// pages, chunks starting on a page boundary, at most 64 query rows per group.
bool token_select_tc_supported(const Shape& s, int chunk_stride, int chunk_content) {
  return s.dtype == 0 && s.d == 128 && s.page == 64 && chunk_stride % 64 == 0 &&
         chunk_content <= ts::MAXC && s.G * s.L_q <= 64 &&
         (uint64_t)s.n_slots * s.H_kv * 64 < (1ull << 31);
}

cudaError_t launch_token_select_tc(const Shape& s, const void* Q, const void* Kp,
                                   const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                                   int chunk_stride, int chunk_content, int topT,
                                   const int32_t* Kexp, int32_t* tok_pos, int32_t* tok_cnt,
                                   unsigned* err, cudaStream_t st) {
  CUtensorMap mk;
  const int n_chunks = (s.L_ctx + chunk_stride - 1) / chunk_stride;
  if (!tc_map_2d(&mk, Kp, ts::D, (uint64_t)s.n_slots * s.H_kv * 64, 64)) return cudaErrorInvalidValue;
  const int n_rows = s.G * s.L_q <= 32 ? 32 : 64;  // N: S^T columns, the Q box's rows
  CUtensorMap mq;
  if (!tc_map_2d(&mq, Q, ts::D, (uint64_t)s.batch * s.H * s.L_q, n_rows)) return cudaErrorInvalidValue;
  // persistent: CTA c takes items c, c + grid, ... (the next one's K loads
  // while the current one's passes run); with exponent words one item per
  // CTA, since the fp64 recheck uses the K ring as scratch
  const int n_items = n_sel * s.batch * s.H_kv;
  const int sms = tc_sm_count();
  const int grid = Kexp != nullptr || n_items < sms ? n_items : sms;
  if (n_items == 0) return cudaSuccess;
  auto* q = reinterpret_cast<const __nv_bfloat16*>(Q);
  auto* k = reinterpret_cast<const __nv_bfloat16*>(Kp);
  cudaError_t e;
  if (s.G * s.L_q <= 32) {
    constexpr int smem = ts::Layout<32>::SMEM;
    if ((e = cudaFuncSetAttribute(token_select_tc_kernel<32>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    DL_LAUNCH(token_select_tc_kernel<32>, grid, ts::THREADS, smem, st, mk, mq, s, q, k, page_table,
              chunk_idx, n_sel, chunk_stride, chunk_content, topT, Kexp, n_chunks, tok_pos,
              tok_cnt, err);
  } else {
    constexpr int smem = ts::Layout<64>::SMEM;
    if ((e = cudaFuncSetAttribute(token_select_tc_kernel<64>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
      return e;
    DL_LAUNCH(token_select_tc_kernel<64>, grid, ts::THREADS, smem, st, mk, mq, s, q, k, page_table,
              chunk_idx, n_sel, chunk_stride, chunk_content, topT, Kexp, n_chunks, tok_pos,
              tok_cnt, err);
  }
  return cudaGetLastError();
}

}  // namespace dl
