// (a4) Certified sink cut: the sinks are the n_sinks columns of largest
// attention mass (ties to the lower position), an integer result decided by
// real numbers.  The mass passes (sinks.cu, sinks_tc.cu) compute the masses
// in fp32; this file makes the cut the one the exact masses give.
//
// Focus-dLLM abstract: sinks are the highly influential attention columns,
// identified once and reused.  mass[t] = sum over heads h and predicted rows
// r of exp(l_hrt - LSE_hr), l_hrt = scale q_hr . k_t, LSE_hr over the
// context and the decode block.
//
// Error model of the fp32 masses (every term, relative): a logit is a dot
// product of d exact products (bf16 x bf16, or fp32 x fp32 on the CUDA
// cores) summed in fp32; its error is taken as at most d 2^-23 sum_i |q_i k_i|
// <= d 2^-23 ||q|| ||k|| (one fp32 ulp per addition with truncation: the
// tensor cores' accumulation is assumed to do no worse).  With B = the
// largest scale ||q_hr|| ||k_t|| (||k_t|| bounded by the norm field that
// dl_pool_keys / dl_cache_write keep in Kexp, and by the decode keys' norms
// taken here), every logit is within delta = (d + 2) 2^-23 B, the row LSE
// within delta plus its summation and exponential error, and every mass
// term within a relative 2 delta + that error; the sums add at most one fp32
// rounding per term.  So every fp32 mass is within a relative
//   eps = 4 delta + (L_ctx / 32 + H nq + 512) 2^-24 + 2^-20
// of the exact one (the constant covers the fast exponentials, 2^-21 each,
// and the sums of at most L_ctx / 32 + H nq + 512 terms along any chain).
//
// Cut: v_n = the n-th largest fp32 mass; a column whose fp32 mass is below
// thr = v_n (1 - eps) / (1 + eps) has an exact mass below every exact mass of
// the n columns at or above v_n, so it is not a sink.  If exactly n columns
// reach thr they are the sinks (certified).  Otherwise the columns reaching
// thr (the candidates; every column when there are more than kCap) get their
// masses again in fp64 -- every row's LSE over all keys, then each
// candidate's sum -- and the top n of those are the sinks.  The fp64 masses
// are exact up to fp64 rounding (products of bf16 or fp32 values are exact
// in fp64).
//
// Kernels (after the top-n kernel of sinks.cu has written its n columns):
// bound (CTA per (b, g): the group's largest ||q|| ||k||), band count (CTAs
// over slices of the columns: eps, v_n = the smallest of the n masses, the
// columns reaching thr), band final (CTA per sequence: certified, or the
// candidates in position order); lse64 (CTA per (512-key chunk, b, h): fp64
// logits of up to 32 predicted rows at a time in shared memory, the chunk's
// (max, sum) per row); lse64 merge; candidate mass (CTA per (candidate, b));
// pick (one CTA per sequence: n rounds of a block argmax in (mass desc,
// position asc) order).  Certified sequences make the last four return at
// once.
#include "common.cuh"
#include "internal.h"
#include "kdigits.cuh"
#include "launch.cuh"

namespace dl {

namespace sc {
constexpr int kCap = 512;         // candidates rechecked one by one
constexpr int kChunk = 512;       // keys per fp64 LSE CTA
constexpr int kRows = 32;         // predicted rows per fp64 pass
constexpr int kThreads = 256;     // fp64 kernels
constexpr int kBandThreads = 1024;
constexpr int kMaxKvHeads = 256;
}  // namespace sc

struct SinkCertWs {
  int* flag;      // [b]: 0 certified, 1 candidates, 2 every column
  int* count;     // [b]: columns reaching the threshold
  float* qk;      // [b][H_kv]: largest ||q|| ||k|| bound of the KV group
  double* thr;    // [b]: the threshold
  int* cand;      // [b][kCap], ascending positions
  double* m64;    // [b][max(kCap, L_ctx)]: fp64 masses of the candidates
  double2* part;  // [b*H][n_chunks][L_q]: (max, sum) of each chunk
  double* lse;    // [b*H][L_q]
};

static int cert_chunks(const Shape& s) {
  return (int)(((long long)s.L_ctx + s.L_q + sc::kChunk - 1) / sc::kChunk);
}
__host__ __device__ inline int cert_m64_len(const Shape& s) {
  return s.L_ctx > sc::kCap ? s.L_ctx : sc::kCap;
}

size_t sink_cert_workspace(const Shape& s) {
  const size_t bh = (size_t)s.batch * s.H;
  return round256((size_t)s.batch * 2 * sizeof(int)) +
         round256((size_t)s.batch * s.H_kv * sizeof(float)) +
         round256((size_t)s.batch * sizeof(double)) +
         round256((size_t)s.batch * sc::kCap * sizeof(int)) +
         round256((size_t)s.batch * cert_m64_len(s) * sizeof(double)) +
         round256(bh * cert_chunks(s) * s.L_q * sizeof(double2)) +
         round256(bh * s.L_q * sizeof(double));
}

static SinkCertWs sink_cert_ws(void* ws, const Shape& s) {
  char* p = reinterpret_cast<char*>(ws);
  const size_t bh = (size_t)s.batch * s.H;
  SinkCertWs w;
  w.flag = reinterpret_cast<int*>(p);
  w.count = w.flag + s.batch;
  p += round256((size_t)s.batch * 2 * sizeof(int));
  w.qk = reinterpret_cast<float*>(p);
  p += round256((size_t)s.batch * s.H_kv * sizeof(float));
  w.thr = reinterpret_cast<double*>(p);
  p += round256((size_t)s.batch * sizeof(double));
  w.cand = reinterpret_cast<int*>(p);
  p += round256((size_t)s.batch * sc::kCap * sizeof(int));
  w.m64 = reinterpret_cast<double*>(p);
  p += round256((size_t)s.batch * cert_m64_len(s) * sizeof(double));
  w.part = reinterpret_cast<double2*>(p);
  p += round256(bh * cert_chunks(s) * s.L_q * sizeof(double2));
  w.lse = reinterpret_cast<double*>(p);
  return w;
}

template <typename T>
__device__ __forceinline__ float to_float(T x);
template <>
__device__ __forceinline__ float to_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ float to_float<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

// Upper bound of the Euclidean norm of n values (fp32 sum of squares, the
// rounding covered by the factor on the sum, square root rounded up).
__device__ __forceinline__ float norm_up(float sq_sum) {
  return __fsqrt_ru(sq_sum * (1.0f + 0x1p-14f));
}

// ---------------------------------------------------------------- band
// (1) CTA per (b, g): the group's bound ||q|| ||k|| -- the largest key norm
// (the blocks' norm fields and the decode keys) times the largest norm of the
// predicted rows of the group's heads.  Also clears the sequence's count.
template <typename T, int D>
__global__ void __launch_bounds__(256)
sink_bound_kernel(Shape s, const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                  const int32_t* __restrict__ q_cnt, const T* __restrict__ Kd,
                  const int32_t* __restrict__ Kexp, int n_units, SinkCertWs w) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_kn, s_qn;  // float bits (non-negative: int order = float order)
  const int bg = blockIdx.x, b = bg / s.H_kv, g = bg % s.H_kv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int NW = 256 / 32;
  if (tid == 0) {
    s_kn = 0;
    s_qn = 0;
    if (g == 0) w.count[b] = 0;
  }
  __syncthreads();
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  float kn = 0.0f;
  for (int u = tid; u < n_units; u += blockDim.x)
    kn = fmaxf(kn, key_norm_of(__ldg(Kexp + (size_t)bg * n_units + u)));
  for (int i = warp; i < s.L_q; i += NW) {  // warp per decode key
    const T* k = Kd + ((size_t)bg * s.L_q + i) * D;
    float sq = 0.0f;
    for (int c = lane; c < D; c += 32) {
      const float v = to_float(k[c]);
      sq = __fmaf_rn(v, v, sq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    kn = fmaxf(kn, norm_up(sq));
  }
  float qn = 0.0f;
  for (int e = warp; e < s.G * nq; e += NW) {  // warp per predicted row of the group
    const int h = g * s.G + e / nq, r = e % nq;
    const int i = q_idx[(size_t)b * s.L_q + r];
    float sq = 0.0f;
    if (i >= 0 && i < s.L_q) {
      const T* q = Q + (((size_t)b * s.H + h) * s.L_q + i) * D;
      for (int c = lane; c < D; c += 32) {
        const float v = to_float(q[c]);
        sq = __fmaf_rn(v, v, sq);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    qn = fmaxf(qn, norm_up(sq));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kn = fmaxf(kn, __shfl_xor_sync(0xffffffffu, kn, o));
    qn = fmaxf(qn, __shfl_xor_sync(0xffffffffu, qn, o));
  }
  if (lane == 0) {
    atomicMax(&s_kn, __float_as_int(kn));
    atomicMax(&s_qn, __float_as_int(qn));
  }
  __syncthreads();
  if (tid == 0) w.qk[bg] = __fmul_ru(__int_as_float(s_qn), __int_as_float(s_kn));
}

// eps and thr of sequence b (every caller computes the same numbers).
__device__ __forceinline__ double sink_threshold(const Shape& s, const SinkCertWs& w, int b,
                                                 int nq, const float* m, const int32_t* top,
                                                 int n_sinks, int D) {
  float qk = 0.0f;
  for (int g = 0; g < s.H_kv; ++g) qk = fmaxf(qk, w.qk[(size_t)b * s.H_kv + g]);
  const double B = s.scale * (double)qk * (1.0 + 0x1p-20);
  const double delta = B * (D + 2) * 0x1p-23;
  const double eps = 4.0 * delta + ((double)s.L_ctx / 32.0 + (double)s.H * nq + 512.0) * 0x1p-24 +
                     0x1p-20;
  float vn = INFINITY;  // the smallest mass among the top n
  for (int i = 0; i < n_sinks; ++i) {
    const int p = top[i];
    vn = fminf(vn, (p >= 0 && p < s.L_ctx) ? fmaxf(m[p], 0.0f) : 0.0f);
  }
  return (double)vn * (1.0 - eps) / (1.0 + eps);
}

// (2) CTA per (slice, b): how many columns of the slice reach thr.
__global__ void __launch_bounds__(256)
sink_band_count_kernel(Shape s, const int32_t* __restrict__ q_cnt, const float* __restrict__ mass,
                       int n_sinks, const int32_t* __restrict__ sink_pos, SinkCertWs w, int D) {
  pdl_trigger();
  pdl_wait();
  __shared__ double s_thr;
  __shared__ int s_cnt;
  const int b = blockIdx.y, tid = threadIdx.x;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  if (nq == 0) return;
  const float* m = mass + (size_t)b * s.L_ctx;
  if (tid == 0) {
    s_thr = sink_threshold(s, w, b, nq, m, sink_pos + (size_t)b * n_sinks, n_sinks, D);
    s_cnt = 0;
    if (blockIdx.x == 0) w.thr[b] = s_thr;
  }
  __syncthreads();
  const double thr = s_thr;
  const long long per = ((long long)s.L_ctx + gridDim.x - 1) / gridDim.x;
  const long long t0 = (long long)blockIdx.x * per;
  const long long t1 = min(t0 + per, (long long)s.L_ctx);
  int cnt = 0;
  for (long long t = t0 + tid; t < t1; t += blockDim.x) cnt += (double)fmaxf(m[t], 0.0f) >= thr;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
  if ((tid & 31) == 0 && cnt) atomicAdd(&s_cnt, cnt);
  __syncthreads();
  if (tid == 0 && s_cnt) atomicAdd(w.count + b, s_cnt);
}

// (3) CTA per sequence: certified when exactly n columns reach thr (the top
// n of sink_pos stand); otherwise the candidates in position order.
__global__ void __launch_bounds__(sc::kBandThreads)
sink_band_final_kernel(Shape s, const int32_t* __restrict__ q_cnt,
                       const float* __restrict__ mass, int n_sinks, SinkCertWs w,
                       int32_t* __restrict__ sink_pos) {
  pdl_trigger();
  pdl_wait();
  __shared__ int s_warp[33];
  const int b = blockIdx.x, tid = threadIdx.x;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  const int total = w.count[b];
  if (nq == 0 || total == n_sinks) {  // no rows: every mass is 0, the top n are 0 .. n-1
    if (tid == 0) w.flag[b] = 0;
    return;
  }
  const float* m = mass + (size_t)b * s.L_ctx;
  const double thr = w.thr[b];
  int done = 0;
  for (int t0 = 0; t0 < s.L_ctx && total <= sc::kCap; t0 += blockDim.x) {
    const int t = t0 + tid;
    const bool in = t < s.L_ctx && (double)fmaxf(m[t], 0.0f) >= thr;
    int chunk_total = 0;
    const int pos = done + block_exclusive_count(in, s_warp, &chunk_total);
    if (in && pos < sc::kCap) w.cand[(size_t)b * sc::kCap + pos] = t;
    done += chunk_total;
  }
  if (tid == 0) w.flag[b] = total <= sc::kCap ? 1 : 2;
}

// ---------------------------------------------------------------- fp64 LSE
// One 512-key chunk of the concatenation (context, decode block) for
// (b, h): fp64 logits of kRows predicted rows at a time in shared memory,
// then the chunk's (max, sum) of each row.
template <typename T, int D>
__device__ __forceinline__ void sink_lse64_chunk(const Shape& s, const T* __restrict__ Q,
                                                 const int32_t* __restrict__ q_idx,
                                                 const int32_t* __restrict__ q_cnt,
                                                 const T* __restrict__ Kp,
                                                 const int32_t* __restrict__ page_table,
                                                 const T* __restrict__ Kd, const SinkCertWs& w,
                                                 unsigned* err, int b, int h, int g, int bh,
                                                 int chunk, int nch) {
  extern __shared__ __align__(16) uint8_t smem_b[];
  double* sQ = reinterpret_cast<double*>(smem_b);  // [kRows][D]
  double* sL = sQ + sc::kRows * D;                  // [kRows][kChunk]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  const long long t0 = (long long)chunk * sc::kChunk;
  const long long L_tot = (long long)s.L_ctx + s.L_q;
  for (int r0 = 0; r0 < nq; r0 += sc::kRows) {
    const int nr = min(sc::kRows, nq - r0);
    __syncthreads();
    for (int e = tid; e < nr * D; e += blockDim.x) {
      const int rr = e / D, c = e % D;
      const int i = q_idx[(size_t)b * s.L_q + r0 + rr];
      sQ[rr * D + c] = (i >= 0 && i < s.L_q)
                           ? (double)to_float(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + c])
                           : 0.0;
    }
    __syncthreads();
    for (int kl = tid; kl < sc::kChunk; kl += blockDim.x) {
      const long long t = t0 + kl;
      const T* src = nullptr;
      if (t < s.L_ctx) {
        const int slot = page_table[(size_t)b * s.n_pages + t / s.page];
        if (slot >= 0 && slot < s.n_slots)
          src = Kp + (((size_t)slot * s.H_kv + g) * s.page + t % s.page) * D;
        else
          flag_error(err, ERR_BAD_INDEX);
      } else if (t < L_tot) {
        src = Kd + (((size_t)b * s.H_kv + g) * s.L_q + (t - s.L_ctx)) * D;
      }
      if (src == nullptr) {
        for (int rr = 0; rr < nr; ++rr) sL[rr * sc::kChunk + kl] = -INFINITY;
        continue;
      }
      float k[D];
      constexpr int EPT = Vec16<T>::N;
#pragma unroll
      for (int c = 0; c < D; c += EPT) Vec16<T>::load(src + c, k + c);
      for (int rr = 0; rr < nr; ++rr) {
        const double* q = sQ + rr * D;
        double acc = 0.0;
#pragma unroll
        for (int c = 0; c < D; ++c) acc = fma(q[c], (double)k[c], acc);
        sL[rr * sc::kChunk + kl] = acc * s.scale;
      }
    }
    __syncthreads();
    for (int rr = warp; rr < nr; rr += sc::kThreads / 32) {  // warp per row
      const double* l = sL + rr * sc::kChunk;
      double mx = -INFINITY;
      for (int e = lane; e < sc::kChunk; e += 32) mx = fmax(mx, l[e]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      double sum = 0.0;
      if (mx != -INFINITY)
        for (int e = lane; e < sc::kChunk; e += 32) sum += exp(l[e] - mx);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      if (lane == 0)
        w.part[((size_t)bh * nch + chunk) * s.L_q + r0 + rr] = make_double2(mx, sum);
    }
  }
}

// CTA (x, b*H + h): chunks x, x + gridDim.x, ... of (b, h); returns at once
// for a certified sequence.
template <typename T, int D>
__global__ void __launch_bounds__(sc::kThreads)
sink_lse64_kernel(Shape s, const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                  const int32_t* __restrict__ q_cnt, const T* __restrict__ Kp,
                  const int32_t* __restrict__ page_table, const T* __restrict__ Kd,
                  SinkCertWs w, int nch, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.y, b = bh / s.H, h = bh % s.H, g = h / s.G;
  if (w.flag[b] == 0) return;
  for (int chunk = blockIdx.x; chunk < nch; chunk += gridDim.x) {
    __syncthreads();
    sink_lse64_chunk<T, D>(s, Q, q_idx, q_cnt, Kp, page_table, Kd, w, err, b, h, g, bh, chunk,
                           nch);
  }
}

// LSE of every (b, h, predicted row) from the chunks' (max, sum), in chunk order.
__global__ void __launch_bounds__(256)
sink_lse64_merge_kernel(Shape s, const int32_t* __restrict__ q_cnt, int nch, SinkCertWs w) {
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.x, b = bh / s.H;
  if (w.flag[b] == 0) return;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  for (int r = threadIdx.x; r < nq; r += blockDim.x) {
    double M = -INFINITY;
    for (int c = 0; c < nch; ++c) M = fmax(M, w.part[((size_t)bh * nch + c) * s.L_q + r].x);
    double S = 0.0;
    for (int c = 0; c < nch; ++c) {
      const double2 p = w.part[((size_t)bh * nch + c) * s.L_q + r];
      if (p.x != -INFINITY) S += p.y * exp(p.x - M);
    }
    w.lse[(size_t)bh * s.L_q + r] = M + log(S);
  }
}

// ---------------------------------------------------------------- fp64 mass
// Candidate c of sequence b: its fp64 mass, summed in (h, r) order (per
// thread, then over the threads in a fixed tree).
template <typename T, int D>
__device__ __forceinline__ void sink_cand_mass_one(const Shape& s, const T* __restrict__ Q,
                                                   const int32_t* __restrict__ q_idx,
                                                   const int32_t* __restrict__ q_cnt,
                                                   const T* __restrict__ Kp,
                                                   const int32_t* __restrict__ page_table,
                                                   const SinkCertWs& w, unsigned* err, int b,
                                                   int c, int flag, double* s_red) {
  const int t = flag == 1 ? w.cand[(size_t)b * sc::kCap + c] : c;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  const int slot = page_table[(size_t)b * s.n_pages + t / s.page];
  double sum = 0.0;
  if (slot >= 0 && slot < s.n_slots) {
    for (int p = threadIdx.x; p < s.H * nq; p += blockDim.x) {
      const int h = p / nq, r = p % nq, g = h / s.G;
      const int i = q_idx[(size_t)b * s.L_q + r];
      const T* k = Kp + (((size_t)slot * s.H_kv + g) * s.page + t % s.page) * D;
      double acc = 0.0;
      if (i >= 0 && i < s.L_q) {
        const T* q = Q + (((size_t)b * s.H + h) * s.L_q + i) * D;
        constexpr int EPT = Vec16<T>::N;
        for (int c0 = 0; c0 < D; c0 += EPT) {
          float qv[EPT], kv[EPT];
          Vec16<T>::load(q + c0, qv);
          Vec16<T>::load(k + c0, kv);
#pragma unroll
          for (int e = 0; e < EPT; ++e) acc = fma((double)qv[e], (double)kv[e], acc);
        }
      }
      sum += exp(acc * s.scale - w.lse[((size_t)b * s.H + h) * s.L_q + r]);
    }
  } else if (threadIdx.x == 0) {
    flag_error(err, ERR_BAD_INDEX);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = sum;
  __syncthreads();
  if (threadIdx.x == 0) {
    double tot = 0.0;
    for (int i = 0; i < sc::kThreads / 32; ++i) tot += s_red[i];
    w.m64[(size_t)b * cert_m64_len(s) + c] = tot;
  }
}

// CTA (x, b): candidates x, x + gridDim.x, ... (every column when there are
// more than kCap); returns at once for a certified sequence.
template <typename T, int D>
__global__ void __launch_bounds__(sc::kThreads)
sink_cand_mass_kernel(Shape s, const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                      const int32_t* __restrict__ q_cnt, const T* __restrict__ Kp,
                      const int32_t* __restrict__ page_table, SinkCertWs w, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ double s_red[sc::kThreads / 32];
  const int b = blockIdx.y;
  const int flag = w.flag[b];
  if (flag == 0) return;
  const int n_cols = flag == 1 ? w.count[b] : s.L_ctx;
  for (int c = blockIdx.x; c < n_cols; c += gridDim.x) {
    __syncthreads();
    sink_cand_mass_one<T, D>(s, Q, q_idx, q_cnt, Kp, page_table, w, err, b, c, flag, s_red);
  }
}

// ---------------------------------------------------------------- pick
// The n largest fp64 masses (ties to the lower position), ascending: round k
// takes the best entry strictly after round k-1's in (mass desc, position
// asc) order.
__global__ void __launch_bounds__(1024)
sink_pick_kernel(Shape s, int n_sinks, SinkCertWs w, int32_t* __restrict__ sink_pos) {
  pdl_trigger();
  pdl_wait();
  __shared__ double s_v[32];
  __shared__ int s_p[32];
  __shared__ int chosen[64];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int flag = w.flag[b];
  if (flag == 0) return;
  const int N = flag == 1 ? w.count[b] : s.L_ctx;
  const double* mv = w.m64 + (size_t)b * cert_m64_len(s);
  double pv = INFINITY;  // the previous winner
  int pp = -1;
  for (int k = 0; k < n_sinks; ++k) {
    double bv = -INFINITY;
    int bp = 0x7fffffff;
    for (int e = tid; e < N; e += blockDim.x) {
      const double v = mv[e];
      const int p = flag == 1 ? w.cand[(size_t)b * sc::kCap + e] : e;
      const bool after = v < pv || (v == pv && p > pp);
      if (after && (v > bv || (v == bv && p < bp))) {
        bv = v;
        bp = p;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int op = __shfl_xor_sync(0xffffffffu, bp, o);
      if (ov > bv || (ov == bv && op < bp)) {
        bv = ov;
        bp = op;
      }
    }
    if (lane == 0) {
      s_v[warp] = bv;
      s_p[warp] = bp;
    }
    __syncthreads();
    if (tid == 0) {
      double v = s_v[0];
      int p = s_p[0];
      for (int i = 1; i < (int)(blockDim.x >> 5); ++i)
        if (s_v[i] > v || (s_v[i] == v && s_p[i] < p)) {
          v = s_v[i];
          p = s_p[i];
        }
      s_v[0] = v;
      s_p[0] = p;
      chosen[k] = p < s.L_ctx ? p : -1;
    }
    __syncthreads();
    pv = s_v[0];
    pp = s_p[0];
    __syncthreads();
  }
  if (tid == 0) {
    for (int i = 1; i < n_sinks; ++i) {  // insertion sort, ascending
      const int x = chosen[i];
      int j = i - 1;
      while (j >= 0 && chosen[j] > x) { chosen[j + 1] = chosen[j]; --j; }
      chosen[j + 1] = x;
    }
    for (int i = 0; i < n_sinks; ++i) sink_pos[(size_t)b * n_sinks + i] = chosen[i];
  }
}

// ---------------------------------------------------------------- host
bool sink_cert_supported(const Shape& s, int n_sinks) {
  return n_sinks < s.L_ctx && s.H_kv <= sc::kMaxKvHeads && (s.d == 64 || s.d == 128);
}

template <typename T, int D>
static cudaError_t run_cert(const Shape& s, const void* Q, const int32_t* q_idx,
                            const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                            const void* Kd, const int32_t* Kexp, int n_units, const float* mass,
                            int n_sinks, int32_t* sink_pos, void* ws, unsigned* err,
                            cudaStream_t st) {
  const SinkCertWs w = sink_cert_ws(ws, s);
  const T* q = reinterpret_cast<const T*>(Q);
  const T* kp = reinterpret_cast<const T*>(Kp);
  const T* kd = reinterpret_cast<const T*>(Kd);
  DL_LAUNCH(sink_bound_kernel<T, D>, s.batch * s.H_kv, 256, 0, st, s, q, q_idx, q_cnt, kd, Kexp,
            n_units, w);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DL_LAUNCH(sink_band_count_kernel, dim3(32, s.batch), 256, 0, st, s, q_cnt, mass, n_sinks,
            (const int32_t*)sink_pos, w, D);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DL_LAUNCH(sink_band_final_kernel, s.batch, sc::kBandThreads, 0, st, s, q_cnt, mass, n_sinks, w,
            sink_pos);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  const int nch = cert_chunks(s);
  const int smem = (sc::kRows * D + sc::kRows * sc::kChunk) * (int)sizeof(double);
  if ((e = cudaFuncSetAttribute(sink_lse64_kernel<T, D>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
    return e;
  DL_LAUNCH(sink_lse64_kernel<T, D>, dim3(nch < 8 ? nch : 8, s.batch * s.H), sc::kThreads, smem,
            st, s, q, q_idx, q_cnt, kp, page_table, kd, w, nch, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DL_LAUNCH(sink_lse64_merge_kernel, s.batch * s.H, 256, 0, st, s, q_cnt, nch, w);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DL_LAUNCH(sink_cand_mass_kernel<T, D>, dim3(sc::kCap, s.batch), sc::kThreads, 0, st, s, q,
            q_idx, q_cnt, kp, page_table, w, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DL_LAUNCH(sink_pick_kernel, s.batch, 1024, 0, st, s, n_sinks, w, sink_pos);
  return cudaGetLastError();
}

cudaError_t launch_sink_cert(const Shape& s, const void* Q, const int32_t* q_idx,
                             const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                             const void* Kd, const int32_t* Kexp, int n_units, const float* mass,
                             int n_sinks, int32_t* sink_pos, void* ws, unsigned* err,
                             cudaStream_t st) {
  if (s.dtype == 0)
    return s.d == 128 ? run_cert<__nv_bfloat16, 128>(s, Q, q_idx, q_cnt, Kp, page_table, Kd,
                                                     Kexp, n_units, mass, n_sinks, sink_pos, ws,
                                                     err, st)
                      : run_cert<__nv_bfloat16, 64>(s, Q, q_idx, q_cnt, Kp, page_table, Kd,
                                                    Kexp, n_units, mass, n_sinks, sink_pos, ws,
                                                    err, st);
  return s.d == 128 ? run_cert<float, 128>(s, Q, q_idx, q_cnt, Kp, page_table, Kd, Kexp, n_units,
                                           mass, n_sinks, sink_pos, ws, err, st)
                    : run_cert<float, 64>(s, Q, q_idx, q_cnt, Kp, page_table, Kd, Kexp, n_units,
                                          mass, n_sinks, sink_pos, ws, err, st);
}

}  // namespace dl
