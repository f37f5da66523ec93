// (a4) Attention-sink detection by attention mass.
//
// Focus-dLLM abstract: sink-aware pruning keeps highly influential attention
// sinks and reuses the identified sink locations across layers.  Sinks are
// the context columns of largest attention mass of the predicted queries,
// summed over every head; they are found once, at the first sparse layer.
//
// The softmax of each row runs over the whole context plus the decode block,
// so its normaliser must be known before any column mass can be formed.
// bf16 inputs take the tensor-core passes (sinks_tc.cu); the CUDA-core
// passes below serve fp32 inputs and query groups of more than 256 rows:
//   pass 1  grid (token tiles, b*H): per tile and predicted row, the max and
//           the sum of exponentials of the tile's logits (one thread per
//           token, key row in registers, query rows broadcast from shared
//           memory, warp-shuffle reductions);
//   pass 2  one thread per (b, h, row): merge the tiles into the row's LSE;
//   pass 3  grid (token tiles, b): one thread per context token sums
//           exp(logit - LSE) over every head and row, in a fixed order;
//   pass 4  one CTA per sequence: n_sinks rounds of block argmax (mass desc,
//           position asc), written ascending.
#include "common.cuh"
#include "internal.h"
#include "launch.cuh"

namespace dl {

constexpr int kSinkRows = 32;  // predicted rows staged per pass

struct SinkWs {
  float2* part;  // [b*H][n_tiles][L_q] (max, sum)
  float* lse;    // [b*H][L_q]
  float* mass;   // [b][L_ctx]
};

__host__ __device__ inline int sink_tiles(const Shape& s) {
  return (s.L_ctx + kSinkTile - 1) / kSinkTile + (s.L_q + kSinkTile - 1) / kSinkTile;
}

__host__ __device__ inline SinkWs sink_ws(void* ws, const Shape& s) {
  char* p = reinterpret_cast<char*>(ws);
  SinkWs w;
  w.part = reinterpret_cast<float2*>(p);
  p += round256((size_t)s.batch * s.H * sink_tiles(s) * s.L_q * sizeof(float2));
  w.lse = reinterpret_cast<float*>(p);
  p += round256((size_t)s.batch * s.H * s.L_q * sizeof(float));
  w.mass = reinterpret_cast<float*>(p);
  return w;
}

// Tensor-core path: [attention partials][O scratch][LSE of every row][mass]
struct SinkTcWs {
  void* attn;
  void* O;
  float* lse;
  float* mass;
};

static SinkTcWs sink_tc_ws(void* ws, const Shape& s) {
  char* p = reinterpret_cast<char*>(ws);
  SinkTcWs w;
  w.attn = p;
  p += attn_workspace(s);
  w.O = p;
  p += round256((size_t)s.batch * s.L_q * s.H * s.d * 2);
  w.lse = reinterpret_cast<float*>(p);
  p += round256((size_t)s.batch * s.H * s.L_q * sizeof(float));
  w.mass = reinterpret_cast<float*>(p);
  return w;
}

// [mass-pass workspace (CUDA-core or tensor-core layout)][certified cut]
static size_t sinks_mass_workspace(const Shape& s) {
  const size_t simt = round256((size_t)s.batch * s.H * sink_tiles(s) * s.L_q * sizeof(float2)) +
                      round256((size_t)s.batch * s.H * s.L_q * sizeof(float)) +
                      round256((size_t)s.batch * s.L_ctx * sizeof(float));
  const size_t tc = attn_workspace(s) + round256((size_t)s.batch * s.L_q * s.H * s.d * 2) +
                    round256((size_t)s.batch * s.H * s.L_q * sizeof(float)) +
                    round256((size_t)s.batch * s.L_ctx * sizeof(float));
  return simt > tc ? simt : tc;
}

size_t sinks_workspace(const Shape& s) { return sinks_mass_workspace(s) + sink_cert_workspace(s); }

// Loads key row `t` of KV head g (context t < L_ctx, else decode key t-L_ctx)
// into k[]; returns false when the row holds no key.
template <typename T, int D>
__device__ __forceinline__ bool load_key(const Shape& s, const T* Kp, const T* Kd,
                                         const int32_t* page_table, int b, int g, long long t,
                                         float* k, unsigned* err) {
  const T* src = nullptr;
  if (t < s.L_ctx) {
    const int slot = page_table[(size_t)b * s.n_pages + t / s.page];
    if (slot < 0 || slot >= s.n_slots) {
      flag_error(err, ERR_BAD_INDEX);
      return false;
    }
    src = Kp + (((size_t)slot * s.H_kv + g) * s.page + t % s.page) * D;
  } else if (t < (long long)s.L_ctx + s.L_q) {
    src = Kd + (((size_t)b * s.H_kv + g) * s.L_q + (t - s.L_ctx)) * D;
  } else {
    return false;
  }
  constexpr int EPT = Vec16<T>::N;
#pragma unroll
  for (int c = 0; c < D; c += EPT) Vec16<T>::load(src + c, k + c);
  return true;
}

template <typename T>
__device__ __forceinline__ void stage_rows(const Shape& s, const T* Q, const int32_t* q_idx,
                                           int b, int h, int r0, int nq, int D, float* sQ) {
  for (int e = threadIdx.x; e < kSinkRows * D; e += blockDim.x) {
    const int rr = e / D, c = e % D, r = r0 + rr;
    float v = 0.0f;
    if (r < nq) {
      const int i = q_idx[(size_t)b * s.L_q + r];
      if (i >= 0 && i < s.L_q) v = to_f32(Q[(((size_t)b * s.H + h) * s.L_q + i) * D + c]);
    }
    sQ[rr * D + c] = v;
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(kSinkTile)
sink_partial_kernel(Shape s, const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                    const int32_t* __restrict__ q_cnt, const T* __restrict__ Kp,
                    const int32_t* __restrict__ page_table, const T* __restrict__ Kd,
                    SinkWs w, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sQ[kSinkRows * D];
  __shared__ float2 sRed[kSinkTile / 32][kSinkRows];
  const int tile = blockIdx.x, bh = blockIdx.y;
  const int b = bh / s.H, h = bh % s.H, g = h / s.G;
  const int n_ctx_tiles = (s.L_ctx + kSinkTile - 1) / kSinkTile;
  const long long t = tile < n_ctx_tiles
                          ? (long long)tile * kSinkTile + threadIdx.x
                          : (long long)s.L_ctx + (long long)(tile - n_ctx_tiles) * kSinkTile +
                                threadIdx.x;
  const bool in_range = tile < n_ctx_tiles ? t < s.L_ctx : t < (long long)s.L_ctx + s.L_q;
  float k[D];
  const bool ok = in_range && load_key<T, D>(s, Kp, Kd, page_table, b, g, t, k, err);
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const float scale = (float)s.scale;
  for (int r0 = 0; r0 < nq; r0 += kSinkRows) {
    __syncthreads();
    stage_rows<T>(s, Q, q_idx, b, h, r0, nq, D, sQ);
    __syncthreads();
    for (int rr = 0; rr < kSinkRows && r0 + rr < nq; ++rr) {
      float x = -INFINITY;
      if (ok) {
        float acc = 0.0f;
#pragma unroll 16
        for (int c = 0; c < D; ++c) acc = fmaf(sQ[rr * D + c], k[c], acc);
        x = acc * scale;
      }
      const float mx = warp_max(x);
      const float sm = warp_sum(mx == -INFINITY ? 0.0f : __expf(x - mx));
      if (lane == 0) sRed[warp][rr] = make_float2(mx, sm);
    }
    __syncthreads();
    if (threadIdx.x < kSinkRows && r0 + threadIdx.x < nq) {
      const int rr = threadIdx.x;
      float M = -INFINITY;
      for (int v = 0; v < kSinkTile / 32; ++v) M = fmaxf(M, sRed[v][rr].x);
      float L = 0.0f;
      if (M != -INFINITY)
        for (int v = 0; v < kSinkTile / 32; ++v)
          if (sRed[v][rr].x != -INFINITY) L += sRed[v][rr].y * __expf(sRed[v][rr].x - M);
      w.part[((size_t)bh * sink_tiles(s) + tile) * s.L_q + r0 + rr] = make_float2(M, L);
    }
  }
}

__global__ void sink_lse_kernel(Shape s, const int32_t* __restrict__ q_cnt, SinkWs w) {
  pdl_trigger();
  pdl_wait();
  const int bh = blockIdx.x, r = threadIdx.x;
  const int b = bh / s.H;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  if (r >= nq) return;
  const int nt = sink_tiles(s);
  float M = -INFINITY;
  for (int t = 0; t < nt; ++t) M = fmaxf(M, w.part[((size_t)bh * nt + t) * s.L_q + r].x);
  float L = 0.0f;
  for (int t = 0; t < nt; ++t) {
    const float2 p = w.part[((size_t)bh * nt + t) * s.L_q + r];
    if (p.x != -INFINITY) L += p.y * __expf(p.x - M);
  }
  w.lse[(size_t)bh * s.L_q + r] = M + __logf(L);
}

template <typename T, int D>
__global__ void __launch_bounds__(kSinkTile)
sink_mass_kernel(Shape s, const T* __restrict__ Q, const int32_t* __restrict__ q_idx,
                 const int32_t* __restrict__ q_cnt, const T* __restrict__ Kp,
                 const int32_t* __restrict__ page_table, SinkWs w, unsigned* err) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sQ[kSinkRows * D];
  __shared__ float sL[kSinkRows];
  const int b = blockIdx.y;
  const long long t = (long long)blockIdx.x * kSinkTile + threadIdx.x;
  const bool in_range = t < s.L_ctx;
  const int nq = min(max(q_cnt[b], 0), s.L_q);
  const float scale = (float)s.scale;
  float mass = 0.0f;
  float k[D];
  bool ok = false;
  for (int h = 0; h < s.H; ++h) {
    const int g = h / s.G;
    if (h % s.G == 0) ok = in_range && load_key<T, D>(s, Kp, nullptr, page_table, b, g, t, k, err);
    for (int r0 = 0; r0 < nq; r0 += kSinkRows) {
      __syncthreads();
      stage_rows<T>(s, Q, q_idx, b, h, r0, nq, D, sQ);
      if (threadIdx.x < kSinkRows)
        sL[threadIdx.x] = r0 + threadIdx.x < nq
                              ? w.lse[((size_t)b * s.H + h) * s.L_q + r0 + threadIdx.x]
                              : 0.0f;
      __syncthreads();
      if (!ok) continue;
      for (int rr = 0; rr < kSinkRows && r0 + rr < nq; ++rr) {
        float acc = 0.0f;
#pragma unroll 16
        for (int c = 0; c < D; ++c) acc = fmaf(sQ[rr * D + c], k[c], acc);
        mass += __expf(acc * scale - sL[rr]);
      }
    }
  }
  if (in_range) w.mass[(size_t)b * s.L_ctx + t] = mass;
}

// Top-n columns by mass (ties to the lower position), ascending.  Any n:
// n rounds of a block argmax over a scan of the masses, round k over the
// columns strictly after round k-1's winner in (mass desc, position asc)
// order (the masses are left as they are).
__global__ void __launch_bounds__(1024)
sink_topn_scan_kernel(Shape s, int n_sinks, SinkWs w, int32_t* __restrict__ sink_pos) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int chosen[64];
  const int b = blockIdx.x;
  const float* mass = w.mass + (size_t)b * s.L_ctx;
  float pv = INFINITY;  // the previous winner
  int pi = -1;
  for (int round = 0; round < n_sinks; ++round) {
    float v = -INFINITY;
    int idx = 0x7fffffff;
    for (int t = threadIdx.x; t < s.L_ctx; t += blockDim.x) {
      const float m = mass[t];
      const bool after = m < pv || (m == pv && t > pi);
      if (after && (m > v || (m == v && t < idx))) { v = m; idx = t; }
    }
    float bv;
    int bi;
    block_argmax(v, idx, sv, si, bv, bi);
    if (threadIdx.x == 0) chosen[round] = bi < s.L_ctx ? bi : -1;
    pv = bv;
    pi = bi;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    for (int i = 1; i < n_sinks; ++i) {  // insertion sort, ascending
      const int x = chosen[i];
      int j = i - 1;
      while (j >= 0 && chosen[j] > x) { chosen[j + 1] = chosen[j]; --j; }
      chosen[j + 1] = x;
    }
    for (int i = 0; i < n_sinks; ++i) sink_pos[(size_t)b * n_sinks + i] = chosen[i];
  }
}

// n <= KL: one pass in which every thread keeps the KL largest masses of its
// own positions (descending; a thread meets its positions in increasing order,
// so equal masses keep the lower position first), then n rounds of a block
// argmax over the threads' leading entries, the winner dropping its lead.
// Every global top-n column is among its thread's top n, so the result is
// that of the scan.
template <int KL>
__global__ void __launch_bounds__(512)
sink_topn_kernel(Shape s, int n_sinks, const float* __restrict__ mass_all,
                 int32_t* __restrict__ sink_pos) {
  pdl_trigger();
  pdl_wait();
  __shared__ float sv[32];
  __shared__ int si[32];
  __shared__ int chosen[KL];
  constexpr int U = 8;  // loads in flight per thread
  const int b = blockIdx.x;
  const float* mass = mass_all + (size_t)b * s.L_ctx;
  float lv[KL];
  int li[KL];
#pragma unroll
  for (int k = 0; k < KL; ++k) {
    lv[k] = -INFINITY;
    li[k] = 0x7fffffff;
  }
  auto push = [&](float m, int t) {
    if (!(m > lv[KL - 1])) return;
    lv[KL - 1] = m;
    li[KL - 1] = t;
#pragma unroll
    for (int k = KL - 1; k > 0; --k) {
      if (lv[k] > lv[k - 1]) {
        const float tv = lv[k]; lv[k] = lv[k - 1]; lv[k - 1] = tv;
        const int ti = li[k]; li[k] = li[k - 1]; li[k - 1] = ti;
      }
    }
  };
  const int L = s.L_ctx;
  if ((L & 3) == 0 && (reinterpret_cast<uintptr_t>(mass) & 15) == 0) {
    const float4* m4 = reinterpret_cast<const float4*>(mass);
    const int n4 = L >> 2;
    for (int base = threadIdx.x; base < n4; base += U * blockDim.x) {
      float4 v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * blockDim.x;
        v[u] = i < n4 ? __ldg(m4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * blockDim.x;
        if (i < n4) {
          push(v[u].x, 4 * i);
          push(v[u].y, 4 * i + 1);
          push(v[u].z, 4 * i + 2);
          push(v[u].w, 4 * i + 3);
        }
      }
    }
  } else {
    for (int base = threadIdx.x; base < L; base += U * blockDim.x) {
      float v[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = base + u * blockDim.x;
        v[u] = i < L ? __ldg(mass + i) : 0.0f;
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (base + u * (int)blockDim.x < L) push(v[u], base + u * blockDim.x);
    }
  }
  for (int r = 0; r < n_sinks; ++r) {
    float bv;
    int bi;
    block_argmax(lv[0], li[0], sv, si, bv, bi);
    const bool found = bv != -INFINITY && bi < L;
    if (found && li[0] == bi) {  // positions are unique: this thread led
#pragma unroll
      for (int k = 0; k < KL - 1; ++k) {
        lv[k] = lv[k + 1];
        li[k] = li[k + 1];
      }
      lv[KL - 1] = -INFINITY;
      li[KL - 1] = 0x7fffffff;
    }
    if (threadIdx.x == 0) chosen[r] = found ? bi : -1;
  }
  if (threadIdx.x == 0) {
    for (int i = 1; i < n_sinks; ++i) {  // insertion sort, ascending
      const int x = chosen[i];
      int j = i - 1;
      while (j >= 0 && chosen[j] > x) { chosen[j + 1] = chosen[j]; --j; }
      chosen[j + 1] = x;
    }
    for (int i = 0; i < n_sinks; ++i) sink_pos[(size_t)b * n_sinks + i] = chosen[i];
  }
}

static cudaError_t launch_sink_topn(const Shape& s, int n_sinks, const SinkWs& w,
                                    int32_t* sink_pos, cudaStream_t st) {
  if (n_sinks <= 8) {
    DL_LAUNCH(sink_topn_kernel<8>, s.batch, 512, 0, st, s, n_sinks, (const float*)w.mass,
              sink_pos);
  } else {
    DL_LAUNCH(sink_topn_scan_kernel, s.batch, 1024, 0, st, s, n_sinks, w, sink_pos);
  }
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t run_sink_mass(const Shape& s, const void* Q, const int32_t* q_idx,
                                 const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                                 const void* Kd, float* mass, void* ws, unsigned* err,
                                 cudaStream_t st) {
  SinkWs w = sink_ws(ws, s);
  w.mass = mass;
  const T* q = reinterpret_cast<const T*>(Q);
  const T* kp = reinterpret_cast<const T*>(Kp);
  const T* kd = reinterpret_cast<const T*>(Kd);
  DL_LAUNCH(sink_partial_kernel<T, D>, dim3(sink_tiles(s), s.batch * s.H), kSinkTile, 0, st, 
      s, q, q_idx, q_cnt, kp, page_table, kd, w, err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  DL_LAUNCH(sink_lse_kernel, s.batch * s.H, ((s.L_q + 31) / 32) * 32, 0, st, s, q_cnt, w);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  DL_LAUNCH(sink_mass_kernel<T, D>, dim3((s.L_ctx + kSinkTile - 1) / kSinkTile, s.batch), kSinkTile, 0,
                           st, s, q, q_idx, q_cnt, kp, page_table, w, err);
  return cudaGetLastError();
}

bool attn_tc_supported(const AttnArgs& a);
bool attn_tc_kt_supported(const AttnArgs& a);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);
cudaError_t launch_sink_mass_tc(const Shape& s, const void* Q, const int32_t* q_idx,
                                const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                                const float* lse, float* mass, unsigned* err, cudaStream_t st);

// Column masses of the predicted rows of this descriptor's heads into
// mass[b][L_ctx] (NULL: the workspace's mass array).  bf16 with at most 256
// query rows per KV group: tensor cores (pass 1 = dense attention for the
// row LSEs -- LSE-only on the key-major kernel, otherwise with V = K and the
// output discarded --, pass 2 = sinks_tc.cu); otherwise the CUDA-core passes
// above.
cudaError_t launch_sink_mass(const Shape& s, const void* Q, const int32_t* q_idx,
                             const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                             const void* Kd, float* mass, void* ws, unsigned* err,
                             cudaStream_t st) {
  SinkTcWs tw = sink_tc_ws(ws, s);
  AttnArgs a{};
  a.s = s; a.Q = Q; a.Kp = Kp; a.Vp = Kp; a.page_table = page_table; a.mode = kDense;
  a.idx = nullptr; a.cnt = nullptr; a.max_idx = 0; a.Kd = Kd; a.Vd = Kd; a.O = tw.O;
  a.lse = tw.lse; a.ws = tw.attn; a.ws_bytes = attn_workspace(s); a.err = err;
  if (s.dtype == 0 && s.G * s.L_q <= 256 && attn_tc_supported(a)) {
    // the key-major kernel can skip V and O: only the row LSEs are needed
    if (attn_tc_kt_supported(a)) a.O = nullptr;
    cudaError_t e = launch_attn(a, st);
    if (e != cudaSuccess) return e;
    return launch_sink_mass_tc(s, Q, q_idx, q_cnt, Kp, page_table, tw.lse,
                               mass ? mass : tw.mass, err, st);
  }
  float* m = mass ? mass : sink_ws(ws, s).mass;
  if (s.dtype == 0)
    return s.d == 128 ? run_sink_mass<__nv_bfloat16, 128>(s, Q, q_idx, q_cnt, Kp, page_table, Kd,
                                                          m, ws, err, st)
                      : run_sink_mass<__nv_bfloat16, 64>(s, Q, q_idx, q_cnt, Kp, page_table, Kd,
                                                         m, ws, err, st);
  return s.d == 128 ? run_sink_mass<float, 128>(s, Q, q_idx, q_cnt, Kp, page_table, Kd, m, ws,
                                                err, st)
                    : run_sink_mass<float, 64>(s, Q, q_idx, q_cnt, Kp, page_table, Kd, m, ws,
                                               err, st);
}

// The n_sinks columns of largest mass (ties to the lower position), ascending.
cudaError_t launch_sink_topn_mass(float* mass, int batch, int L_ctx, int n_sinks,
                                  int32_t* sink_pos, cudaStream_t st) {
  Shape s{};
  s.batch = batch;
  s.L_ctx = L_ctx;
  SinkWs w{};
  w.mass = mass;
  return launch_sink_topn(s, n_sinks, w, sink_pos, st);
}

// With Kexp (the norm bounds of this layer's pooled keys) the cut is
// certified (sinks_cert.cu); without it, the top-n of the fp32 masses.
cudaError_t launch_sinks(const Shape& s, const void* Q, const int32_t* q_idx,
                         const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                         const void* Kd, const int32_t* Kexp, int n_sinks, int32_t* sink_pos,
                         void* ws, unsigned* err, cudaStream_t st) {
  const bool tc = s.dtype == 0 && s.G * s.L_q <= 256;
  float* mass = tc ? sink_tc_ws(ws, s).mass : sink_ws(ws, s).mass;
  cudaError_t e = launch_sink_mass(s, Q, q_idx, q_cnt, Kp, page_table, Kd, mass, ws, err, st);
  if (e != cudaSuccess) return e;
  if ((e = launch_sink_topn_mass(mass, s.batch, s.L_ctx, n_sinks, sink_pos, st)) != cudaSuccess)
    return e;
  if (Kexp && sink_cert_supported(s, n_sinks))  // certify the top n (sinks_cert.cu)
    return launch_sink_cert(s, Q, q_idx, q_cnt, Kp, page_table, Kd, Kexp,
                            (s.L_ctx + s.page - 1) / s.page, mass, n_sinks, sink_pos,
                            reinterpret_cast<char*>(ws) + sinks_mass_workspace(s), err, st);
  return cudaSuccess;
}

}  // namespace dl
