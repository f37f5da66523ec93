// C ABI of the sparse denoising-step library: argument validation,
// workspace sizing, the device error word, and the kernel launches.
// Every entry point checks its arguments on the host before launching
// anything, launches asynchronously on the caller's stream, and never
// throws.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <atomic>
#include <mutex>

#include "../../include/dl.h"
#include "internal.h"

namespace {

thread_local char g_msg[512] = "";

dl_status fail(dl_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return st;
}

dl_status ok() {
  g_msg[0] = 0;
  return DL_OK;
}

dl_status cuda_fail(cudaError_t e, const char* what) {
  return fail(DL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Device error word: one per device (a __device__ variable exists in every
// device context that loads the library).  Its address is looked up once per
// device.
__device__ unsigned g_dev_error;

constexpr int kMaxDevices = 64;
unsigned* g_err_ptr[kMaxDevices] = {};
std::mutex g_err_mu;

dl_status error_word(unsigned** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(DL_ERR_UNSUPPORTED, "device id %d", dev);
  std::lock_guard<std::mutex> lk(g_err_mu);
  if (!g_err_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_dev_error);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    g_err_ptr[dev] = static_cast<unsigned*>(p);
  }
  *out = g_err_ptr[dev];
  return DL_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

dl_status check_desc(const dl_attn_desc* d, dl::Shape* s) {
  if (!d) return fail(DL_ERR_INVALID_ARG, "desc is NULL");
  if (d->batch < 1 || d->batch > 65535) return fail(DL_ERR_INVALID_ARG, "batch=%d", d->batch);
  if (d->H < 1 || d->H_kv < 1 || d->H % d->H_kv != 0)
    return fail(DL_ERR_INVALID_ARG, "H=%d H_kv=%d (need H %% H_kv == 0)", d->H, d->H_kv);
  if ((long long)d->batch * d->H > 65535)
    return fail(DL_ERR_INVALID_ARG, "batch*H=%lld exceeds 65535", (long long)d->batch * d->H);
  if (d->d != 64 && d->d != 128) return fail(DL_ERR_UNSUPPORTED, "head_dim %d (need 64 or 128)", d->d);
  if (d->page != 64) return fail(DL_ERR_UNSUPPORTED, "page size %d (need 64)", d->page);
  if (d->L_q < 1 || d->L_q > 256) return fail(DL_ERR_INVALID_ARG, "L_q=%d (need 1..256)", d->L_q);
  if (d->L_ctx < 0) return fail(DL_ERR_INVALID_ARG, "L_ctx=%d", d->L_ctx);
  if (d->n_pages < 0 || (long long)d->n_pages * d->page < d->L_ctx)
    return fail(DL_ERR_INVALID_ARG, "n_pages*page=%lld < L_ctx=%d",
                (long long)d->n_pages * d->page, d->L_ctx);
  if (d->n_slots < 1) return fail(DL_ERR_INVALID_ARG, "n_slots=%d", d->n_slots);
  if ((long long)d->n_slots * d->H_kv * d->page > (1ll << 40))
    return fail(DL_ERR_INVALID_ARG, "pool too large");
  if (d->dtype != DL_BF16 && d->dtype != DL_FP32)
    return fail(DL_ERR_UNSUPPORTED, "dtype %d", d->dtype);
  s->batch = d->batch; s->H = d->H; s->H_kv = d->H_kv; s->G = d->H / d->H_kv; s->d = d->d;
  s->L_ctx = d->L_ctx; s->L_q = d->L_q; s->page = d->page; s->n_pages = d->n_pages;
  s->n_slots = d->n_slots; s->dtype = d->dtype;
  s->scale = 1.0 / std::sqrt((double)d->d);
  return DL_OK;
}

dl_status need_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (need == 0) return DL_OK;
  if (!ws) return fail(DL_ERR_WORKSPACE, "workspace is NULL (need %zu bytes)", need);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(DL_ERR_WORKSPACE, "workspace not 256-byte aligned");
  if (ws_bytes < need) return fail(DL_ERR_WORKSPACE, "workspace %zu < %zu bytes", ws_bytes, need);
  return DL_OK;
}

inline cudaStream_t as_stream(void* st) { return reinterpret_cast<cudaStream_t>(st); }

dl_status launched(cudaError_t e, const char* what) {
  if (e != cudaSuccess) return cuda_fail(e, what);
  return ok();
}

int n_blk_of(const dl::Shape& s) { return (s.L_ctx + s.page - 1) / s.page; }

std::atomic<unsigned> g_kernel_flags{0u};

}  // namespace

// Validation and error-word access for entry points defined in other files.
namespace dl {
dl_status api_check_desc(const dl_attn_desc* d, Shape* s) { return check_desc(d, s); }
dl_status api_error_word(unsigned** out) { return error_word(out); }
dl_status api_fail(dl_status st, const char* msg) { return fail(st, "%s", msg); }
dl_status api_ok() { return ok(); }
unsigned kernel_flags() { return g_kernel_flags.load(std::memory_order_relaxed); }
}  // namespace dl

extern "C" {

int dl_version(void) { return 200; }

unsigned dl_set_kernel_flags(unsigned flags) { return g_kernel_flags.exchange(flags); }

dl_status dl_read_counters(unsigned long long* fast, unsigned long long* fallback) {
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  if ((e = dl::read_select_counts(fast, fallback)) != cudaSuccess)
    return cuda_fail(e, "dl_read_counters");
  return ok();
}

const char* dl_last_error_message(void) { return g_msg; }

dl_status dl_get_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  unsigned* w = nullptr;
  dl_status st = error_word(&w);
  if (st != DL_OK) return st;
  unsigned v = 0;
  e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  const unsigned zero = 0;
  e = cudaMemcpy(w, &zero, sizeof(zero), cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "clear error word");
  if (v & dl::ERR_TIMEOUT) return fail(DL_ERR_TIMEOUT, "a bounded device wait gave up");
  if (v & dl::ERR_BAD_INDEX)
    return fail(DL_ERR_BAD_INDEX, "a kernel met an out-of-range index (tile skipped)");
  return ok();
}

dl_status dl_workspace_size(const dl_attn_desc* desc, size_t* bytes) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!bytes) return fail(DL_ERR_INVALID_ARG, "bytes is NULL");
  const int units = n_blk_of(s) > s.n_pages ? n_blk_of(s) : s.n_pages;
  size_t need = dl::attn_workspace(s);
  size_t x = dl::scores_workspace(s, units);
  need = x > need ? x : need;
  x = dl::sinks_workspace(s);
  need = x > need ? x : need;
  *bytes = need;
  return ok();
}

dl_status dl_predict_queries(const float* conf_prev, const uint8_t* still_masked, int batch,
                             int L_q, int k, int w, int32_t* q_idx, int32_t* q_cnt,
                             void* stream) {
  if (!conf_prev || !still_masked || !q_idx || !q_cnt)
    return fail(DL_ERR_INVALID_ARG, "dl_predict_queries: NULL pointer");
  if (batch < 1 || batch > 65535) return fail(DL_ERR_INVALID_ARG, "batch=%d", batch);
  if (L_q < 1 || L_q > 1024) return fail(DL_ERR_INVALID_ARG, "L_q=%d (need 1..1024)", L_q);
  if (k < 0 || w < 0) return fail(DL_ERR_INVALID_ARG, "k=%d w=%d", k, w);
  return launched(dl::launch_predict(conf_prev, still_masked, batch, L_q, k, w, q_idx, q_cnt,
                                     as_stream(stream)),
                  "dl_predict_queries launch");
}

dl_status dl_pool_keys(const dl_attn_desc* desc, const void* K_pool, const int32_t* page_table,
                       int n_units, int unit_stride, int unit_offset, int unit_len, float* Kbar,
                       int8_t* Kdig, int32_t* Kexp, void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!K_pool || !page_table || !Kbar) return fail(DL_ERR_INVALID_ARG, "dl_pool_keys: NULL pointer");
  if ((Kdig == nullptr) != (Kexp == nullptr))
    return fail(DL_ERR_INVALID_ARG, "dl_pool_keys: Kdig and Kexp go together");
  if (Kdig && !aligned16(Kdig)) return fail(DL_ERR_INVALID_ARG, "Kdig not 16-byte aligned");
  if (!aligned16(K_pool)) return fail(DL_ERR_INVALID_ARG, "K_pool not 16-byte aligned");
  if (n_units < 1 || n_units > (1 << 24)) return fail(DL_ERR_INVALID_ARG, "n_units=%d", n_units);
  if (unit_stride < 1 || unit_offset < 0 || unit_len < 1)
    return fail(DL_ERR_INVALID_ARG, "unit stride=%d offset=%d len=%d", unit_stride, unit_offset,
                unit_len);
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_pool(s, K_pool, page_table, n_units, unit_stride, unit_offset,
                                  unit_len, Kbar, Kdig, Kexp, err, as_stream(stream)),
                  "dl_pool_keys launch");
}

dl_status dl_cache_write(const dl_attn_desc* desc, const void* K_new, const void* V_new,
                         int n_new, const int32_t* start, const int32_t* page_table,
                         void* K_pool, void* V_pool, float* Kbar, int8_t* Kdig, int32_t* Kexp,
                         void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!K_new || !V_new || !start || !page_table || !K_pool || !V_pool || !Kbar)
    return fail(DL_ERR_INVALID_ARG, "dl_cache_write: NULL pointer");
  if ((Kdig == nullptr) != (Kexp == nullptr))
    return fail(DL_ERR_INVALID_ARG, "dl_cache_write: Kdig and Kexp go together");
  if (!aligned16(K_new) || !aligned16(V_new) || !aligned16(K_pool) || !aligned16(V_pool))
    return fail(DL_ERR_INVALID_ARG, "dl_cache_write: K/V buffers must be 16-byte aligned");
  if (n_new < 1 || n_new > s.L_ctx)
    return fail(DL_ERR_INVALID_ARG, "n_new=%d (need 1..L_ctx=%d)", n_new, s.L_ctx);
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_cache_write(s, K_new, V_new, n_new, start, page_table, K_pool,
                                         V_pool, Kbar, Kdig, Kexp, err, as_stream(stream)),
                  "dl_cache_write launch");
}

dl_status dl_block_scores(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, int n_units, double* score,
                          void* ws, size_t ws_bytes, void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !Kbar || !score || (q_idx && !q_cnt))
    return fail(DL_ERR_INVALID_ARG, "dl_block_scores: NULL pointer");
  if (n_units < 1 || n_units > (1 << 20)) return fail(DL_ERR_INVALID_ARG, "n_units=%d", n_units);
  if ((st = need_ws(ws, ws_bytes, dl::scores_workspace(s, n_units))) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_scores(s, Q_dec, q_idx, q_cnt, Kbar, n_units, score, ws, err,
                                    as_stream(stream)),
                  "dl_block_scores launch");
}

dl_status dl_find_sinks(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                        const int32_t* q_cnt, const void* K_pool, const int32_t* page_table,
                        const void* K_dec, const int32_t* Kexp, int n_sinks, int32_t* sink_pos,
                        void* ws, size_t ws_bytes, void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !q_idx || !q_cnt || !K_pool || !page_table || !K_dec || !sink_pos)
    return fail(DL_ERR_INVALID_ARG, "dl_find_sinks: NULL pointer");
  if (!aligned16(K_pool) || !aligned16(K_dec))
    return fail(DL_ERR_INVALID_ARG, "K_pool/K_dec not 16-byte aligned");
  if (n_sinks < 1 || n_sinks > 64) return fail(DL_ERR_INVALID_ARG, "n_sinks=%d (need 1..64)", n_sinks);
  if (s.L_ctx < 1) return fail(DL_ERR_INVALID_ARG, "dl_find_sinks: empty context");
  if ((st = need_ws(ws, ws_bytes, dl::sinks_workspace(s))) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_sinks(s, Q_dec, q_idx, q_cnt, K_pool, page_table, K_dec, Kexp,
                                   n_sinks, sink_pos, ws, err, as_stream(stream)),
                  "dl_find_sinks launch");
}

dl_status dl_sink_mass(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                       const int32_t* q_cnt, const void* K_pool, const int32_t* page_table,
                       const void* K_dec, float* mass, void* ws, size_t ws_bytes, void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !q_idx || !q_cnt || !K_pool || !page_table || !K_dec || !mass)
    return fail(DL_ERR_INVALID_ARG, "dl_sink_mass: NULL pointer");
  if (!aligned16(K_pool) || !aligned16(K_dec))
    return fail(DL_ERR_INVALID_ARG, "K_pool/K_dec not 16-byte aligned");
  if (s.L_ctx < 1) return fail(DL_ERR_INVALID_ARG, "dl_sink_mass: empty context");
  if ((st = need_ws(ws, ws_bytes, dl::sinks_workspace(s))) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_sink_mass(s, Q_dec, q_idx, q_cnt, K_pool, page_table, K_dec, mass,
                                       ws, err, as_stream(stream)),
                  "dl_sink_mass launch");
}

dl_status dl_sink_topn(float* mass, int batch, int L_ctx, int n_sinks, int32_t* sink_pos,
                       void* stream) {
  if (!mass || !sink_pos) return fail(DL_ERR_INVALID_ARG, "dl_sink_topn: NULL pointer");
  if (batch < 1 || L_ctx < 1)
    return fail(DL_ERR_INVALID_ARG, "dl_sink_topn: batch=%d L_ctx=%d", batch, L_ctx);
  if (n_sinks < 1 || n_sinks > 64) return fail(DL_ERR_INVALID_ARG, "n_sinks=%d (need 1..64)", n_sinks);
  return launched(dl::launch_sink_topn_mass(mass, batch, L_ctx, n_sinks, sink_pos,
                                            as_stream(stream)),
                  "dl_sink_topn launch");
}

dl_status dl_select(const double* score, int batch, int H_kv, int n_units, int unit_size, int topK,
                    const int32_t* sink_pos, int n_sinks, int32_t* blk_idx, int32_t* blk_cnt,
                    int max_sel, void* stream) {
  if (!score || !blk_idx || !blk_cnt || (n_sinks > 0 && !sink_pos))
    return fail(DL_ERR_INVALID_ARG, "dl_select: NULL pointer");
  if (batch < 1 || H_kv < 1 || (long long)batch * H_kv > 65535)
    return fail(DL_ERR_INVALID_ARG, "batch=%d H_kv=%d", batch, H_kv);
  if (n_units < 1 || n_units > 16384)
    return fail(DL_ERR_INVALID_ARG, "n_units=%d (need 1..16384)", n_units);
  if (unit_size < 1 || topK < 0 || n_sinks < 0 || n_sinks > 1024)
    return fail(DL_ERR_INVALID_ARG, "unit_size=%d topK=%d n_sinks=%d", unit_size, topK, n_sinks);
  const int need = (topK < n_units ? topK : n_units) + n_sinks;
  if (max_sel < need)
    return fail(DL_ERR_INVALID_ARG, "max_sel=%d < min(topK, n_units) + n_sinks = %d", max_sel, need);
  unsigned* err = nullptr;
  dl_status st = error_word(&err);
  if (st != DL_OK) return st;
  return launched(dl::launch_select(score, batch, H_kv, n_units, unit_size, topK, sink_pos,
                                    n_sinks, blk_idx, blk_cnt, max_sel, err, as_stream(stream)),
                  "dl_select launch");
}

dl_status dl_block_select(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                          const int32_t* Kexp, int n_units, int unit_size,
                          int topK, const int32_t* sink_pos, int n_sinks, double* score,
                          int32_t* blk_idx, int32_t* blk_cnt, int max_sel, int max_q, void* ws,
                          size_t ws_bytes, void* stream) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !Kbar || !score || (q_idx && !q_cnt) || !blk_idx || !blk_cnt ||
      (n_sinks > 0 && !sink_pos))
    return fail(DL_ERR_INVALID_ARG, "dl_block_select: NULL pointer");
  if ((Kdig == nullptr) != (Kexp == nullptr))
    return fail(DL_ERR_INVALID_ARG, "dl_block_select: Kdig and Kexp go together");
  if (Kdig && !aligned16(Kdig)) return fail(DL_ERR_INVALID_ARG, "Kdig not 16-byte aligned");
  if (!aligned16(Q_dec) || !aligned16(Kbar))
    return fail(DL_ERR_INVALID_ARG, "dl_block_select: Q_dec and Kbar must be 16-byte aligned");
  if (n_units < 1 || n_units > 16384)
    return fail(DL_ERR_INVALID_ARG, "n_units=%d (need 1..16384)", n_units);
  if (unit_size < 1 || topK < 0 || n_sinks < 0 || n_sinks > 1024)
    return fail(DL_ERR_INVALID_ARG, "unit_size=%d topK=%d n_sinks=%d", unit_size, topK, n_sinks);
  const int need = (topK < n_units ? topK : n_units) + n_sinks;
  if (max_sel < need)
    return fail(DL_ERR_INVALID_ARG, "max_sel=%d < min(topK, n_units) + n_sinks = %d", max_sel, need);
  if (max_q < 0) return fail(DL_ERR_INVALID_ARG, "max_q=%d (need >= 0)", max_q);
  if ((st = need_ws(ws, ws_bytes, dl::scores_workspace(s, n_units))) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_block_select(s, Q_dec, q_idx, q_cnt, Kbar, Kdig, Kexp, n_units, score,
                                          unit_size, topK, sink_pos, n_sinks, blk_idx, blk_cnt,
                                          max_sel, max_q, ws, err, as_stream(stream)),
                  "dl_block_select launch");
}

static dl_status attn_common(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                             const void* V_pool, const int32_t* page_table, int mode,
                             const int32_t* idx, const int32_t* cnt, int max_idx,
                             const void* K_dec, const void* V_dec, void* O, float* lse, void* ws,
                             size_t ws_bytes, void* stream, const char* name) {
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !K_pool || !V_pool || !page_table || !K_dec || !V_dec || !O)
    return fail(DL_ERR_INVALID_ARG, "%s: NULL pointer", name);
  if (mode != dl::kDense && (!idx || !cnt))
    return fail(DL_ERR_INVALID_ARG, "%s: NULL index/count", name);
  if (!aligned16(Q_dec) || !aligned16(K_pool) || !aligned16(V_pool) || !aligned16(K_dec) ||
      !aligned16(V_dec) || !aligned16(O))
    return fail(DL_ERR_INVALID_ARG, "%s: Q/K/V/O pointers must be 16-byte aligned", name);
  if (mode != dl::kDense && (max_idx < 0 || max_idx > (1 << 24)))
    return fail(DL_ERR_INVALID_ARG, "%s: max index count %d", name, max_idx);
  if ((st = need_ws(ws, ws_bytes, dl::attn_workspace(s))) != DL_OK) return st;
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  dl::AttnArgs a{};
  a.s = s; a.Q = Q_dec; a.Kp = K_pool; a.Vp = V_pool; a.page_table = page_table;
  a.mode = mode; a.idx = idx; a.cnt = cnt; a.max_idx = mode == dl::kDense ? 0 : max_idx;
  a.Kd = K_dec; a.Vd = V_dec; a.O = O; a.lse = lse; a.ws = ws; a.ws_bytes = ws_bytes; a.err = err;
  return launched(dl::launch_attn(a, as_stream(stream)), name);
}

dl_status dl_sparse_attn(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                         const void* V_pool, const int32_t* page_table, const int32_t* blk_idx,
                         const int32_t* blk_cnt, int max_sel, const void* K_dec,
                         const void* V_dec, void* O, float* lse, void* ws, size_t ws_bytes,
                         void* stream) {
  const int mode = blk_idx ? dl::kBlocks : dl::kDense;
  return attn_common(desc, Q_dec, K_pool, V_pool, page_table, mode, blk_idx, blk_cnt, max_sel,
                     K_dec, V_dec, O, lse, ws, ws_bytes, stream, "dl_sparse_attn");
}

dl_status dl_sparse_attn_gather(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                                const void* V_pool, const int32_t* page_table,
                                const int32_t* tok_pos, const int32_t* tok_cnt, int max_tok,
                                const void* K_dec, const void* V_dec, void* O, float* lse,
                                void* ws, size_t ws_bytes, void* stream) {
  if (!tok_pos) return fail(DL_ERR_INVALID_ARG, "dl_sparse_attn_gather: tok_pos is NULL");
  return attn_common(desc, Q_dec, K_pool, V_pool, page_table, dl::kGather, tok_pos, tok_cnt,
                     max_tok, K_dec, V_dec, O, lse, ws, ws_bytes, stream,
                     "dl_sparse_attn_gather");
}

dl_status dl_token_select(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                          const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                          int chunk_stride, int chunk_content, int topT, const int32_t* Kexp,
                          int32_t* tok_pos, int32_t* tok_cnt, void* ws, size_t ws_bytes,
                          void* stream) {
  (void)ws;
  (void)ws_bytes;
  dl::Shape s;
  dl_status st = check_desc(desc, &s);
  if (st != DL_OK) return st;
  if (!Q_dec || !K_pool || !page_table || !chunk_idx || !tok_pos || !tok_cnt)
    return fail(DL_ERR_INVALID_ARG, "dl_token_select: NULL pointer");
  if (!aligned16(K_pool)) return fail(DL_ERR_INVALID_ARG, "K_pool not 16-byte aligned");
  if (n_sel < 1 || n_sel > 65535) return fail(DL_ERR_INVALID_ARG, "n_sel=%d", n_sel);
  if (chunk_content < 1 || chunk_content > 1024)
    return fail(DL_ERR_INVALID_ARG, "chunk_content=%d (need 1..1024)", chunk_content);
  if (topT < 0 || topT > chunk_content)
    return fail(DL_ERR_INVALID_ARG, "topT=%d (need 0..chunk_content)", topT);
  if (chunk_stride < chunk_content + 1)
    return fail(DL_ERR_INVALID_ARG, "chunk_stride=%d < chunk_content+1", chunk_stride);
  unsigned* err = nullptr;
  if ((st = error_word(&err)) != DL_OK) return st;
  return launched(dl::launch_token_select(s, Q_dec, K_pool, page_table, chunk_idx, n_sel,
                                          chunk_stride, chunk_content, topT, Kexp, tok_pos,
                                          tok_cnt, err, as_stream(stream)),
                  "dl_token_select launch");
}

}  // extern "C"
