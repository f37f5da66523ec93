// Internal launcher interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/dl.h"

namespace dl {

// Device error word codes (bit flags, OR-ed into the word).
constexpr unsigned ERR_BAD_INDEX = 1u;
constexpr unsigned ERR_TIMEOUT = 2u;

// Validated shape of one layer's attention problem.
struct Shape {
  int batch, H, H_kv, G, d, L_ctx, L_q, page, n_pages, n_slots, dtype;
  double scale;  // 1/sqrt(d)
};

constexpr int kTile = 64;          // keys per attention tile (= page size)
constexpr int kMaxSplits = 64;     // split-KV partitions per (b, g)
constexpr int kSinkTile = 256;     // context tokens per sink-pass CTA

// Attention key sources.
enum AttnMode { kDense = 0, kBlocks = 1, kGather = 2 };

struct AttnArgs {
  Shape s;
  const void* Q;
  const void* Kp;
  const void* Vp;
  const int32_t* page_table;
  int mode;
  const int32_t* idx;   // blk_idx or tok_pos
  const int32_t* cnt;   // blk_cnt or tok_cnt
  int max_idx;          // row length of idx (max_sel or max_tok)
  const void* Kd;
  const void* Vd;
  void* O;
  float* lse;
  void* ws;
  size_t ws_bytes;
  unsigned* err;
};

// ---- workspace sizing (bytes; each region rounded up to 256) ----
size_t attn_workspace(const Shape& s);
size_t scores_workspace(const Shape& s, int n_units);
size_t sinks_workspace(const Shape& s);
int attn_splits(const Shape& s, int max_ctx_tiles);

// ---- launchers (return the launch error) ----
cudaError_t launch_predict(const float* conf, const uint8_t* masked, int batch, int L_q, int k,
                           int w, int32_t* q_idx, int32_t* q_cnt, cudaStream_t st);

cudaError_t launch_pool(const Shape& s, const void* Kp, const int32_t* page_table, int n_units,
                        int stride, int offset, int len, float* Kbar, int8_t* Kdig,
                        int32_t* Kexp, unsigned* err, cudaStream_t st);

cudaError_t launch_scores(const Shape& s, const void* Q, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, int n_units, double* score,
                          void* ws, unsigned* err, cudaStream_t st);

cudaError_t launch_select(const double* score, int batch, int H_kv, int n_units, int unit_size,
                          int topK, const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                          int32_t* blk_cnt, int max_sel, unsigned* err, cudaStream_t st);
cudaError_t launch_block_select(const Shape& s, const void* Q, const int32_t* q_idx,
                                const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                                const int32_t* Kexp, int n_units, double* score, int unit_size,
                                int topK, const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                                int32_t* blk_cnt, int max_sel, int max_q, void* ws,
                                unsigned* err, cudaStream_t st);

bool block_select_tc_supported(const Shape& s, int rows, int n_units);
cudaError_t launch_block_select_tc(const Shape& s, const void* Q, const int32_t* q_idx,
                                   const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                                   const int32_t* Kexp, int n_units, double* score,
                                   int unit_size, int topK, const int32_t* sink_pos,
                                   int n_sinks, int32_t* blk_idx, int32_t* blk_cnt, int max_sel,
                                   int rows, unsigned* err, cudaStream_t st);
cudaError_t read_select_counts(unsigned long long* fast, unsigned long long* fallback);

bool block_select_wide_supported(const Shape& s, int rows, int n_units);
cudaError_t launch_block_select_wide(const Shape& s, const void* Q, const int32_t* q_idx,
                                     const int32_t* q_cnt, const float* Kbar, int n_units,
                                     double* score, int unit_size, int topK,
                                     const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                                     int32_t* blk_cnt, int max_sel, int rows, unsigned* err,
                                     cudaStream_t st);
cudaError_t launch_sink_mass(const Shape& s, const void* Q, const int32_t* q_idx,
                             const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                             const void* Kd, float* mass, void* ws, unsigned* err,
                             cudaStream_t st);
cudaError_t launch_sink_topn_mass(float* mass, int batch, int L_ctx, int n_sinks,
                                  int32_t* sink_pos, cudaStream_t st);
cudaError_t launch_sinks(const Shape& s, const void* Q, const int32_t* q_idx,
                         const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                         const void* Kd, const int32_t* Kexp, int n_sinks, int32_t* sink_pos,
                         void* ws, unsigned* err, cudaStream_t st);
size_t sink_cert_workspace(const Shape& s);
bool sink_cert_supported(const Shape& s, int n_sinks);
cudaError_t launch_sink_cert(const Shape& s, const void* Q, const int32_t* q_idx,
                             const int32_t* q_cnt, const void* Kp, const int32_t* page_table,
                             const void* Kd, const int32_t* Kexp, int n_units, const float* mass,
                             int n_sinks, int32_t* sink_pos, void* ws, unsigned* err,
                             cudaStream_t st);

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);

cudaError_t launch_cache_write(const Shape& s, const void* K_new, const void* V_new, int n_new,
                               const int32_t* start, const int32_t* page_table, void* Kp,
                               void* Vp, float* Kbar, int8_t* Kdig, int32_t* Kexp, unsigned* err,
                               cudaStream_t st);
cudaError_t launch_token_select(const Shape& s, const void* Q, const void* Kp,
                                const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                                int chunk_stride, int chunk_content, int topT,
                                const int32_t* Kexp, int32_t* tok_pos, int32_t* tok_cnt,
                                unsigned* err, cudaStream_t st);

// Shared by entry points in several files (defined in api.cu).
dl_status api_check_desc(const dl_attn_desc* d, Shape* s);
dl_status api_error_word(unsigned** out);
dl_status api_fail(dl_status st, const char* msg);
dl_status api_ok();
unsigned kernel_flags();  // dl_set_kernel_flags (DL_FLAG_*)

__host__ __device__ inline size_t round256(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace dl
