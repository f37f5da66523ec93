/*
 * dl.h -- C ABI of the B200 (sm_100a) library for one denoising step of
 * sink-aware, query-predicted, block-sparse bidirectional attention over a
 * cached long-context KV (diffusion LLM inference).
 *
 * Method sources (page title, then the part of the page):
 *   [F1] "Focus-dLLM: Accelerating Long-Context Diffusion LLM Inference via
 *        Confidence-Guided Context Focusing" -- abstract.
 *   [F2] same paper -- research.elamur.ai summary and key points.
 *   [P1] "Prefilling-dLLM: Predictive Prefilling for Long-Context Inference
 *        in Diffusion Language Models" -- abstract.
 *
 * Conventions shared by every call
 *   - Every pointer argument is caller-owned DEVICE memory unless stated.
 *     The library allocates nothing; calls that need scratch take a
 *     caller-provided workspace (size from dl_workspace_size).
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as
 *     void*; NULL means the legacy default stream) and returns a dl_status.
 *     Argument errors are reported before anything is launched; the message
 *     is available from dl_last_error_message() on the calling thread.
 *   - Out-of-range indices read from device memory (page-table slots, block
 *     indices, token positions, sink positions) are detected by the kernels:
 *     the offending tile is skipped and a device error word is set, which
 *     dl_get_status() reports as DL_ERR_BAD_INDEX.  No kernel traps.
 *   - Shapes: b = sequence, h = query head, g = KV head, G = H / H_kv query
 *     heads per KV head, d = head dimension, L_q = decode-block length.
 *   - scale = 1/sqrt(d) for scoring and attention (the pages give none; the
 *     standard scaled dot product is used).
 *   - Layouts (row-major, innermost last):
 *       Q_dec          [batch][H][L_q][d]          bf16 or fp32
 *       K_dec, V_dec   [batch][H_kv][L_q][d]       same dtype as Q_dec
 *       K_pool, V_pool [n_slots][H_kv][page][d]    same dtype; one page of one
 *                                                  KV head is page*d contiguous
 *       page_table     int32 [batch][n_pages]      logical page -> pool slot
 *       O              [batch][L_q][H][d]          dtype of the inputs
 *       lse            fp32 [batch][H][L_q]        natural-log LSE of the
 *                                                  scaled logits of each row
 *     Logical token t of sequence b lives in slot page_table[b][t / page],
 *     row t % page.  A contiguous cache uses the identity page table.
 */
#ifndef DL_H
#define DL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DL_OK = 0,
  DL_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, shape out of range      */
  DL_ERR_UNSUPPORTED = 2,  /* d not in {64,128}, page != 64, dtype mix, ...    */
  DL_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required       */
  DL_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed             */
  DL_ERR_BAD_INDEX = 5,    /* device-detected out-of-range index (dl_get_status) */
  DL_ERR_TIMEOUT = 6       /* a bounded device wait gave up (dl_get_status)    */
} dl_status;

typedef enum { DL_BF16 = 0, DL_FP32 = 1 } dl_dtype;

/* Shape of one layer's attention problem. */
typedef struct {
  int batch;    /* sequences                                               */
  int H;        /* query heads                                             */
  int H_kv;     /* KV heads; H % H_kv == 0                                 */
  int d;        /* head dimension: 64 or 128                               */
  int L_ctx;    /* logical context tokens per sequence (same for all b);   */
                /* tokens at t >= L_ctx are never read                     */
  int L_q;      /* decode-block length, 1..256                             */
  int page;     /* tokens per pool page = key-block size B; must be 64     */
  int n_pages;  /* logical pages per sequence (row length of page_table);  */
                /* n_pages * page >= L_ctx                                 */
  int n_slots;  /* pages in the pool                                       */
  int dtype;    /* dl_dtype of Q_dec, K/V pools, K_dec/V_dec and O         */
} dl_attn_desc;

/* Kernel-choice switches.  They exist for the tests, which run every kernel
 * of a step against the oracle: each switch sends a call to another kernel
 * that computes the same result.  The default, 0, is the product path.
 *   DL_FLAG_TOKEN_SIMT   dl_token_select on its CUDA-core kernel
 *   DL_FLAG_GATHER_SIMT  dl_sparse_attn_gather on its CUDA-core kernel
 *   DL_FLAG_PDL          every kernel launched with programmatic dependent
 *                        launch (measured no faster inside a CUDA graph)
 *   DL_FLAG_SCORE_FP64   dl_block_select always on the fp64 scoring kernel
 *                        (skips the certified integer tensor-core scoring)
 * Process-wide; read by each later call at launch time.  No environment
 * variable changes the kernel choice.  Returns the previous flags. */
enum { DL_FLAG_TOKEN_SIMT = 1u, DL_FLAG_GATHER_SIMT = 2u, DL_FLAG_PDL = 4u,
       DL_FLAG_SCORE_FP64 = 8u };
unsigned dl_set_kernel_flags(unsigned flags);

/* Counters of dl_block_select's int8 tensor-core kernel on the current
 * device since the last call (then cleared): fast = (b, g) selections kept
 * from the certified integer scores, fallback = (b, g) recomputed in fp64
 * because the certificate did not hold.  Synchronises the device. */
dl_status dl_read_counters(unsigned long long* fast, unsigned long long* fallback);

/* Library version (major*10000 + minor*100 + patch). */
int dl_version(void);

/* Message of the last error returned on this thread ("" if none). */
const char* dl_last_error_message(void);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device.  Returns DL_OK, DL_ERR_BAD_INDEX, DL_ERR_TIMEOUT or
 * DL_ERR_CUDA. */
dl_status dl_get_status(void* stream);

/* Bytes of workspace that suffice for every call below made with `desc`
 * (any number of selected blocks or gathered tokens).  The workspace needs
 * 256-byte alignment; its contents need no initialisation and are not
 * preserved between calls.  Calls that share one workspace must be ordered
 * (same stream). */
dl_status dl_workspace_size(const dl_attn_desc* desc, size_t* bytes);

/* (a1) Past-confidence-guided query prediction.  [F2 summary; key point 1]
 * For each sequence: among positions with still_masked != 0 take the top-k
 * by conf_prev (ties -> lower index; all of them if fewer than k are masked),
 * widen each chosen p to [p-w, p+w] clipped to [0, L_q), and write the union
 * in ascending order.
 *   conf_prev    fp32  [batch][L_q]   finite values
 *   still_masked uint8 [batch][L_q]
 *   q_idx        int32 [batch][L_q]   out: positions, then -1 padding
 *   q_cnt        int32 [batch]        out: number of predicted positions
 * Requires 1 <= L_q <= 1024, k >= 0, w >= 0. */
dl_status dl_predict_queries(const float* conf_prev, const uint8_t* still_masked, int batch,
                             int L_q, int k, int w, int32_t* q_idx, int32_t* q_cnt,
                             void* stream);

/* (a2) Mean-pooled keys.  [F2 summary: predicted queries select the most
 * relevant KV; pooling reading: one mean key per block]
 * Unit u of sequence b covers logical tokens
 *   [u*unit_stride + unit_offset, u*unit_stride + unit_offset + unit_len)
 * clipped to [0, L_ctx).  Kbar[b][g][u] = (sum of those K rows) / n, the
 * sum taken in fp64 (exact for bf16 keys; for fp32 keys exact while the
 * summed values' exponents lie within 29 - log2(n) binades of each other),
 * rounded once to fp32 (units with no valid token get 0).  Key blocks use
 * (stride, offset, len) = (page, 0, page); Prefilling-dLLM chunks [P1] with a
 * BOS anchor first use (chunk_stride, 1, chunk_content).
 *   K_pool  see layouts;  Kbar fp32 [batch][H_kv][n_units][d]  (out)
 * Kdig/Kexp (both NULL, or both set): the same pooled keys also written as
 * integer digits, the form dl_block_select's int8 tensor-core scoring reads
 * (an implementation format; the pages describe no such thing):
 *   Kdig int8  [batch][H_kv][5][n_units][d]  (out; 16-byte aligned)
 *   Kexp int32 [batch][H_kv][n_units]        (out)
 * With E the largest biased exponent field of the unit's d values (at least
 * 1), every value x = sign * m * 2^(e - 150) is held as the integer
 * V = trunc(m * 2^(11 - (E - e))), negated for x < 0, i.e. x~ = V * 2^(E-161),
 * and V = d0*2^28 + d1*2^21 + d2*2^14 + d3*2^7 + d4 with d0 in [-128, 127]
 * (plane 0) and d1..d4 in [0, 127] (planes 1..4).  Kexp = E | (number of the
 * unit's values with x~ != x) << 8. */
dl_status dl_pool_keys(const dl_attn_desc* desc, const void* K_pool, const int32_t* page_table,
                       int n_units, int unit_stride, int unit_offset, int unit_len,
                       float* Kbar, int8_t* Kdig, int32_t* Kexp, void* stream);

/* Cache refresh with the block pooling fused into the write.  [F2 summary:
 * the context is held in a KV cache; blocks are scored by their mean key]
 * A finished decode block's n_new tokens of every sequence b join the cached
 * context at logical positions start[b] .. start[b] + n_new - 1: they are
 * written into the pools through the page table, and the pooled key of every
 * block those positions touch is recomputed as dl_pool_keys (page, 0, page)
 * would (mean over the block's positions < L_ctx, in fp64, rounded once to
 * fp32; the block's other rows are read back from the pool).  For bf16 the
 * result equals dl_pool_keys' bit for bit; for fp32 keys the fp64 sums of
 * the two calls are taken in different orders and the pooled key can differ
 * by one fp32 ulp.  Other blocks of Kbar are left as they are.  The
 * descriptor describes the context after the write: start[b] + n_new <=
 * L_ctx, else that sequence is skipped entirely and DL_ERR_BAD_INDEX is
 * reported.  Blocks are checked one by one: a touched block whose page slot
 * is out of range is skipped (its pool rows and its Kbar entry are not
 * written) and DL_ERR_BAD_INDEX is reported, while the sequence's other
 * touched blocks are still written, so that sequence's cache is then
 * partly updated.
 *   K_new, V_new  [batch][H_kv][n_new][d] (bf16/fp32, 16-byte aligned)
 *   start         int32 [batch] (device)
 *   K_pool, V_pool, page_table  see layouts (written / read)
 *   Kbar          fp32 [batch][H_kv][n_blk][d]  (touched blocks written)
 *   Kdig, Kexp    NULL, or the digit form of Kbar as dl_pool_keys writes it
 *                 (touched blocks rewritten, n_units = n_blk) */
dl_status dl_cache_write(const dl_attn_desc* desc, const void* K_new, const void* V_new,
                         int n_new, const int32_t* start, const int32_t* page_table,
                         void* K_pool, void* V_pool, float* Kbar, int8_t* Kdig, int32_t* Kexp,
                         void* stream);

/* (a3) Block scores with a fused block-level softmax.  [F2 summary]
 * For KV head g, rows r = (h in g's query heads, i in predicted positions):
 *   score[b][g][j] = sum_r softmax_j( scale * q_{h,i} . Kbar[b][g][j] )
 * computed in fp64 from the bf16/fp32 queries and fp32 pooled keys.
 * q_idx/q_cnt as written by dl_predict_queries; q_idx == NULL means every
 * decode position is a row (q_cnt ignored).  q_cnt[b] == 0 gives all-zero
 * scores.
 *   score fp64 [batch][H_kv][n_units]  (out) */
dl_status dl_block_scores(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, int n_units, double* score,
                          void* ws, size_t ws_bytes, void* stream);

/* (a4) Attention-sink detection by attention mass.  [F1 abstract: sinks are
 * kept and their locations reused across layers]
 * mass[b][t] = sum over all heads h and predicted positions i of
 *   softmax over (context tokens t < L_ctx, and the L_q decode keys) of
 *   scale * q_{h,i} . k_t, for context columns t.
 * sink_pos[b] = the n_sinks columns of largest mass (ties -> lower index),
 * ascending.  Computed once, at the first sparse layer, and passed unchanged
 * to dl_select of every deeper layer.
 *   Kexp  int32 [batch][H_kv][ceil(L_ctx / page)] or NULL: the exponent words
 *         that dl_pool_keys (unit = page) or dl_cache_write wrote for this
 *         layer's current K pool; their norm field bounds every key's norm.
 *         Given, the cut is certified: the masses are taken in fp32, and
 *         where a proven bound on their error does not separate the n-th
 *         largest from the next, the undecided columns (or, past 512 of
 *         them, every column) get their masses again in fp64 and the sinks
 *         are those of the fp64 masses (exact up to fp64 rounding).  NULL:
 *         the top n of the fp32 masses (relative error about 1e-6).
 *   sink_pos int32 [batch][n_sinks]  (out);  1 <= n_sinks <= 64 */
dl_status dl_find_sinks(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                        const int32_t* q_cnt, const void* K_pool, const int32_t* page_table,
                        const void* K_dec, const int32_t* Kexp, int n_sinks, int32_t* sink_pos,
                        void* ws, size_t ws_bytes, void* stream);

/* (a4), split in its two halves for head-sharded execution.  The sink mass
 * is a sum over heads, so a GPU that holds only some KV heads (desc->H_kv
 * and desc->H of its shard, Q_dec / K_pool / K_dec of those heads only)
 * computes its shard's part of mass[b][t] with dl_sink_mass; the parts are
 * summed over the shards (an all-reduce of batch x L_ctx floats) and
 * dl_sink_topn picks the sinks from the sum.  On one GPU the two calls give
 * what dl_find_sinks gives.
 * dl_sink_mass: mass fp32 [batch][L_ctx] (out, device; every element
 *   written); the same arguments, checks and workspace as dl_find_sinks.
 *   The split calls take the top n of the fp32 sum without the certified
 *   recheck of dl_find_sinks.
 * dl_sink_topn: mass fp32 [batch][L_ctx] (device; in, not modified);
 *   sink_pos int32 [batch][n_sinks] (out), the n_sinks columns of largest
 *   mass (ties -> lower index), ascending.  1 <= n_sinks <= 64.
 *   No workspace.  Returns DL_ERR_INVALID_ARG for NULL pointers or sizes out
 *   of range, before any launch. */
dl_status dl_sink_mass(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                       const int32_t* q_cnt, const void* K_pool, const int32_t* page_table,
                       const void* K_dec, float* mass, void* ws, size_t ws_bytes, void* stream);
dl_status dl_sink_topn(float* mass, int batch, int L_ctx, int n_sinks, int32_t* sink_pos,
                       void* stream);

/* (a5) Sink-aware top-K block selection.  [F1 abstract; F2 summary]
 * For each (b, g): the sink units SB = { sink_pos[b][s] / unit_size : s,
 * sink_pos >= 0 } are always kept; the topK remaining units of largest score
 * (ties -> lower index) are added; the result is written ascending.
 *   score    fp64  [batch][H_kv][n_units]
 *   sink_pos int32 [batch][n_sinks] or NULL (n_sinks == 0)
 *   blk_idx  int32 [batch][H_kv][max_sel]  out: ascending units, -1 padding
 *   blk_cnt  int32 [batch][H_kv]           out: min(topK, n_units-|SB|)+|SB|
 * Requires max_sel >= min(topK, n_units) + n_sinks, n_units <= 16384. */
dl_status dl_select(const double* score, int batch, int H_kv, int n_units, int unit_size,
                    int topK, const int32_t* sink_pos, int n_sinks, int32_t* blk_idx,
                    int32_t* blk_cnt, int max_sel, void* stream);

/* (a3 + a5) Block scores and selection in one call: the results of
 * dl_block_scores followed by dl_select with the same arguments (score is
 * written too).  [F2 summary: the predicted queries rank the blocks; F1
 * abstract: the sinks are always kept]
 * Kernels, by shape:
 *  - bf16 queries, d 128, G * max_q <= 24, n_units <= 512, Kdig/Kexp given
 *    (the digits of these very Kbar, from dl_pool_keys / dl_cache_write) and
 *    DL_FLAG_SCORE_FP64 not set:
 *    one CTA per (b, g) takes the logits q . Kbar exactly on the int8 tensor
 *    cores (query digits times key digits, int32 sums), in fp64 from there
 *    on, with a proven bound on each logit's error (the truncated digits);
 *    the selection is kept when the gap between the K-th and (K+1)-th score
 *    exceeds the bound, and otherwise that (b, g) is recomputed by the fp64
 *    kernel below inside the same CTA.  The selected blocks are then those of
 *    the exact scores; score holds values within a relative 1e-9 of them.
 *  - otherwise, G * max_q <= 32 and n_units <= 512: one kernel per (b, g)
 *    computing the scores in fp64 (the scores then stay on chip between the
 *    two steps; bf16 or fp32 queries, d 64 or 128);
 *  - otherwise the two separate kernels.
 * max_q: an upper bound of q_cnt[b] that the caller guarantees (with the
 *   prediction of dl_predict_queries: min(L_q, k * (2w + 1))); 0 = L_q.  The
 *   fused kernels are compiled for that many rows; a sequence with more rows
 *   is cut to the bound and reported as DL_ERR_BAD_INDEX by dl_get_status.
 * Other arguments, layouts and requirements as for dl_block_scores and
 * dl_select; ws: workspace of dl_workspace_size (used only by the separate
 * kernels). */
dl_status dl_block_select(const dl_attn_desc* desc, const void* Q_dec, const int32_t* q_idx,
                          const int32_t* q_cnt, const float* Kbar, const int8_t* Kdig,
                          const int32_t* Kexp, int n_units, int unit_size, int topK,
                          const int32_t* sink_pos, int n_sinks, double* score, int32_t* blk_idx,
                          int32_t* blk_cnt, int max_sel, int max_q, void* ws, size_t ws_bytes,
                          void* stream);

/* (a6) Block-sparse bidirectional attention.  [F1 abstract; F2 summary]
 * For every query head h (KV head g) and decode position i:
 *   o_{h,i} = sum_{t in S} softmax_t(scale * q_{h,i} . k_t) v_t
 * where S = valid tokens (< L_ctx) of the blocks blk_idx[b][g][0..blk_cnt)
 * (read through the page table, possibly non-contiguous) plus all L_q
 * decode keys; no causal mask.  bf16 in, fp32 accumulation, online softmax;
 * O rounded to nearest-even in the input dtype; lse optional (NULL: not
 * written).  blk_idx == NULL selects every block (dense shallow layers).
 *   blk_idx int32 [batch][H_kv][max_sel], blk_cnt int32 [batch][H_kv]
 * Q_dec/K_pool/V_pool/K_dec/V_dec/O must be 16-byte aligned. */
dl_status dl_sparse_attn(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                         const void* V_pool, const int32_t* page_table, const int32_t* blk_idx,
                         const int32_t* blk_cnt, int max_sel, const void* K_dec,
                         const void* V_dec, void* O, float* lse, void* ws, size_t ws_bytes,
                         void* stream);

/* (a7) Intra-chunk token selection for a chunked prefix.  [P1 abstract]
 * For each (b, g) and each selected chunk c = chunk_idx[b][g][s]: rows r =
 * every decode query of g's heads;
 *   tau[t] = sum_r softmax_t(scale * q_r . k_t) over the chunk's content
 *            tokens t = c*chunk_stride + 1 .. c*chunk_stride + chunk_content
 * The topT tokens of largest tau (ties -> lower position) and the chunk's BOS
 * anchor at c*chunk_stride are kept.  tok_pos[b][g] receives all kept
 * logical positions of the n_sel selected chunks, ascending; tok_cnt[b][g]
 * their number (n_sel * (min(topT, chunk_content) + 1)).
 *   chunk_idx int32 [batch][H_kv][n_sel] (from dl_select over chunks)
 *   Kexp      int32 [batch][H_kv][ceil(L_ctx / chunk_stride)] or NULL: the
 *             exponent words of the chunk keys (dl_pool_keys over the chunks'
 *             content tokens); their norm field bounds the content keys'
 *             norms.  Given (tensor-core kernel: bf16, d 128), the top-T cut
 *             is certified: where a proven bound on the fp32 masses' error
 *             does not separate the T-th from the next, the CTA recomputes
 *             the undecided tokens' masses in fp64 and keeps the top T of
 *             those.  NULL (or the CUDA-core kernel): the top T of the fp32
 *             masses.
 *   tok_pos   int32 [batch][H_kv][n_sel*(topT+1)]  (out)
 * Requires 1 <= chunk_content <= 1024, 0 <= topT <= chunk_content. */
dl_status dl_token_select(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                          const int32_t* page_table, const int32_t* chunk_idx, int n_sel,
                          int chunk_stride, int chunk_content, int topT, const int32_t* Kexp,
                          int32_t* tok_pos, int32_t* tok_cnt, void* ws, size_t ws_bytes,
                          void* stream);

/* (a7) Attention over gathered, non-contiguous cached tokens plus the decode
 * block.  [P1 abstract: a kernel that parallelises decoding over the
 * non-contiguously cached chunk KV]
 * As dl_sparse_attn with S = logical positions tok_pos[b][g][0..tok_cnt)
 * (each < n_pages*page) plus the L_q decode keys.  A position out of range,
 * or one whose page-table slot is, is reported through dl_get_status
 * (DL_ERR_BAD_INDEX) and that (b, g)'s output is then unspecified.
 *   tok_pos int32 [batch][H_kv][max_tok], tok_cnt int32 [batch][H_kv] */
dl_status dl_sparse_attn_gather(const dl_attn_desc* desc, const void* Q_dec, const void* K_pool,
                                const void* V_pool, const int32_t* page_table,
                                const int32_t* tok_pos, const int32_t* tok_cnt, int max_tok,
                                const void* K_dec, const void* V_dec, void* O, float* lse,
                                void* ws, size_t ws_bytes, void* stream);

/* Allocation-free variant of dl_block_scores.  The pages describe no
 * counterpart: this serves callers that cannot allocate device memory (a
 * runtime that owns all allocations and has no workspace to give, code where
 * cudaMalloc is not allowed because it may synchronise the device, a process
 * whose footprint is fixed after start-up).
 * Same arguments and results as dl_block_scores, minus the workspace: the
 * scratch is a 32 MiB array built into the library (held on every GPU that
 * loads it until exit).  Calls needing more return DL_ERR_WORKSPACE; the
 * need is batch*H*L_q*(8*n128 + 16*n128/128) bytes, n128 = n_units rounded
 * up to a multiple of 128.  All calls on a
 * device share the array; calls whose kernels may overlap on the GPU race on
 * it and must be ordered (one stream).  The first call on each device looks
 * up the array's device address, so make it before any stream capture.  The
 * call allocates nothing. */
dl_status dl_block_scores_noalloc(const dl_attn_desc* desc, const void* Q_dec,
                                  const int32_t* q_idx, const int32_t* q_cnt, const float* Kbar,
                                  int n_units, double* score, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DL_H */
