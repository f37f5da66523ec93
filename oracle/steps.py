"""The steps of the sparse denoising step, one plain fp64 definition each.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.  Arrays are numpy float64 unless stated; integer outputs are
numpy int64.  Functions work on one sequence (and one KV head where stated).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "scale_for", "topk_lower_index", "predict_queries", "pool_mean", "pooled_keys",
    "block_scores", "select_blocks", "find_sinks", "attention_rows",
    "gather_context", "sparse_attention", "dense_attention", "chunk_pooled_keys",
    "chunk_scores", "token_select", "chunk_attention", "cache_write",
]


def f64(x) -> np.ndarray:
    """Exact conversion of a torch tensor (bf16/fp32/...) or array to float64."""
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def scale_for(d: int) -> float:
    """Reading R1: the pages give no scale; standard 1/sqrt(d)."""
    return 1.0 / np.sqrt(np.float64(d))


def topk_lower_index(values: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest values in rank order; equal values rank by the
    lower index (stable sort of the negated values)."""
    order = np.argsort(-np.asarray(values, dtype=np.float64), kind="stable")
    return order[: max(0, min(k, len(order)))]


def _softmax_rows(S: np.ndarray) -> np.ndarray:
    """Two-pass softmax along the last axis: max, sum of exponentials, divide."""
    m = S.max(axis=-1, keepdims=True)
    E = np.exp(S - m)
    return E / E.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------
# a1. past-confidence-guided prediction of the query positions
# --------------------------------------------------------------------------
def predict_queries(conf_prev, still_masked, k: int, w: int) -> np.ndarray:
    """Predicted query positions of one sequence, ascending.

    Focus-dLLM [F2, summary]: the previous step's confidence over the
    still-masked positions predicts which positions unmask next; those guesses
    are widened into local windows.  [F2, key point 1]: the k=4 highest-
    confidence masked tokens.  Reading R5: take the top-k masked positions by
    confidence (ties to the lower index; all of them if fewer than k are
    masked), mark [p-w, p+w] clipped to the decode block, return the union.
    """
    conf = f64(conf_prev).reshape(-1)
    masked = np.asarray(f64(still_masked)).reshape(-1) != 0
    L = conf.shape[0]
    cand = np.nonzero(masked)[0]                     # ascending positions
    order = cand[np.argsort(-conf[cand], kind="stable")]
    chosen = order[: min(k, len(order))]
    mark = np.zeros(L, dtype=bool)
    for p in chosen:
        mark[max(0, p - w): min(L, p + w + 1)] = True
    return np.nonzero(mark)[0]


# --------------------------------------------------------------------------
# a2. mean-pooled keys of a key block
# --------------------------------------------------------------------------
def pool_mean(tokens) -> np.ndarray:
    """Mean over the rows of `tokens` ([n][d]) in fp64."""
    t = f64(tokens)
    return t.sum(axis=0) / np.float64(t.shape[0])


def pooled_keys(K_ctx, L_ctx: int, B: int) -> np.ndarray:
    """Pooled keys of one KV head: [n_blk][d].

    Block j averages its valid tokens [jB, min((j+1)B, L_ctx)).  Reading R6:
    the fp64 mean is rounded once to fp32 (the stored precision) and returned
    as float64 holding those fp32 values."""
    K = f64(K_ctx)
    n_blk = -(-L_ctx // B)
    out = np.empty((n_blk, K.shape[-1]))
    for j in range(n_blk):
        out[j] = pool_mean(K[j * B: min((j + 1) * B, L_ctx)])
    return out.astype(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# a3. block scores with a block-level softmax
# --------------------------------------------------------------------------
def block_scores(Q_rows, Kbar, scale: float) -> np.ndarray:
    """score[j] = sum_r softmax_j(scale * q_r . Kbar_j)   (reading R2).

    Q_rows: [R][d] predicted query rows of every query head of one KV group;
    Kbar: [n][d] pooled keys.  With R = 0 every score is 0."""
    Q = f64(Q_rows)
    Kb = f64(Kbar)
    if Q.shape[0] == 0:
        return np.zeros(Kb.shape[0])
    S = scale * (Q @ Kb.T)
    return _softmax_rows(S).sum(axis=0)


# --------------------------------------------------------------------------
# a5. top-K blocks plus the sink blocks
# --------------------------------------------------------------------------
def select_blocks(score, sink_pos, B: int, topK: int) -> np.ndarray:
    """Selected blocks of one KV head, ascending (reading R3).

    Sink blocks SB = {p // B} of the (non-negative) sink positions are always
    kept [F1 abstract: sink-aware pruning preserves the sinks]; the top-K of
    the remaining blocks by score (ties to the lower index) are added."""
    score = f64(score).reshape(-1)
    n_blk = score.shape[0]
    sb = sorted({int(p) // B for p in np.asarray(sink_pos).reshape(-1) if int(p) >= 0})
    in_sb = np.zeros(n_blk, dtype=bool)
    in_sb[sb] = True
    cand = np.nonzero(~in_sb)[0]
    top = cand[np.argsort(-score[cand], kind="stable")][: min(topK, len(cand))]
    return np.sort(np.concatenate([top, np.asarray(sb, dtype=np.int64)]).astype(np.int64))


# --------------------------------------------------------------------------
# a4. sink columns by attention mass
# --------------------------------------------------------------------------
def find_sinks(Q, K_ctx, K_dec, q_idx, n_sinks: int, scale: float):
    """Sink positions of one sequence (reading R4) and the column masses.

    Q: [H][L_q][d]; K_ctx: [H_kv][L_ctx][d] (logical order); K_dec:
    [H_kv][L_q][d].  mass[t] = sum over heads h and predicted rows i of
    softmax over (context + decode keys) of scale * q_hi . k_t, for context
    columns t.  Returns (top n_sinks columns by mass with ties to the lower
    index, ascending; mass)."""
    Qf, Kc, Kd = f64(Q), f64(K_ctx), f64(K_dec)
    H, H_kv = Qf.shape[0], Kc.shape[0]
    G = H // H_kv
    L_ctx = Kc.shape[1]
    rows = np.asarray(q_idx, dtype=np.int64)
    mass = np.zeros(L_ctx)
    if len(rows):
        for h in range(H):
            g = h // G
            keys = np.concatenate([Kc[g], Kd[g]], axis=0)
            P = _softmax_rows(scale * (Qf[h, rows] @ keys.T))
            mass += P[:, :L_ctx].sum(axis=0)
    top = topk_lower_index(mass, n_sinks)
    return np.sort(top), mass


# --------------------------------------------------------------------------
# a6. attention over an explicit key set
# --------------------------------------------------------------------------
def attention_rows(Q_rows, keys, values, scale: float):
    """Textbook softmax(scale Q K^T) V with the natural-log LSE of each row."""
    Q, K, V = f64(Q_rows), f64(keys), f64(values)
    S = scale * (Q @ K.T)
    m = S.max(axis=1, keepdims=True)
    E = np.exp(S - m)
    Z = E.sum(axis=1, keepdims=True)
    return (E @ V) / Z, (m + np.log(Z)).reshape(-1)


def gather_context(pool, page_row, g: int, positions, B: int) -> np.ndarray:
    """Rows of KV head g at logical positions, read through the page table:
    position t lives in slot page_row[t // B], row t % B."""
    pos = np.asarray(positions, dtype=np.int64)
    P = f64(pool) if not isinstance(pool, np.ndarray) else pool
    slots = np.asarray(page_row, dtype=np.int64)[pos // B]
    return P[slots, g, pos % B]


def sparse_attention(Q, K_pool, V_pool, page_row, blk_sel, L_ctx: int, B: int,
                     K_dec, V_dec, scale: float):
    """Block-sparse bidirectional attention of one sequence.

    Focus-dLLM [F1, F2]: the decode-block queries attend only to the selected
    KV blocks plus the decode block itself, with no causal mask.  For KV head g
    the key set is the valid tokens (< L_ctx) of blocks blk_sel[g] and all
    L_q decode keys; every query head of the group uses it.
    Returns O [L_q][H][d] and lse [H][L_q]."""
    Qf = f64(Q)
    Kp = f64(K_pool)
    Vp = f64(V_pool)
    Kd, Vd = f64(K_dec), f64(V_dec)
    H, L_q, d = Qf.shape
    H_kv = Kd.shape[0]
    G = H // H_kv
    O = np.empty((L_q, H, d))
    lse = np.empty((H, L_q))
    for g in range(H_kv):
        blocks = np.asarray(blk_sel[g], dtype=np.int64)
        pos = (blocks[:, None] * B + np.arange(B)[None, :]).reshape(-1)
        pos = pos[pos < L_ctx]
        keys = np.concatenate([gather_context(Kp, page_row, g, pos, B), Kd[g]], axis=0)
        vals = np.concatenate([gather_context(Vp, page_row, g, pos, B), Vd[g]], axis=0)
        for h in range(g * G, (g + 1) * G):
            o, l = attention_rows(Qf[h], keys, vals, scale)
            O[:, h] = o
            lse[h] = l
    return O, lse


def dense_attention(Q, K_pool, V_pool, page_row, L_ctx: int, B: int, K_dec, V_dec,
                    scale: float):
    """Full bidirectional attention: every block selected (shallow layers,
    Focus-dLLM [F2 summary])."""
    H_kv = K_dec.shape[0]
    n_blk = -(-L_ctx // B)
    sel = [np.arange(n_blk)] * H_kv
    return sparse_attention(Q, K_pool, V_pool, page_row, sel, L_ctx, B, K_dec, V_dec, scale)


# --------------------------------------------------------------------------
# a7. chunked prefix: chunk scores, intra-chunk token selection, attention
# --------------------------------------------------------------------------
def chunk_pooled_keys(K_pool, page_row, g: int, n_chunks: int, stride: int,
                      content: int, B: int) -> np.ndarray:
    """Pooled key of each chunk of KV head g (reading R7): the mean of its
    content tokens at logical positions c*stride + 1 .. c*stride + content
    (the BOS anchor at c*stride is left out), rounded once to fp32 (R6)."""
    out = np.empty((n_chunks, K_pool.shape[-1]))
    for c in range(n_chunks):
        pos = c * stride + 1 + np.arange(content)
        out[c] = pool_mean(gather_context(K_pool, page_row, g, pos, B))
    return out.astype(np.float32).astype(np.float64)


def chunk_scores(Q_rows, Kbar_chunks, scale: float) -> np.ndarray:
    """Prefilling-dLLM [P1]: rank chunks for relevance.  Same block-softmax
    score as a3 with chunks as the blocks and every decode query as a row."""
    return block_scores(Q_rows, Kbar_chunks, scale)


def token_select(Q_rows, chunk_keys, T: int, scale: float):
    """Intra-chunk token sparsity [P1]: tau[t] = sum_r softmax_t(scale q_r.k_t)
    over the chunk's content tokens; the top-T tokens (ties to the lower
    index), ascending, as offsets into the content.  Returns (offsets, tau)."""
    P = _softmax_rows(scale * (f64(Q_rows) @ f64(chunk_keys).T))
    tau = P.sum(axis=0)
    return np.sort(topk_lower_index(tau, T)), tau


def chunk_attention(Q, K_pool, V_pool, page_row, positions_per_g, B: int, K_dec, V_dec,
                    scale: float):
    """Attention of one sequence over explicit logical token positions per KV
    head plus the decode block.  Returns O [L_q][H][d], lse [H][L_q]."""
    Qf = f64(Q)
    Kp, Vp = f64(K_pool), f64(V_pool)
    Kd, Vd = f64(K_dec), f64(V_dec)
    H, L_q, d = Qf.shape
    H_kv = Kd.shape[0]
    G = H // H_kv
    O = np.empty((L_q, H, d))
    lse = np.empty((H, L_q))
    for g in range(H_kv):
        pos = np.asarray(positions_per_g[g], dtype=np.int64)
        keys = np.concatenate([gather_context(Kp, page_row, g, pos, B), Kd[g]], axis=0)
        vals = np.concatenate([gather_context(Vp, page_row, g, pos, B), Vd[g]], axis=0)
        for h in range(g * G, (g + 1) * G):
            O[:, h], lse[h] = attention_rows(Qf[h], keys, vals, scale)
    return O, lse


# --------------------------------------------------------------------------
# cache refresh: a finished decode block written into the paged cache, with
# the pooled keys of the blocks it touches
# --------------------------------------------------------------------------
def cache_write(K_pool, V_pool, page_row, K_new, V_new, start: int, L_ctx: int, B: int):
    """The decode block's tokens join the cached context (Focus-dLLM summary:
    the context is held in a KV cache; its pooled block keys are what the
    block scores read).  K_new, V_new: [H_kv][n_new][d] at logical positions
    start .. start + n_new - 1, written through the page table (slot
    page_row[t // B], row t % B); then every block j those positions touch
    gets the pooled key of pooled_keys (mean of its positions < L_ctx, read
    back through the page table, rounded once to fp32).  Returns the updated
    pools (copies) and {j: Kbar_j [H_kv][d]}."""
    Kp = np.array(f64(K_pool), copy=True)
    Vp = np.array(f64(V_pool), copy=True)
    Kn, Vn = f64(K_new), f64(V_new)
    row = np.asarray(page_row, dtype=np.int64)
    n_new = Kn.shape[1]
    for t in range(n_new):
        pos = start + t
        Kp[row[pos // B], :, pos % B] = Kn[:, t]
        Vp[row[pos // B], :, pos % B] = Vn[:, t]
    kbar = {}
    for j in range(start // B, (start + n_new - 1) // B + 1):
        pos = np.arange(j * B, min((j + 1) * B, L_ctx))
        kbar[j] = np.stack([pool_mean(gather_context(Kp, row, g, pos, B))
                            for g in range(Kp.shape[1])]).astype(np.float32).astype(np.float64)
    return Kp, Vp, kbar
