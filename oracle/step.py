"""One layer of the denoising step, and the chunked-prefix step, assembled
from the per-step definitions in `steps.py`, in the order the pages give:
predict the queries, score the blocks, (find sinks,) select, attend.

TEST INFRASTRUCTURE ONLY: never imported by the product path.

Outputs use the same array layouts as the library (so tests compare them
element by element): padding entries of index arrays are -1.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from . import steps as S


@dataclasses.dataclass
class StepResult:
    q_idx: np.ndarray      # int [batch][L_q], ascending, -1 padded
    q_cnt: np.ndarray      # int [batch]
    Kbar: np.ndarray       # fp32 values as fp64 [batch][H_kv][n_blk][d]
    score: np.ndarray      # fp64 [batch][H_kv][n_blk]
    sink_pos: np.ndarray   # int [batch][n_sinks] (or empty)
    blk_idx: np.ndarray    # int [batch][H_kv][max_sel], ascending, -1 padded
    blk_cnt: np.ndarray    # int [batch][H_kv]
    O: np.ndarray          # fp64 [batch][L_q][H][d]
    lse: np.ndarray        # fp64 [batch][H][L_q]
    sink_mass: Optional[np.ndarray] = None  # fp64 [batch][L_ctx] when detected


def _pad(rows, width):
    out = np.full((len(rows), width), -1, dtype=np.int64)
    for i, r in enumerate(rows):
        out[i, : len(r)] = r
    return out


def logical_context(pool, page_row, g, L_ctx, B):
    """K (or V) of KV head g for logical positions 0..L_ctx-1, [L_ctx][d]."""
    return S.gather_context(pool, page_row, g, np.arange(L_ctx), B)


def predict_all(conf_prev, still_masked, k, w):
    """a1 for every sequence: (q_idx padded, q_cnt)."""
    conf = S.f64(conf_prev)
    masked = S.f64(still_masked)
    rows = [S.predict_queries(conf[b], masked[b], k, w) for b in range(conf.shape[0])]
    return _pad(rows, conf.shape[1]), np.array([len(r) for r in rows], dtype=np.int64)


def layer_step(q_dec, k_pool, v_pool, page_table, k_dec, v_dec, L_ctx: int, B: int,
               topK: int, *, conf_prev=None, still_masked=None, k: int = 4, w: int = 2,
               q_idx=None, q_cnt=None, sink_pos=None, detect_sinks: int = 0,
               dense: bool = False, n_sinks_cap: Optional[int] = None) -> StepResult:
    """One layer of one denoising step for a batch.

    Either predicts the queries from (conf_prev, still_masked) or takes them
    (q_idx, q_cnt).  Sinks are given (sink_pos [batch][n], entries < 0
    ignored) or detected over this layer (detect_sinks columns).  dense=True
    selects every block (shallow layers keep full attention)."""
    Q = S.f64(q_dec)
    Kp, Vp = S.f64(k_pool), S.f64(v_pool)
    Kd, Vd = S.f64(k_dec), S.f64(v_dec)
    pt = np.asarray(page_table, dtype=np.int64)
    batch, H, L_q, d = Q.shape
    H_kv = Kd.shape[1]
    G = H // H_kv
    n_blk = -(-L_ctx // B)
    scale = S.scale_for(d)

    if q_idx is None:
        q_idx, q_cnt = predict_all(conf_prev, still_masked, k, w)
    q_idx = np.asarray(q_idx, dtype=np.int64)
    q_cnt = np.asarray(q_cnt, dtype=np.int64)

    Kbar = np.zeros((batch, H_kv, n_blk, d))
    score = np.zeros((batch, H_kv, n_blk))
    for b in range(batch):
        rows = q_idx[b, : q_cnt[b]]
        for g in range(H_kv):
            Kbar[b, g] = S.pooled_keys(logical_context(Kp, pt[b], g, L_ctx, B), L_ctx, B)
            Qg = Q[b, g * G:(g + 1) * G][:, rows].reshape(-1, d)
            score[b, g] = S.block_scores(Qg, Kbar[b, g], scale)

    mass = None
    if detect_sinks:
        sinks = np.zeros((batch, detect_sinks), dtype=np.int64)
        mass = np.zeros((batch, L_ctx))
        for b in range(batch):
            Kc = np.stack([logical_context(Kp, pt[b], g, L_ctx, B) for g in range(H_kv)])
            rows = q_idx[b, : q_cnt[b]]
            sinks[b], mass[b] = S.find_sinks(Q[b], Kc, Kd[b], rows, detect_sinks, scale)
    elif sink_pos is not None:
        sinks = np.asarray(sink_pos, dtype=np.int64).reshape(batch, -1)
    else:
        sinks = np.zeros((batch, 0), dtype=np.int64)

    n_s = sinks.shape[1] if n_sinks_cap is None else n_sinks_cap
    max_sel = n_blk if dense else min(topK, n_blk) + n_s
    blk_idx = np.full((batch, H_kv, max_sel), -1, dtype=np.int64)
    blk_cnt = np.zeros((batch, H_kv), dtype=np.int64)
    O = np.zeros((batch, L_q, H, d))
    lse = np.zeros((batch, H, L_q))
    for b in range(batch):
        sel = []
        for g in range(H_kv):
            if dense:
                s = np.arange(n_blk)
            else:
                s = S.select_blocks(score[b, g], sinks[b], B, topK)
            blk_idx[b, g, : len(s)] = s
            blk_cnt[b, g] = len(s)
            sel.append(s)
        O[b], lse[b] = S.sparse_attention(Q[b], Kp, Vp, pt[b], sel, L_ctx, B, Kd[b], Vd[b],
                                          scale)
    return StepResult(q_idx=q_idx, q_cnt=q_cnt, Kbar=Kbar, score=score, sink_pos=sinks,
                      blk_idx=blk_idx, blk_cnt=blk_cnt, O=O, lse=lse, sink_mass=mass)


def denoise_block(k_pool, v_pool, page_table, steps, L_ctx: int, B: int, topK: int, *,
                  first_sparse: int, n_sinks: int, k: int = 4, w: int = 2):
    """The denoising steps of one decode block over a multi-layer model
    (reading R8).

    k_pool / v_pool: per layer, the cached context, unchanged while the block
    is decoded; steps: per step, a dict with conf_prev, still_masked and the
    per-layer lists q_dec, k_dec, v_dec.  Every step predicts its own query
    positions; layers below first_sparse attend densely; the first step finds
    the n_sinks sinks at layer first_sparse, and every sparse layer of every
    step keeps them (the cached context they index does not change before
    the block is committed).  Returns, per step, the list of per-layer
    StepResults."""
    out = []
    sinks = None
    for t, st in enumerate(steps):
        q_idx, q_cnt = predict_all(st["conf_prev"], st["still_masked"], k, w)
        layers = []
        for l in range(len(k_pool)):
            args = (st["q_dec"][l], k_pool[l], v_pool[l], page_table, st["k_dec"][l],
                    st["v_dec"][l], L_ctx, B, topK)
            common = dict(q_idx=q_idx, q_cnt=q_cnt, k=k, w=w)
            if l < first_sparse:
                r = layer_step(*args, dense=True, **common)
            elif l == first_sparse and t == 0:
                r = layer_step(*args, detect_sinks=n_sinks, **common)
                sinks = r.sink_pos
            else:
                r = layer_step(*args, sink_pos=sinks, **common)
            layers.append(r)
        out.append(layers)
    return out


@dataclasses.dataclass
class ChunkResult:
    Kbar: np.ndarray       # fp64 (fp32 values) [batch][H_kv][n_chunks][d]
    score: np.ndarray      # fp64 [batch][H_kv][n_chunks]
    chunk_idx: np.ndarray  # int [batch][H_kv][K_c], ascending
    tok_pos: np.ndarray    # int [batch][H_kv][K_c*(T+1)], logical positions, ascending
    tau: np.ndarray        # fp64 [batch][H_kv][K_c][content]
    O: np.ndarray          # fp64 [batch][L_q][H][d]
    lse: np.ndarray        # fp64 [batch][H][L_q]


def chunked_step(q_dec, k_pool, v_pool, page_table, k_dec, v_dec, *, n_chunks: int,
                 stride: int, content: int, B: int, topK_chunks: int,
                 topT: int) -> ChunkResult:
    """Prefilling-dLLM-style step over a chunked, paged prefix (reading R7).

    Chunk c holds its BOS anchor at logical position c*stride and content
    tokens at c*stride+1 .. c*stride+content.  Per KV head: score chunks by
    pooled key with every decode query, keep the top-K chunks, keep the top-T
    content tokens of each by summed softmax mass, always add the chunk's BOS,
    then attend over those tokens plus the decode block."""
    Q = S.f64(q_dec)
    Kp, Vp = S.f64(k_pool), S.f64(v_pool)
    Kd, Vd = S.f64(k_dec), S.f64(v_dec)
    pt = np.asarray(page_table, dtype=np.int64)
    batch, H, L_q, d = Q.shape
    H_kv = Kd.shape[1]
    G = H // H_kv
    scale = S.scale_for(d)
    Kc = min(topK_chunks, n_chunks)
    Kbar = np.zeros((batch, H_kv, n_chunks, d))
    score = np.zeros((batch, H_kv, n_chunks))
    chunk_idx = np.zeros((batch, H_kv, Kc), dtype=np.int64)
    tok_pos = np.zeros((batch, H_kv, Kc * (topT + 1)), dtype=np.int64)
    tau = np.zeros((batch, H_kv, Kc, content))
    O = np.zeros((batch, L_q, H, d))
    lse = np.zeros((batch, H, L_q))
    for b in range(batch):
        per_g = []
        for g in range(H_kv):
            rows = Q[b, g * G:(g + 1) * G].reshape(-1, d)
            Kbar[b, g] = S.chunk_pooled_keys(Kp, pt[b], g, n_chunks, stride, content, B)
            score[b, g] = S.chunk_scores(rows, Kbar[b, g], scale)
            chosen = np.sort(S.topk_lower_index(score[b, g], Kc))
            chunk_idx[b, g] = chosen
            pos = []
            for ci, c in enumerate(chosen):
                keys = S.gather_context(Kp, pt[b], g, c * stride + 1 + np.arange(content), B)
                offs, tau[b, g, ci] = S.token_select(rows, keys, topT, scale)
                pos.append(np.concatenate([[c * stride], c * stride + 1 + offs]))
            pos = np.sort(np.concatenate(pos)).astype(np.int64)
            tok_pos[b, g] = pos
            per_g.append(pos)
        O[b], lse[b] = S.chunk_attention(Q[b], Kp, Vp, pt[b], per_g, B, Kd[b], Vd[b], scale)
    return ChunkResult(Kbar=Kbar, score=score, chunk_idx=chunk_idx, tok_pos=tok_pos,
                       tau=tau, O=O, lse=lse)
