"""Host-side sequencing of the library's entry points into one layer of a
denoising step, the chunked-prefix step, and the multi-layer step.

Focus-dLLM (research.elamur.ai summary): the queries are predicted once per
step from the previous step's confidence; shallow layers attend densely; the
first sparse layer finds the attention sinks, which every deeper layer reuses
unchanged (abstract: sink locations reused across layers); each sparse layer
scores blocks with the predicted queries, keeps the top-K plus the sinks and
attends over them.  Prefilling-dLLM (abstract): chunk selection, then token
selection inside the kept chunks, then attention over the gathered tokens.

This module only allocates torch tensors for outputs and workspaces and calls
the C ABI (`_abi`) in order on one stream; all arithmetic runs in the
library's kernels.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

from . import _abi as A


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


def workspace(desc: A.dl_attn_desc, device) -> torch.Tensor:
    n = A.dl_workspace_size(desc)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


@dataclasses.dataclass
class LayerOutputs:
    q_idx: Optional[torch.Tensor]
    q_cnt: Optional[torch.Tensor]
    Kbar: Optional[torch.Tensor]
    score: Optional[torch.Tensor]
    sink_pos: Optional[torch.Tensor]
    blk_idx: Optional[torch.Tensor]
    blk_cnt: Optional[torch.Tensor]
    O: torch.Tensor
    lse: torch.Tensor


def layer_step(desc: A.dl_attn_desc, q_dec, k_pool, v_pool, page_table, k_dec, v_dec, *,
               topK: int, conf_prev=None, still_masked=None, k: int = 4, w: int = 2,
               q_idx=None, q_cnt=None, sink_pos=None, detect_sinks: int = 0,
               dense: bool = False, Kbar=None, Kdig=None, Kexp=None, ws=None, stream=None,
               fused_select: bool = True) -> LayerOutputs:
    """One layer for a batch: (predict,) pool, (find sinks,) score and select
    (one call, or dl_block_scores then dl_select when fused_select is False),
    attend -- or dense attention.  Mirrors the oracle's layer_step.  When the
    layer pools its own keys it also writes their integer digits (Kdig, Kexp),
    which the selection then reads; a caller passing Kbar may pass them too."""
    dev = q_dec.device
    B, L_q, d, H, H_kv = desc.batch, desc.L_q, desc.d, desc.H, desc.H_kv
    n_blk = -(-desc.L_ctx // desc.page)
    if ws is None:
        ws = workspace(desc, dev)
    if q_idx is None and conf_prev is not None:
        q_idx = _empty((B, L_q), torch.int32, dev)
        q_cnt = _empty((B,), torch.int32, dev)
        A.dl_predict_queries(conf_prev, still_masked, k, w, q_idx, q_cnt, stream)
    O = _empty((B, L_q, H, d), q_dec.dtype, dev)
    lse = _empty((B, H, L_q), torch.float32, dev)
    if dense:
        A.dl_sparse_attn(desc, q_dec, k_pool, v_pool, page_table, None, None, k_dec, v_dec, O,
                         lse, ws, stream)
        return LayerOutputs(q_idx, q_cnt, None, None, sink_pos, None, None, O, lse)
    if Kbar is None:
        Kbar = _empty((B, H_kv, n_blk, d), torch.float32, dev)
        Kdig, Kexp = A.key_digit_buffers(B, H_kv, n_blk, d, dev)
        A.dl_pool_keys(desc, k_pool, page_table, n_blk, desc.page, 0, desc.page, Kbar, stream,
                       Kdig=Kdig, Kexp=Kexp)
    score = _empty((B, H_kv, n_blk), torch.float64, dev)
    if detect_sinks:
        sink_pos = _empty((B, detect_sinks), torch.int32, dev)
        A.dl_find_sinks(desc, q_dec, q_idx, q_cnt, k_pool, page_table, k_dec, detect_sinks,
                        sink_pos, ws, stream, Kexp=Kexp)
    n_s = 0 if sink_pos is None else sink_pos.shape[-1]
    max_sel = min(topK, n_blk) + n_s
    blk_idx = _empty((B, H_kv, max(max_sel, 1)), torch.int32, dev)
    blk_cnt = _empty((B, H_kv), torch.int32, dev)
    if fused_select:
        # rows per sequence: the prediction gives at most k windows of 2w+1
        max_q = min(L_q, k * (2 * w + 1)) if conf_prev is not None else 0
        A.dl_block_select(desc, q_dec, q_idx, q_cnt, Kbar, n_blk, desc.page, topK, sink_pos,
                          score, blk_idx, blk_cnt, ws, stream, max_q=max_q, Kdig=Kdig, Kexp=Kexp)
    else:
        A.dl_block_scores(desc, q_dec, q_idx, q_cnt, Kbar, n_blk, score, ws, stream)
        A.dl_select(score, desc.page, topK, sink_pos, blk_idx, blk_cnt, stream)
    A.dl_sparse_attn(desc, q_dec, k_pool, v_pool, page_table, blk_idx, blk_cnt, k_dec, v_dec, O,
                     lse, ws, stream)
    return LayerOutputs(q_idx, q_cnt, Kbar, score, sink_pos, blk_idx, blk_cnt, O, lse)


@dataclasses.dataclass
class ChunkOutputs:
    Kbar: torch.Tensor
    score: torch.Tensor
    chunk_idx: torch.Tensor
    chunk_cnt: torch.Tensor
    tok_pos: torch.Tensor
    tok_cnt: torch.Tensor
    O: torch.Tensor
    lse: torch.Tensor


def chunked_step(desc: A.dl_attn_desc, q_dec, k_pool, v_pool, page_table, k_dec, v_dec, *,
                 n_chunks: int, stride: int, content: int, topK_chunks: int, topT: int,
                 Kbar=None, Kexp=None, ws=None, stream=None,
                 certify_tokens: bool = False) -> ChunkOutputs:
    """Chunked-prefix step: chunk keys (BOS excluded), chunk scores from
    every decode query, top-K chunks, top-T tokens per chunk plus its BOS,
    attention over the gathered tokens and the decode block.

    certify_tokens: the top-T cut certified with the chunk keys' exponent
    words (an undecided cut recomputed in fp64 inside the token kernel).  Off
    by default: the bound on the fp32 tensor-core logits is about 1e-3 of the
    masses, wider than the spacing of the masses at the cut of dense chunks,
    so nearly every chunk would take the fp64 recheck (about 20 times the
    step's time on the 32-chunk workload)."""
    dev = q_dec.device
    B, L_q, d, H, H_kv = desc.batch, desc.L_q, desc.d, desc.H, desc.H_kv
    if ws is None:
        ws = workspace(desc, dev)
    if Kbar is None:
        # chunk keys with their exponent words (the token cut is certified with them)
        Kbar = _empty((B, H_kv, n_chunks, d), torch.float32, dev)
        Kdig, Kexp = A.key_digit_buffers(B, H_kv, n_chunks, d, dev)
        A.dl_pool_keys(desc, k_pool, page_table, n_chunks, stride, 1, content, Kbar, stream,
                       Kdig=Kdig, Kexp=Kexp)
    score = _empty((B, H_kv, n_chunks), torch.float64, dev)
    kc = min(topK_chunks, n_chunks)
    chunk_idx = _empty((B, H_kv, kc), torch.int32, dev)
    chunk_cnt = _empty((B, H_kv), torch.int32, dev)
    # chunk scores from every decode row, then the top chunks: one call
    A.dl_block_select(desc, q_dec, None, None, Kbar, n_chunks, stride, kc, None, score, chunk_idx,
                      chunk_cnt, ws, stream)
    tok_pos = _empty((B, H_kv, kc * (topT + 1)), torch.int32, dev)
    tok_cnt = _empty((B, H_kv), torch.int32, dev)
    A.dl_token_select(desc, q_dec, k_pool, page_table, chunk_idx, stride, content, topT, tok_pos,
                      tok_cnt, ws, stream, Kexp=Kexp if certify_tokens else None)
    O = _empty((B, L_q, H, d), q_dec.dtype, dev)
    lse = _empty((B, H, L_q), torch.float32, dev)
    A.dl_sparse_attn_gather(desc, q_dec, k_pool, v_pool, page_table, tok_pos, tok_cnt, k_dec,
                            v_dec, O, lse, ws, stream)
    return ChunkOutputs(Kbar, score, chunk_idx, chunk_cnt, tok_pos, tok_cnt, O, lse)


class DenoiseStep:
    """One denoising step over n_layers layers sharing a page table.

    Per step: predict the queries once; layers below first_sparse attend
    densely; layer first_sparse finds n_sinks sinks and every sparse layer
    selects topK blocks plus those sinks.  Pooled keys are an input (they are
    built when the KV cache is refreshed: `refresh_pooled_keys`).  All output
    buffers are allocated once, so `run` can be captured in a CUDA graph."""

    def __init__(self, desc: A.dl_attn_desc, n_layers: int, first_sparse: int, topK: int,
                 n_sinks: int, k: int, w: int, dtype: torch.dtype, device, sink_group=None):
        self.desc, self.n_layers, self.first_sparse = desc, n_layers, first_sparse
        # head-sharded: desc covers this rank's heads, and the sink mass is
        # summed over sink_group before the sinks are picked (sharded.py)
        self.sink_group = sink_group
        self.topK, self.n_sinks, self.k, self.w = topK, n_sinks, k, w
        B, L_q, d, H, H_kv = desc.batch, desc.L_q, desc.d, desc.H, desc.H_kv
        self.n_blk = -(-desc.L_ctx // desc.page)
        self.max_sel = min(topK, self.n_blk) + n_sinks
        self.max_q = min(L_q, k * (2 * w + 1))  # predicted rows per sequence, at most
        self.device = device
        self.ws = workspace(desc, device)
        self.q_idx = _empty((B, L_q), torch.int32, device)
        self.q_cnt = _empty((B,), torch.int32, device)
        self.sink_pos = _empty((B, n_sinks), torch.int32, device)
        self.mass = _empty((B, desc.L_ctx), torch.float32, device) if sink_group is not None else None
        self.score = _empty((B, H_kv, self.n_blk), torch.float64, device)
        self.blk_idx = [_empty((B, H_kv, self.max_sel), torch.int32, device)
                        for _ in range(n_layers)]
        self.blk_cnt = [_empty((B, H_kv), torch.int32, device) for _ in range(n_layers)]
        self.O = [_empty((B, L_q, H, d), dtype, device) for _ in range(n_layers)]
        self.lse = [_empty((B, H, L_q), torch.float32, device) for _ in range(n_layers)]

    def key_cache(self):
        """Pooled keys of one layer with their integer digits: (Kbar, Kdig,
        Kexp), to be filled by refresh_pooled_keys / commit_block."""
        dsc = self.desc
        Kbar = _empty((dsc.batch, dsc.H_kv, self.n_blk, dsc.d), torch.float32, self.device)
        return (Kbar, *A.key_digit_buffers(dsc.batch, dsc.H_kv, self.n_blk, dsc.d, self.device))

    def refresh_pooled_keys(self, layer: int, k_pool, page_table, kc, stream=None):
        """Pooled keys (and digits) of a whole layer, for a cache whose K rows
        were all rewritten (built or recomputed).  kc = key_cache()."""
        d = self.desc
        A.dl_pool_keys(d, k_pool, page_table, self.n_blk, d.page, 0, d.page, kc[0], stream,
                       Kdig=kc[1], Kexp=kc[2])

    def commit_block(self, k_new, v_new, start, k_pool, v_pool, page_table, kc, stream=None):
        """A finished decode block joins one layer's cached context at
        positions start[b] ..: written into the pools, the touched blocks'
        pooled keys (and digits) recomputed in the same pass (dl_cache_write)."""
        A.dl_cache_write(self.desc, k_new, v_new, start, page_table, k_pool, v_pool, kc[0], stream,
                         Kdig=kc[1], Kexp=kc[2])

    def run(self, conf_prev, still_masked, q_dec: List, k_pool: List, v_pool: List,
            page_table, k_dec: List, v_dec: List, key_caches: List, stream=None,
            attn_events: Optional[list] = None, find_sinks: bool = True):
        """Launches the step on `stream`.  key_caches[l] = (Kbar, Kdig, Kexp)
        of layer l (key_cache()).  find_sinks=False keeps the sinks found by
        an earlier step (sink_pos): the later steps of one decode block reuse
        the sinks of its first step, until the block is committed to the
        cache.  If attn_events is a list, a pair of timing events (recorded as
        graph nodes when captured) brackets every attention call and
        (layer, start, end) is appended to it."""
        d = self.desc
        A.dl_predict_queries(conf_prev, still_masked, self.k, self.w, self.q_idx, self.q_cnt,
                             stream)
        for l in range(self.n_layers):
            if l < self.first_sparse:
                ev = self._begin(attn_events, stream)
                A.dl_sparse_attn(d, q_dec[l], k_pool[l], v_pool[l], page_table, None, None,
                                 k_dec[l], v_dec[l], self.O[l], self.lse[l], self.ws, stream)
                self._end(attn_events, ev, l, stream)
                continue
            if l == self.first_sparse and find_sinks:
                self._find_sinks(q_dec[l], k_pool[l], page_table, k_dec[l], key_caches[l][2],
                                 stream)
            Kbar, Kdig, Kexp = key_caches[l]
            A.dl_block_select(d, q_dec[l], self.q_idx, self.q_cnt, Kbar, self.n_blk, d.page,
                              self.topK, self.sink_pos, self.score, self.blk_idx[l],
                              self.blk_cnt[l], self.ws, stream, max_q=self.max_q, Kdig=Kdig,
                              Kexp=Kexp)
            ev = self._begin(attn_events, stream)
            A.dl_sparse_attn(d, q_dec[l], k_pool[l], v_pool[l], page_table, self.blk_idx[l],
                             self.blk_cnt[l], k_dec[l], v_dec[l], self.O[l], self.lse[l],
                             self.ws, stream)
            self._end(attn_events, ev, l, stream)

    def _find_sinks(self, q_dec, k_pool, page_table, k_dec, Kexp, stream):
        d = self.desc
        if self.sink_group is None:
            A.dl_find_sinks(d, q_dec, self.q_idx, self.q_cnt, k_pool, page_table, k_dec,
                            self.n_sinks, self.sink_pos, self.ws, stream, Kexp=Kexp)
            return
        from .sharded import reduce_and_pick
        A.dl_sink_mass(d, q_dec, self.q_idx, self.q_cnt, k_pool, page_table, k_dec, self.mass,
                       self.ws, stream)
        reduce_and_pick(self.mass, self.sink_pos, self.sink_group, stream=stream)

    @staticmethod
    def _begin(events, stream):
        if events is None:
            return None
        e = torch.cuda.Event(enable_timing=True, external=True)
        e.record(stream)
        return e

    @staticmethod
    def _end(events, start, layer, stream):
        if events is None:
            return
        e = torch.cuda.Event(enable_timing=True, external=True)
        e.record(stream)
        events.append((layer, start, e))
