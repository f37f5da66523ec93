"""GPU parity at the benchmark's full size: layers of the 32K step (batch 4,
32 query / 32 KV heads, d 128, 32K context, top-128 blocks of 64 tokens),
through the same C-ABI calls and sizes the benchmark's DenoiseStep launches,
checked against the oracle on sampled sequences and KV heads computed one by
one (the whole layer in fp64 would take minutes on the host)."""
import numpy as np
import pytest

import long_context_diffusion_b200 as dl
import synth
from long_context_diffusion_b200 import pipeline
from oracle import steps as S
from oracle.step import predict_all
from tests.helpers import BF16_LSE_ABS, BF16_MAX_ABS, BF16_MEAN_ABS, desc_for, np_

pytestmark = pytest.mark.gpu

SAMPLE_B = (0, 3)
SAMPLE_G = (0, 13, 31)


def _logical(pool, page_table, b, g, L_ctx, B):
    """KV head g of sequence b at logical positions [0, L_ctx), gathered on the
    device through the page table, as fp64 on the host."""
    pages = pool[page_table[b].long(), g]            # [n_pages][B][d]
    return S.f64(pages.reshape(-1, pages.shape[-1])[:L_ctx])


def _check_heads(wl, b, g, Q, Kd, Vd, keys_ctx, vals_ctx, O, lse, errs):
    keys = np.concatenate([keys_ctx, S.f64(Kd[b, g])])
    vals = np.concatenate([vals_ctx, S.f64(Vd[b, g])])
    for h in range(g * wl.G, (g + 1) * wl.G):
        o, l = S.attention_rows(S.f64(Q[b, h]), keys, vals, S.scale_for(wl.d))
        errs.append(np.abs(O[b, :, h] - o).reshape(-1))
        lerr = np.abs(lse[b, h] - l).max()
        assert lerr <= BF16_LSE_ABS, f"(b={b}, h={h}): lse max-abs {lerr:.3g}"


def _check_errs(errs):
    err = np.concatenate(errs)
    assert err.max() <= BF16_MAX_ABS, f"max-abs {err.max():.3g}"
    assert err.mean() <= BF16_MEAN_ABS, f"mean-abs {err.mean():.3g}"


def test_llada32k_first_sparse_layer_sampled(cuda_device):
    """The layer that finds the sinks: predict, pool, sinks, fused
    score+select, key-major sparse attention."""
    wl = synth.workload("llada32k_step")
    inp = synth.make_step_inputs(wl, layer=wl.first_sparse_layer, device=cuda_device)
    out = pipeline.layer_step(desc_for(wl), inp.q_dec, inp.k_pool, inp.v_pool,
                              inp.page_table, inp.k_dec, inp.v_dec, topK=wl.topK, k=wl.k,
                              w=wl.w, conf_prev=inp.conf_prev, still_masked=inp.still_masked,
                              detect_sinks=wl.detect_sinks)
    assert dl.dl_get_status() == dl.DL_OK, dl._abi.lib.dl_last_error_message()
    q_idx, q_cnt = predict_all(inp.conf_prev.cpu(), inp.still_masked.cpu(), wl.k, wl.w)
    assert np.array_equal(np_(out.q_idx), q_idx)
    assert np.array_equal(np_(out.q_cnt), q_cnt)
    scale = S.scale_for(wl.d)
    Q, Kd, Vd = inp.q_dec.cpu(), inp.k_dec.cpu(), inp.v_dec.cpu()
    Kbar, score, blk_idx = np_(out.Kbar), np_(out.score), np_(out.blk_idx)
    blk_cnt, sinks = np_(out.blk_cnt), np_(out.sink_pos)
    O, lse = np_(out.O), np_(out.lse)
    errs = []
    for b in SAMPLE_B:
        rows = q_idx[b, : q_cnt[b]]
        # the sinks of sequence b take every head over the whole context
        Kc = np.stack([_logical(inp.k_pool, inp.page_table, b, g, wl.L_ctx, wl.B)
                       for g in range(wl.H_kv)])
        top, _ = S.find_sinks(Q[b], Kc, Kd[b], rows, wl.detect_sinks, scale)
        assert sinks[b].tolist() == top.tolist(), f"b={b}: sinks"
        for g in SAMPLE_G:
            kb = S.pooled_keys(Kc[g], wl.L_ctx, wl.B)
            assert np.array_equal(Kbar[b, g], kb), f"(b={b}, g={g}): pooled keys"
            Qg = S.f64(Q[b, g * wl.G:(g + 1) * wl.G])[:, rows].reshape(-1, wl.d)
            sc = S.block_scores(Qg, kb, scale)
            assert np.allclose(score[b, g], sc, rtol=1e-12, atol=1e-15), f"(b={b}, g={g})"
            sel = S.select_blocks(sc, top, wl.B, wl.topK)
            assert blk_cnt[b, g] == len(sel), f"(b={b}, g={g}): block count"
            assert np.array_equal(blk_idx[b, g, : len(sel)], sel), f"(b={b}, g={g}): blocks"
            pos = (sel[:, None] * wl.B + np.arange(wl.B)[None, :]).reshape(-1)
            pos = pos[pos < wl.L_ctx]
            Vg = _logical(inp.v_pool, inp.page_table, b, g, wl.L_ctx, wl.B)
            _check_heads(wl, b, g, Q, Kd, Vd, Kc[g][pos], Vg[pos], O, lse, errs)
        del Kc
    _check_errs(errs)


def test_llada32k_dense_layer_sampled(cuda_device):
    """A shallow layer: dense attention over the whole 32K context."""
    wl = synth.workload("llada32k_step")
    inp = synth.make_step_inputs(wl, layer=0, device=cuda_device)
    out = pipeline.layer_step(desc_for(wl), inp.q_dec, inp.k_pool, inp.v_pool,
                              inp.page_table, inp.k_dec, inp.v_dec, topK=wl.topK, dense=True)
    assert dl.dl_get_status() == dl.DL_OK, dl._abi.lib.dl_last_error_message()
    Q, Kd, Vd = inp.q_dec.cpu(), inp.k_dec.cpu(), inp.v_dec.cpu()
    O, lse = np_(out.O), np_(out.lse)
    errs = []
    for b in SAMPLE_B:
        for g in SAMPLE_G:
            Kg = _logical(inp.k_pool, inp.page_table, b, g, wl.L_ctx, wl.B)
            Vg = _logical(inp.v_pool, inp.page_table, b, g, wl.L_ctx, wl.B)
            _check_heads(wl, b, g, Q, Kd, Vd, Kg, Vg, O, lse, errs)
    _check_errs(errs)
