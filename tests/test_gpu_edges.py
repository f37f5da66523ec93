"""GPU parity on edge cases: ragged context with NaN-filled page padding,
GQA groups of 1/4/7, head dim 64/128, decode blocks of 1 and 100 tokens,
degenerate predictions (nothing masked, fewer masked than k, w = 0), K = 0,
K covering every block, permuted page slots, and out-of-range indices
reported through the device error word (tiles skipped, nothing traps)."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from long_context_diffusion_b200 import pipeline
from tests.helpers import check_attention, desc_for, np_

pytestmark = pytest.mark.gpu


def _run(wl, cuda_device, sinks_given=None, dense=False):
    inp = synth.make_step_inputs(wl, device=cuda_device)
    n_s = wl.sinks_given if sinks_given is None else sinks_given
    sinks = inp.sinks_planted[:, :n_s].contiguous() if n_s else None
    desc = desc_for(wl)
    out = pipeline.layer_step(desc, inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table,
                              inp.k_dec, inp.v_dec, topK=wl.topK, k=wl.k, w=wl.w,
                              conf_prev=inp.conf_prev, still_masked=inp.still_masked,
                              sink_pos=sinks, dense=dense)
    assert dl.dl_get_status() == dl.DL_OK, dl._abi.lib.dl_last_error_message()
    ref = oracle.layer_step(inp.q_dec.cpu(), inp.k_pool.cpu(), inp.v_pool.cpu(),
                            inp.page_table.cpu(), inp.k_dec.cpu(), inp.v_dec.cpu(), wl.L_ctx,
                            wl.B, wl.topK, conf_prev=inp.conf_prev.cpu(),
                            still_masked=inp.still_masked.cpu(), k=wl.k, w=wl.w,
                            sink_pos=None if sinks is None else sinks.cpu(), dense=dense)
    assert np.array_equal(np_(out.q_idx), ref.q_idx)
    assert np.array_equal(np_(out.q_cnt), ref.q_cnt)
    if not dense:
        assert np.array_equal(np_(out.Kbar), ref.Kbar)
        assert np.allclose(np_(out.score), ref.score, rtol=1e-12, atol=1e-15)
        assert np.array_equal(np_(out.blk_idx), ref.blk_idx)
        assert np.array_equal(np_(out.blk_cnt), ref.blk_cnt)
    check_attention(out.O, out.lse, ref.O, ref.lse, wl.dtype == "fp32", wl.name)
    return inp, out, ref


BASE = synth.workload("dream16k")

CASES = {
    "ragged_nan_gqa7_d64": dict(L_ctx=1000, d=64, L_q=20, topK=5, batch=2, nan_padding=True),
    "gqa4_d128_lq100": dict(H=16, H_kv=4, L_ctx=2048, L_q=100, topK=8, batch=1),
    "mha_lq1": dict(H=4, H_kv=4, L_ctx=777, L_q=1, topK=3, batch=3, n_unmasked=0),
    "nothing_masked": dict(H=8, H_kv=8, L_ctx=1024, topK=4, batch=2, n_unmasked=32),
    "fewer_masked_than_k": dict(H=8, H_kv=2, L_ctx=1024, topK=4, batch=2, n_unmasked=30),
    "w0_k1": dict(H=8, H_kv=8, L_ctx=2048, topK=6, batch=1, k=1, w=0),
    "wide_window": dict(H=8, H_kv=8, L_ctx=2048, topK=6, batch=1, w=40),
    "topk0_sinks_only": dict(H=8, H_kv=8, L_ctx=2048, topK=0, batch=2),
    "topk_covers_all": dict(H=8, H_kv=4, L_ctx=1500, topK=100, batch=1),
    "fp32_gqa4_d128": dict(dtype="fp32", H=8, H_kv=2, L_ctx=1111, topK=4, batch=1,
                           scale_qkv=0.125),
    "fp32_lq64_d64": dict(dtype="fp32", H=4, H_kv=4, d=64, L_ctx=640, L_q=64, topK=2, batch=2,
                          scale_qkv=0.125),
    # key-major tensor-core path (head dim 128, <= 32 rows per KV group):
    # ragged NaN-padded last page, rows < 32, odd and even page counts
    "km_ragged_nan_lq20": dict(H=8, H_kv=8, L_ctx=1000, L_q=20, topK=5, batch=2,
                               nan_padding=True),
    "km_gqa2_lq16_odd": dict(H=8, H_kv=4, L_ctx=2047, L_q=16, topK=6, batch=3,
                             nan_padding=True),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_edge_case(case, cuda_device):
    wl = BASE.replace(name=case, wid=40 + sorted(CASES).index(case), **CASES[case])
    _run(wl, cuda_device)


@pytest.mark.parametrize("L_ctx,L_q,H_kv", [(1500, 24, 8), (4096, 16, 4), (70, 9, 2)])
def test_dense_layer_ragged(L_ctx, L_q, H_kv, cuda_device):
    wl = BASE.replace(name=f"dense{L_ctx}", wid=63, H=8, H_kv=H_kv, L_ctx=L_ctx, L_q=L_q,
                      batch=2, nan_padding=True)
    _run(wl, cuda_device, dense=True)


def test_no_sinks_given(cuda_device):
    wl = BASE.replace(name="nosinks", wid=60, H=8, H_kv=8, L_ctx=2048, topK=5, batch=1)
    _run(wl, cuda_device, sinks_given=0)


def test_page_permutation_invariance(cuda_device):
    wl = BASE.replace(name="perm", wid=61, H=8, H_kv=2, L_ctx=3000, topK=7, batch=2)
    _, out_a, _ = _run(wl, cuda_device)
    _, out_b, _ = _run(wl.replace(permute_pages=True), cuda_device)
    assert torch.equal(out_a.blk_idx, out_b.blk_idx)
    assert torch.equal(out_a.O, out_b.O) and torch.equal(out_a.lse, out_b.lse)


def test_bad_indices_are_reported_not_trapped(cuda_device):
    wl = BASE.replace(name="bad", wid=62, H=4, H_kv=4, L_ctx=1024, topK=4, batch=1)
    inp = synth.make_step_inputs(wl, device=cuda_device)
    desc = desc_for(wl)
    ws = pipeline.workspace(desc, cuda_device)
    O = torch.empty((1, wl.L_q, wl.H, wl.d), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.empty((1, wl.H, wl.L_q), dtype=torch.float32, device=cuda_device)
    blk = torch.tensor([[[0, 3, 16, 5]] * wl.H_kv], dtype=torch.int32, device=cuda_device)
    cnt = torch.full((1, wl.H_kv), 4, dtype=torch.int32, device=cuda_device)
    dl.dl_sparse_attn(desc, inp.q_dec, inp.k_pool, inp.v_pool, inp.page_table, blk, cnt,
                      inp.k_dec, inp.v_dec, O, lse, ws)
    assert dl.dl_get_status() == dl.DL_ERR_BAD_INDEX
    assert torch.isfinite(O.float()).all()
    assert dl.dl_get_status() == dl.DL_OK            # the word is cleared by the read
    bad_pt = inp.page_table.clone()
    bad_pt[0, 2] = wl.n_slots + 5
    blk2 = torch.tensor([[[0, 2, 3, 5]] * wl.H_kv], dtype=torch.int32, device=cuda_device)
    dl.dl_sparse_attn(desc, inp.q_dec, inp.k_pool, inp.v_pool, bad_pt, blk2, cnt, inp.k_dec,
                      inp.v_dec, O, lse, ws)
    assert dl.dl_get_status() == dl.DL_ERR_BAD_INDEX
    assert torch.isfinite(O.float()).all()
