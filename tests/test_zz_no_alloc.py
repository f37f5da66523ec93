"""dl_block_scores_noalloc: the block-score entry point for callers that
cannot allocate device memory (a runtime that owns every allocation and has
no workspace to hand out, code where cudaMalloc may not run because it can
synchronise the device, a process whose footprint is fixed after start-up).
Its scratch is the library's built-in array instead of a caller workspace.

Checked through the C ABI on two calls in a row with different inputs (so
that contents left in the shared array by the first call cannot leak into
the second), each against the fp64 oracle directly and against
dl_block_scores, within the parity tests' score tolerance (1e-12 relative).
This file is collected last; it passes alone and after the other tests."""
import ctypes

import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from long_context_diffusion_b200 import _abi, pipeline
from tests.helpers import desc_for


def _oracle_scores(wl, inp, Kbar, q_idx, q_cnt):
    """oracle.block_scores on the same pooled keys and predicted rows."""
    q = inp.q_dec.cpu()
    kbar = Kbar.cpu()
    qi, qc = q_idx.cpu(), q_cnt.cpu()
    G, scale = wl.H // wl.H_kv, oracle.scale_for(wl.d)
    ref = np.zeros((wl.batch, wl.H_kv, wl.n_blk))
    for b in range(wl.batch):
        pos = [int(qi[b, i]) for i in range(int(qc[b]))]
        for g in range(wl.H_kv):
            rows = [q[b, g * G + j, p] for j in range(G) for p in pos]
            Q_rows = torch.stack(rows) if rows else torch.zeros(0, wl.d, dtype=q.dtype)
            ref[b, g] = oracle.block_scores(Q_rows, kbar[b, g], scale)
    return ref

pytestmark = pytest.mark.gpu


def _scores_both(wl, dev, q_idx=None, q_cnt=None, via_noalloc=True):
    inp = synth.make_step_inputs(wl, device=dev)
    desc = desc_for(wl)
    Kbar = torch.empty((wl.batch, wl.H_kv, wl.n_blk, wl.d), dtype=torch.float32, device=dev)
    dl.dl_pool_keys(desc, inp.k_pool, inp.page_table, wl.n_blk, wl.B, 0, wl.B, Kbar)
    if q_idx is None:
        q_idx = torch.empty((wl.batch, wl.L_q), dtype=torch.int32, device=dev)
        q_cnt = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
        dl.dl_predict_queries(inp.conf_prev, inp.still_masked, wl.k, wl.w, q_idx, q_cnt)
    ref = torch.empty((wl.batch, wl.H_kv, wl.n_blk), dtype=torch.float64, device=dev)
    ws = pipeline.workspace(desc, dev)
    dl.dl_block_scores(desc, inp.q_dec, q_idx, q_cnt, Kbar, wl.n_blk, ref, ws)
    out = torch.full_like(ref, float("nan"))
    st = _abi.lib.dl_block_scores_noalloc(ctypes.byref(desc), _abi._p(inp.q_dec), _abi._p(q_idx),
                                          _abi._p(q_cnt), _abi._p(Kbar), wl.n_blk,
                                          _abi._p(out), _abi._s(None))
    assert st == dl.DL_OK, _abi.lib.dl_last_error_message()
    assert dl.dl_get_status() == dl.DL_OK
    return out.cpu().numpy(), ref.cpu().numpy(), _oracle_scores(wl, inp, Kbar, q_idx, q_cnt)


def test_noalloc_matches_workspace_entry_point_twice(cuda_device):
    # call 1: GQA, 256 blocks, predicted rows
    wl1 = synth.workload("dream16k")
    out1, ref1, orc1 = _scores_both(wl1, cuda_device)
    np.testing.assert_allclose(out1, orc1, rtol=1e-12, atol=1e-15)
    assert np.allclose(out1, ref1, rtol=1e-12, atol=1e-15)
    # call 2: other shape and every decode row, right after call 1
    wl2 = synth.workload("llada8k", L_ctx=4096, H=8, H_kv=8)
    q_idx = torch.arange(wl2.L_q, dtype=torch.int32, device=cuda_device)[None].contiguous()
    q_cnt = torch.full((1,), wl2.L_q, dtype=torch.int32, device=cuda_device)
    out2, ref2, orc2 = _scores_both(wl2, cuda_device, q_idx, q_cnt)
    np.testing.assert_allclose(out2, orc2, rtol=1e-12, atol=1e-15)
    assert np.allclose(out2, ref2, rtol=1e-12, atol=1e-15)
    assert np.isfinite(out2).all()


def test_noalloc_rejects_oversize(cuda_device):
    wl = synth.workload("llada32k_step", batch=16)
    desc = desc_for(wl)
    fake = ctypes.c_void_p(0x10000)
    st = _abi.lib.dl_block_scores_noalloc(ctypes.byref(desc), fake, fake, fake, fake, wl.n_blk,
                                          fake, None)
    assert st == dl.DL_ERR_WORKSPACE
    assert "32 MiB" in _abi.lib.dl_last_error_message().decode()
