"""GPU parity of block scores (a3) and top-K selection (a5) called directly
through the C ABI, at unit counts that span several 128-unit score tiles
with a ragged tail, query-row counts that need several 32-row passes, and
selection sizes that reach each of the selection kernels (one key per
thread up to 1024 units, the shared-memory network up to 4096, the rank
count beyond), with tied scores and duplicate sinks; the fused score +
select call on each of its kernels (fp64 MMA for up to 32 rows, the wide
CUDA-core kernel for more rows over at most 128 units, the separate kernels
beyond)."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from tests.helpers import np_

pytestmark = pytest.mark.gpu

SEED = 20260520


def _desc(batch, H, H_kv, d, L_q, n_units, dtype):
    return dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=n_units * 64, L_q=L_q, page=64,
                        n_pages=n_units, n_slots=batch * n_units,
                        dtype=dl.DL_BF16 if dtype == "bf16" else dl.DL_FP32)


@pytest.mark.parametrize("n_units,H,H_kv,d,L_q,cnts,dtype", [
    (1, 4, 4, 128, 32, [32, 7], "bf16"),
    (129, 8, 2, 128, 32, [20, 32], "bf16"),
    (300, 4, 1, 64, 16, [16, 3], "bf16"),
    (513, 8, 8, 128, 32, [0, 19], "bf16"),
    (1100, 4, 2, 128, 40, [40, 1], "fp32"),
])
def test_block_scores_tiles_and_passes(n_units, H, H_kv, d, L_q, cnts, dtype, cuda_device):
    batch = len(cnts)
    G = H // H_kv
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sid = 9000 + n_units
    q = synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d)
    q = (q * 0.7).to(tdt)
    kbar = synth.normals(SEED, sid + 1, 0, batch * H_kv * n_units * d)
    kbar = (kbar * 0.5).to(torch.float32).reshape(batch, H_kv, n_units, d)
    # predicted query rows: a seeded subset of positions, ascending, cnt each
    q_idx = torch.full((batch, L_q), -1, dtype=torch.int32)
    for b, c in enumerate(cnts):
        keys = synth.uniforms(SEED, sid + 2 + b, 0, L_q)
        q_idx[b, :c] = torch.sort(torch.argsort(keys)[:c]).values.to(torch.int32)
    q_cnt = torch.tensor(cnts, dtype=torch.int32)
    desc = _desc(batch, H, H_kv, d, L_q, n_units, dtype)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    score = torch.full((batch, H_kv, n_units), float("nan"), dtype=torch.float64,
                       device=cuda_device)
    dl.dl_block_scores(desc, q.to(cuda_device), q_idx.to(cuda_device), q_cnt.to(cuda_device),
                       kbar.to(cuda_device), n_units, score, ws)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_OK
    got = np_(score)
    scale = oracle.scale_for(d)
    for b, c in enumerate(cnts):
        for g in range(H_kv):
            rows = [q[b, g * G + j, int(q_idx[b, i])] for j in range(G) for i in range(c)]
            Q_rows = torch.stack(rows) if rows else torch.zeros(0, d, dtype=tdt)
            ref = oracle.block_scores(Q_rows, kbar[b, g], scale)
            np.testing.assert_allclose(got[b, g], ref, rtol=1e-12, atol=1e-15)


def _scores_with_ties(n_units, n_bg, sid):
    u = synth.uniforms(SEED, sid, 0, n_bg * n_units).reshape(n_bg, n_units)
    # a third of the units take one of four shared values: many exact ties
    tie = synth.uniforms(SEED, sid + 1, 0, n_bg * n_units).reshape(n_bg, n_units) < 1 / 3
    level = torch.floor(u * 4) / 4 + 0.125
    return torch.where(tie, level, u)


@pytest.mark.parametrize("n_units,topK", [
    (5, 2), (31, 40), (32, 0), (33, 8), (512, 128), (1000, 64), (1024, 1023),
    (1025, 100), (3000, 128), (4097, 300), (5000, 128),
])
def test_select_all_paths(n_units, topK, cuda_device):
    batch, H_kv, unit_size, n_sinks = 2, 3, 64, 5
    score = _scores_with_ties(n_units, batch * H_kv, 7000 + n_units)
    sp = synth.uniforms(SEED, 7500 + n_units, 0, batch * n_sinks).reshape(batch, n_sinks)
    sink_pos = (sp * n_units * unit_size).to(torch.int64).clamp(max=n_units * unit_size - 1)
    sink_pos[0, 1] = sink_pos[0, 0]           # duplicate position
    sink_pos[1, 2] = -1                       # unused slot
    sink_pos[1, 3] = (sink_pos[1, 4] // unit_size) * unit_size + 1  # same block
    sink_pos = sink_pos.to(torch.int32)
    max_sel = min(topK, n_units) + n_sinks
    blk_idx = torch.full((batch, H_kv, max_sel), -7, dtype=torch.int32, device=cuda_device)
    blk_cnt = torch.full((batch, H_kv), -7, dtype=torch.int32, device=cuda_device)
    dl.dl_select(score.reshape(batch, H_kv, n_units).to(cuda_device), unit_size, topK,
                 sink_pos.to(cuda_device), blk_idx, blk_cnt)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_OK
    got_idx, got_cnt = np_(blk_idx), np_(blk_cnt)
    for b in range(batch):
        for g in range(H_kv):
            ref = oracle.select_blocks(score[b * H_kv + g], sink_pos[b], unit_size, topK)
            assert got_cnt[b, g] == len(ref)
            assert np.array_equal(got_idx[b, g, :len(ref)], ref)
            assert (got_idx[b, g, len(ref):] == -1).all()


@pytest.mark.parametrize("n_units,H,H_kv,d,L_q,cnts,topK,dtype", [
    (1, 4, 4, 128, 32, [32, 7], 4, "bf16"),           # one key
    (129, 8, 8, 128, 32, [20, 32], 16, "bf16"),       # two chunks, ragged
    (300, 4, 2, 64, 16, [16, 3], 40, "bf16"),         # G = 2, d 64, three chunks
    (512, 8, 8, 128, 32, [0, 19], 128, "bf16"),       # four full chunks, a sequence with no rows
    (200, 4, 4, 128, 32, [32, 5], 300, "fp32"),       # fp32 queries, topK beyond the candidates
    (513, 4, 4, 128, 32, [20, 9], 64, "bf16"),        # separate kernels: more than 512 keys
    (100, 8, 2, 128, 32, [20, 32], 10, "bf16"),       # separate kernels: 4 x 32 rows
    (32, 8, 8, 128, 64, [64, 13], 8, "bf16"),         # wide kernel: few units, 64 rows
    (128, 8, 4, 64, 40, [40, 1], 20, "fp32"),         # separate: 80 rows x 128 units > 8192
    (7, 4, 2, 128, 48, [48, 0], 3, "bf16"),           # wide: 96 rows over 7 units, a sequence with none
    (20, 8, 1, 128, 32, [32, 11], 5, "fp32"),         # wide: 256 rows (G = 8), fp32, d 128
    (128, 4, 4, 128, 64, [64, 64], 30, "bf16"),       # wide: 64 rows x 128 units = 8192
    (33, 6, 2, 64, 40, [40, 23], 33, "bf16"),         # wide: ragged units, topK = all, d 64
])
@pytest.mark.parametrize("tight", [False, True])
def test_block_select_matches_oracle(n_units, H, H_kv, d, L_q, cnts, topK, dtype, tight,
                                     cuda_device):
    """dl_block_select (fused score + select) against the oracle, and against
    dl_block_scores followed by dl_select; with max_q = L_q (0) and with the
    tightest bound max(q_cnt) (fewer MMA row tiles)."""
    batch, n_sinks, unit = len(cnts), 3, 64
    G = H // H_kv
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sid = 9500 + n_units + 7 * G
    q = (synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d) * 0.7).to(tdt)
    kbar = (synth.normals(SEED, sid + 1, 0, batch * H_kv * n_units * d) * 0.5).to(
        torch.float32).reshape(batch, H_kv, n_units, d)
    q_idx = torch.full((batch, L_q), -1, dtype=torch.int32)
    for b, c in enumerate(cnts):
        keys = synth.uniforms(SEED, sid + 2 + b, 0, L_q)
        q_idx[b, :c] = torch.sort(torch.argsort(keys)[:c]).values.to(torch.int32)
    q_cnt = torch.tensor(cnts, dtype=torch.int32)
    sp = synth.uniforms(SEED, sid + 9, 0, batch * n_sinks).reshape(batch, n_sinks)
    sink_pos = (sp * n_units * unit).to(torch.int64).clamp(max=n_units * unit - 1)
    sink_pos[0, 1] = sink_pos[0, 0]
    sink_pos = sink_pos.to(torch.int32)
    desc = _desc(batch, H, H_kv, d, L_q, n_units, dtype)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    max_sel = min(topK, n_units) + n_sinks
    dev = lambda x: x.to(cuda_device)  # noqa: E731
    outs = []
    for fused in (True, False):
        score = torch.full((batch, H_kv, n_units), float("nan"), dtype=torch.float64,
                           device=cuda_device)
        blk = torch.full((batch, H_kv, max_sel), -7, dtype=torch.int32, device=cuda_device)
        cnt = torch.full((batch, H_kv), -7, dtype=torch.int32, device=cuda_device)
        if fused:
            dl.dl_block_select(desc, dev(q), dev(q_idx), dev(q_cnt), dev(kbar), n_units, unit,
                               topK, dev(sink_pos), score, blk, cnt, ws,
                               max_q=max(max(cnts), 1) if tight else 0)
        else:
            dl.dl_block_scores(desc, dev(q), dev(q_idx), dev(q_cnt), dev(kbar), n_units, score,
                               ws)
            dl.dl_select(score, unit, topK, dev(sink_pos), blk, cnt)
        torch.cuda.synchronize()
        assert dl.dl_get_status() == dl.DL_OK
        outs.append((np_(score), np_(blk), np_(cnt)))
    (s_f, b_f, c_f), (s_s, b_s, c_s) = outs
    np.testing.assert_allclose(s_f, s_s, rtol=1e-13, atol=1e-16)
    assert np.array_equal(b_f, b_s) and np.array_equal(c_f, c_s)
    scale = oracle.scale_for(d)
    for b, c in enumerate(cnts):
        for g in range(H_kv):
            rows = [q[b, g * G + j, int(q_idx[b, i])] for j in range(G) for i in range(c)]
            Q_rows = torch.stack(rows) if rows else torch.zeros(0, d, dtype=tdt)
            ref = oracle.block_scores(Q_rows, kbar[b, g], scale)
            np.testing.assert_allclose(s_f[b, g], ref, rtol=1e-12, atol=1e-15)
            sel = oracle.select_blocks(ref, sink_pos[b], unit, topK)
            assert c_f[b, g] == len(sel)
            assert np.array_equal(b_f[b, g, :len(sel)], sel)
            assert (b_f[b, g, len(sel):] == -1).all()


def test_block_select_rows_past_the_bound_are_reported(cuda_device):
    """A sequence with more predicted rows than max_q: reported through the
    device error word (its rows are cut to the bound), nothing traps."""
    batch, H, H_kv, d, L_q, n_units, unit = 2, 8, 8, 128, 32, 256, 64
    q = (synth.normals(SEED, 9900, 0, batch * H * L_q * d).reshape(batch, H, L_q, d) * 0.7).to(
        torch.bfloat16)
    kbar = (synth.normals(SEED, 9901, 0, batch * H_kv * n_units * d) * 0.5).to(
        torch.float32).reshape(batch, H_kv, n_units, d)
    q_idx = torch.arange(L_q, dtype=torch.int32).repeat(batch, 1)
    q_cnt = torch.tensor([12, 20], dtype=torch.int32)
    desc = _desc(batch, H, H_kv, d, L_q, n_units, "bf16")
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    score = torch.empty((batch, H_kv, n_units), dtype=torch.float64, device=cuda_device)
    blk = torch.empty((batch, H_kv, 8), dtype=torch.int32, device=cuda_device)
    cnt = torch.empty((batch, H_kv), dtype=torch.int32, device=cuda_device)
    dl.dl_block_select(desc, q.to(cuda_device), q_idx.to(cuda_device), q_cnt.to(cuda_device),
                       kbar.to(cuda_device), n_units, unit, 8, None, score, blk, cnt, ws,
                       max_q=16)
    assert dl.dl_get_status() == dl.DL_ERR_BAD_INDEX
    assert torch.isfinite(score).all()
    assert dl.dl_get_status() == dl.DL_OK
