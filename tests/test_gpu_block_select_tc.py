"""The int8 tensor-core block scores and selection of dl_block_select against
the fp64 oracle: the integer digit form of the pooled keys written by
dl_pool_keys and dl_cache_write (checked value by value against its
definition in include/dl.h), the selected blocks exactly equal to the
oracle's on every (b, g) of shapes with ragged tiles, GQA groups, every row
count and sinks, the scores within the kernel's certified relative bound,
near-ties handed to the fp64 recomputation, and the kernel's choice equal to
the fp64 kernel's on the 32K layer shape."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from tests.helpers import check_norm_field, key_digits_np, np_

pytestmark = pytest.mark.gpu

SEED = 20261210


def _desc(batch, H, H_kv, d, L_q, n_units):
    n_pages = n_units
    return dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=n_units * 64, L_q=L_q, page=64,
                        n_pages=n_pages, n_slots=batch * n_pages, dtype=dl.DL_BF16)


def _digits_on(dev, kbar):
    kdig, kexp = key_digits_np(kbar.numpy())
    # [b][g][n][5][d] -> [b][g][5][n][d]
    kdig = np.ascontiguousarray(np.moveaxis(kdig, -2, 2))
    return torch.from_numpy(kdig).to(dev), torch.from_numpy(kexp).to(dev)


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("bf16", 64), ("fp32", 128)])
def test_pool_writes_key_digits(dtype, d, cuda_device):
    wl = synth.workload("llada8k", L_ctx=2000, H=4, H_kv=2, d=d, batch=2, dtype=dtype)
    inp = synth.make_step_inputs(wl, device=cuda_device)
    desc = dl.make_desc(wl.batch, wl.H, wl.H_kv, wl.d, wl.L_ctx, wl.L_q, wl.B, wl.n_pages,
                        wl.n_slots, dl.DL_BF16 if dtype == "bf16" else dl.DL_FP32)
    kbar = torch.empty((wl.batch, wl.H_kv, wl.n_blk, d), dtype=torch.float32, device=cuda_device)
    kdig, kexp = dl.key_digit_buffers(wl.batch, wl.H_kv, wl.n_blk, d, cuda_device)
    dl.dl_pool_keys(desc, inp.k_pool, inp.page_table, wl.n_blk, wl.B, 0, wl.B, kbar,
                    Kdig=kdig, Kexp=kexp)
    assert dl.dl_get_status() == dl.DL_OK
    ref_dig, ref_exp = key_digits_np(kbar.cpu().numpy())
    assert np.array_equal(kdig.cpu().numpy(), np.moveaxis(ref_dig, -2, 2))
    assert np.array_equal(kexp.cpu().numpy() & 0xFFFF, ref_exp)
    check_norm_field(kexp.cpu().numpy(), inp.k_pool.cpu(), inp.page_table.cpu(), wl.L_ctx,
                     wl.B)


def test_digits_reconstruct_within_their_bound():
    """The digit form itself (host definition): x~ = V 2^(E-161) differs from
    x by less than one unit, and exactly where no set bit was cut."""
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 128)) * np.exp2(rng.integers(-30, 4, (64, 128)))).astype(
        np.float32)
    x[3] = 0.0
    x[5, :7] = -0.0
    kdig, kexp = key_digits_np(x)
    E = kexp & 255
    V = (kdig[:, 0].astype(np.int64) << 28) + sum(
        kdig[:, t].astype(np.int64) << (7 * (4 - t)) for t in range(1, 5))
    assert (kdig[:, 1:] >= 0).all()
    xt = V * np.exp2(E[:, None] - 161.0)
    unit = np.exp2(E[:, None] - 161.0)
    err = np.abs(x.astype(np.float64) - xt)
    assert (err < unit).all()
    assert ((err > 0).sum(axis=1) <= (kexp >> 8)).all()


CASES = [  # n_units, H, H_kv, L_q, cnts (predicted rows per sequence), topK, n_sinks
    (512, 4, 4, 32, [20, 15], 128, 4),    # the 32K layer's shape per (b, g)
    (300, 4, 2, 32, [12, 10], 40, 2),     # ragged third tile, G = 2, 24 rows
    (128, 2, 2, 20, [20, 1], 30, 1),      # one tile, one row
    (200, 8, 2, 32, [6, 3], 10, 0),       # G = 4, 24 rows, no sinks
    (512, 2, 2, 32, [0, 12], 64, 3),      # a sequence with no predicted rows
    (385, 3, 3, 16, [16, 9], 300, 2),     # four tiles, the last with one key; topK near n
    (256, 2, 2, 32, [8, 8], 16, 1),       # one row block (8 rows)
]


@pytest.mark.parametrize("n_units,H,H_kv,L_q,cnts,topK,n_sinks", CASES)
def test_block_select_tc_matches_oracle(n_units, H, H_kv, L_q, cnts, topK, n_sinks, cuda_device):
    batch, d = len(cnts), 128
    G = H // H_kv
    max_q = max(cnts)
    assert G * max_q <= 24  # the int8 kernel's row bound
    sid = 31000 + n_units + 7 * H + L_q
    q = synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d).to(
        torch.bfloat16)
    kbar = (synth.normals(SEED, sid + 1, 0, batch * H_kv * n_units * d) / 8).to(
        torch.float32).reshape(batch, H_kv, n_units, d)
    q_idx = torch.full((batch, L_q), -1, dtype=torch.int32)
    for b, c in enumerate(cnts):
        keys = synth.uniforms(SEED, sid + 2 + b, 0, L_q)
        q_idx[b, :c] = torch.sort(torch.argsort(keys)[:c]).values.to(torch.int32)
    q_cnt = torch.tensor(cnts, dtype=torch.int32)
    sinks = None
    if n_sinks:
        u = synth.uniforms(SEED, sid + 9, 0, batch * n_sinks)
        sinks = (u * n_units * 64).to(torch.int32).reshape(batch, n_sinks)
    kdig, kexp = _digits_on(cuda_device, kbar)
    desc = _desc(batch, H, H_kv, d, L_q, n_units)
    n_s = 0 if sinks is None else n_sinks
    max_sel = min(topK, n_units) + n_s
    dev = lambda t: None if t is None else t.to(cuda_device)  # noqa: E731
    score = torch.full((batch, H_kv, n_units), float("nan"), dtype=torch.float64,
                       device=cuda_device)
    blk = torch.empty((batch, H_kv, max_sel), dtype=torch.int32, device=cuda_device)
    cnt = torch.empty((batch, H_kv), dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    dl.dl_read_counters()
    dl.dl_block_select(desc, dev(q), dev(q_idx), dev(q_cnt), dev(kbar), n_units, 64, topK,
                       dev(sinks), score, blk, cnt, ws, max_q=max_q, Kdig=kdig, Kexp=kexp)
    assert dl.dl_get_status() == dl.DL_OK
    fast, fallback = dl.dl_read_counters()
    assert fast + fallback == batch * H_kv
    _check_against_oracle(q, kbar, q_idx, cnts, sinks, n_sinks, topK, H_kv, G, d, score, blk,
                          cnt)


def _check_against_oracle(q, kbar, q_idx, cnts, sinks, n_sinks, topK, H_kv, G, d, score, blk,
                          cnt):
    got_s, got_b, got_c = np_(score), np_(blk), np_(cnt)
    scale = oracle.scale_for(d)
    for b, c in enumerate(cnts):
        for g in range(H_kv):
            rows = [q[b, g * G + j, int(q_idx[b, i])] for j in range(G) for i in range(c)]
            Q_rows = torch.stack(rows) if rows else torch.zeros(0, d, dtype=torch.bfloat16)
            ref = oracle.block_scores(Q_rows, kbar[b, g], scale)
            np.testing.assert_allclose(got_s[b, g], ref, rtol=1e-9, atol=1e-300)
            sp = [] if sinks is None else [int(p) for p in sinks[b]]
            sel = oracle.select_blocks(ref, sp, 64, topK)
            assert got_c[b, g] == len(sel), (b, g)
            assert got_b[b, g, :len(sel)].tolist() == list(sel), (b, g)
            assert (got_b[b, g, len(sel):] == -1).all()


def test_more_than_24_rows_take_the_fp64_kernel(cuda_device):
    """25 .. 32 rows per group: the fused fp64 kernel (the int8 kernel holds at
    most three row blocks), same results."""
    n_units, H, H_kv, L_q, cnts, topK, n_sinks = 300, 8, 2, 32, [8, 7], 40, 2
    batch, d, G = 2, 128, 4
    sid = 31500
    q = synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d).to(
        torch.bfloat16)
    kbar = (synth.normals(SEED, sid + 1, 0, batch * H_kv * n_units * d) / 8).to(
        torch.float32).reshape(batch, H_kv, n_units, d)
    q_idx = torch.full((batch, L_q), -1, dtype=torch.int32)
    for b, c in enumerate(cnts):
        keys = synth.uniforms(SEED, sid + 2 + b, 0, L_q)
        q_idx[b, :c] = torch.sort(torch.argsort(keys)[:c]).values.to(torch.int32)
    q_cnt = torch.tensor(cnts, dtype=torch.int32)
    u = synth.uniforms(SEED, sid + 9, 0, batch * n_sinks)
    sinks = (u * n_units * 64).to(torch.int32).reshape(batch, n_sinks)
    kdig, kexp = _digits_on(cuda_device, kbar)
    desc = _desc(batch, H, H_kv, d, L_q, n_units)
    dev = lambda t: t.to(cuda_device)  # noqa: E731
    score = torch.empty((batch, H_kv, n_units), dtype=torch.float64, device=cuda_device)
    blk = torch.empty((batch, H_kv, topK + n_sinks), dtype=torch.int32, device=cuda_device)
    cnt = torch.empty((batch, H_kv), dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    dl.dl_read_counters()
    dl.dl_block_select(desc, dev(q), dev(q_idx), dev(q_cnt), dev(kbar), n_units, 64, topK,
                       dev(sinks), score, blk, cnt, ws, max_q=8, Kdig=kdig, Kexp=kexp)
    assert dl.dl_get_status() == dl.DL_OK
    assert dl.dl_read_counters() == (0, 0)
    _check_against_oracle(q, kbar, q_idx, cnts, sinks, n_sinks, topK, H_kv, G, d, score, blk,
                          cnt)


def test_near_ties_fall_back_to_fp64(cuda_device):
    """Blocks with identical pooled keys score exactly alike; at the cut that
    leaves no certified gap, so the CTA recomputes in fp64 and keeps the lower
    indices, as the oracle does."""
    batch, H, H_kv, L_q, d, n_units, topK = 1, 2, 2, 32, 128, 256, 20
    q = synth.normals(SEED, 32000, 0, batch * H * L_q * d).reshape(batch, H, L_q, d).to(
        torch.bfloat16)
    base = (synth.normals(SEED, 32001, 0, n_units * d) / 8).to(torch.float32).reshape(n_units, d)
    kbar = base.repeat(batch, H_kv, 1, 1).contiguous()
    q_idx = torch.arange(L_q, dtype=torch.int32)[None].repeat(batch, 1).contiguous()
    q_cnt = torch.full((batch,), 16, dtype=torch.int32)
    # 41 identical keys (7 and 100..139), pushed towards the mean query so that
    # they rank first and the tie straddles the cut of 20
    for g in range(H_kv):
        qm = q[0, g, :16].float().mean(0)
        tied = (kbar[0, g, 7] + 0.5 * qm / qm.norm()).to(torch.float32)
        for j in [7] + list(range(100, 140)):
            kbar[:, g, j] = tied
    kdig, kexp = _digits_on(cuda_device, kbar)
    desc = _desc(batch, H, H_kv, d, L_q, n_units)
    score = torch.empty((batch, H_kv, n_units), dtype=torch.float64, device=cuda_device)
    blk = torch.empty((batch, H_kv, topK), dtype=torch.int32, device=cuda_device)
    cnt = torch.empty((batch, H_kv), dtype=torch.int32, device=cuda_device)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    dl.dl_read_counters()
    dl.dl_block_select(desc, q.to(cuda_device), q_idx.to(cuda_device), q_cnt.to(cuda_device),
                       kbar.to(cuda_device), n_units, 64, topK, None, score, blk, cnt, ws,
                       max_q=16, Kdig=kdig, Kexp=kexp)
    assert dl.dl_get_status() == dl.DL_OK
    fast, fallback = dl.dl_read_counters()
    assert fallback == batch * H_kv and fast == 0
    scale = oracle.scale_for(d)
    for g in range(H_kv):
        ref = oracle.block_scores(q[0, g, :16], kbar[0, g], scale)
        sel = oracle.select_blocks(ref, [], 64, topK)
        assert np_(blk)[0, g].tolist() == list(sel)
        assert sel.tolist() == [7] + list(range(100, 119))


def test_int8_and_fp64_kernels_choose_alike(cuda_device, kernel_flags):
    """One sparse layer of the 32K step's shape (batch 2, 32 KV heads, 512
    blocks, predicted rows): both kernels of dl_block_select, same blocks."""
    wl = synth.workload("llada32k_step", batch=2, n_layers=3)
    layer = wl.first_sparse_layer
    q = synth.make_q_dec(wl, layer, cuda_device)
    pt = synth.page_permutation(wl).to(cuda_device)
    kp, _ = synth.make_layer_kv(wl, layer, q, cuda_device, pt.cpu())
    confs, masks = zip(*(synth.confidence(wl, b) for b in range(wl.batch)))
    conf, masked = torch.stack(confs).to(cuda_device), torch.stack(masks).to(cuda_device)
    desc = dl.make_desc(wl.batch, wl.H, wl.H_kv, wl.d, wl.L_ctx, wl.L_q, wl.B, wl.n_pages,
                        wl.n_slots, dl.DL_BF16)
    q_idx = torch.empty((wl.batch, wl.L_q), dtype=torch.int32, device=cuda_device)
    q_cnt = torch.empty((wl.batch,), dtype=torch.int32, device=cuda_device)
    dl.dl_predict_queries(conf, masked, wl.k, wl.w, q_idx, q_cnt)
    kbar = torch.empty((wl.batch, wl.H_kv, wl.n_blk, wl.d), dtype=torch.float32, device=cuda_device)
    kdig, kexp = dl.key_digit_buffers(wl.batch, wl.H_kv, wl.n_blk, wl.d, cuda_device)
    dl.dl_pool_keys(desc, kp, pt, wl.n_blk, wl.B, 0, wl.B, kbar, Kdig=kdig, Kexp=kexp)
    sinks = torch.tensor([synth.sink_positions(wl, b) for b in range(wl.batch)],
                         dtype=torch.int32, device=cuda_device)
    ws = torch.empty(dl.dl_workspace_size(desc), dtype=torch.uint8, device=cuda_device)
    max_sel = wl.topK + sinks.shape[1]
    out = []
    for flags in (0, dl.DL_FLAG_SCORE_FP64):
        kernel_flags(flags)
        score = torch.empty((wl.batch, wl.H_kv, wl.n_blk), dtype=torch.float64, device=cuda_device)
        blk = torch.empty((wl.batch, wl.H_kv, max_sel), dtype=torch.int32, device=cuda_device)
        cnt = torch.empty((wl.batch, wl.H_kv), dtype=torch.int32, device=cuda_device)
        dl.dl_read_counters()
        dl.dl_block_select(desc, q, q_idx, q_cnt, kbar, wl.n_blk, wl.B, wl.topK, sinks, score, blk,
                           cnt, ws, max_q=wl.k * (2 * wl.w + 1), Kdig=kdig, Kexp=kexp)
        assert dl.dl_get_status() == dl.DL_OK
        counts = dl.dl_read_counters()
        out.append((np_(score), np_(blk), np_(cnt), counts))
    (s_tc, b_tc, c_tc, n_tc), (s_64, b_64, c_64, n_64) = out
    assert n_tc[0] + n_tc[1] == wl.batch * wl.H_kv and n_64 == (0, 0)
    assert np.array_equal(b_tc, b_64) and np.array_equal(c_tc, c_64)
    np.testing.assert_allclose(s_tc, s_64, rtol=1e-9, atol=0)


def test_cache_write_updates_key_digits(cuda_device):
    batch, H_kv, d, page, L_ctx, n_new = 2, 2, 128, 64, 640, 40
    n_pages = L_ctx // page
    n_slots = batch * n_pages
    shape = (n_slots, H_kv, page, d)
    kp = synth.normals(SEED, 33000, 0, int(np.prod(shape))).reshape(shape).to(torch.bfloat16)
    kn = synth.normals(SEED, 33001, 0, batch * H_kv * n_new * d).reshape(
        batch, H_kv, n_new, d).to(torch.bfloat16)
    page_table = torch.arange(n_slots, dtype=torch.int32).reshape(batch, n_pages)
    desc = dl.make_desc(batch=batch, H=H_kv, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=32, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    K_dev, V_dev = kp.to(cuda_device), kp.to(cuda_device).clone()
    kbar = torch.empty((batch, H_kv, n_pages, d), dtype=torch.float32, device=cuda_device)
    kdig, kexp = dl.key_digit_buffers(batch, H_kv, n_pages, d, cuda_device)
    pt = page_table.to(cuda_device)
    dl.dl_pool_keys(desc, K_dev, pt, n_pages, page, 0, page, kbar, Kdig=kdig, Kexp=kexp)
    before = kdig.cpu().numpy().copy()
    start = torch.tensor([100, 600], dtype=torch.int32, device=cuda_device)
    dl.dl_cache_write(desc, kn.to(cuda_device), kn.to(cuda_device), start, pt, K_dev, V_dev,
                      kbar, Kdig=kdig, Kexp=kexp)
    assert dl.dl_get_status() == dl.DL_OK
    ref_dig, ref_exp = key_digits_np(kbar.cpu().numpy())
    assert np.array_equal(kdig.cpu().numpy(), np.moveaxis(ref_dig, -2, 2))
    assert np.array_equal(kexp.cpu().numpy() & 0xFFFF, ref_exp)
    check_norm_field(kexp.cpu().numpy(), K_dev.cpu(), page_table, L_ctx, page)
    # the cache write's words equal a fresh pooling of the updated pool's
    kbar2 = torch.empty_like(kbar)
    kdig2, kexp2 = dl.key_digit_buffers(batch, H_kv, n_pages, d, cuda_device)
    dl.dl_pool_keys(desc, K_dev, pt, n_pages, page, 0, page, kbar2, Kdig=kdig2, Kexp=kexp2)
    assert torch.equal(kexp2, kexp)
    after = kdig.cpu().numpy()
    touched = {0: {1, 2}, 1: {9}}
    for b in range(batch):
        for j in range(n_pages):
            if j not in touched[b]:
                assert np.array_equal(after[b, :, :, j], before[b, :, :, j]), (b, j)
