"""GPU parity of intra-chunk token selection (the chunked-prefix path) called
directly through the C ABI: chunks of 1024 content tokens (eight key tiles
and the token past them), ragged chunks, one and two query heads per KV
group, 16 to 64 query rows, T from 0 to the whole chunk, and a chunk stride
off the page grid (the CUDA-core kernel).  Every page-aligned case also runs
through the CUDA-core kernel.  With the chunk keys' exponent words the
tensor-core kernel's cut is certified and the kept tokens must equal the
oracle's exactly; otherwise (fp32 cut) they must equal them wherever the
oracle's cut has a margin above the fp32 error of the masses, and be within
that error of the cut elsewhere."""

import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from oracle import steps as S
from tests.helpers import cut_margin, np_

pytestmark = pytest.mark.gpu

SEED = 20261202


def _chunk_exps(desc, kp, page_table, n_chunks, stride, content, dev):
    """Exponent words (with the norm bounds) of the chunk keys: each chunk's
    content tokens pooled, the BOS left out."""
    batch, H_kv, d = desc.batch, desc.H_kv, desc.d
    kbar = torch.empty((batch, H_kv, n_chunks, d), dtype=torch.float32, device=dev)
    kdig, kexp = dl.key_digit_buffers(batch, H_kv, n_chunks, d, dev)
    dl.dl_pool_keys(desc, kp.to(dev), page_table.to(dev), n_chunks, stride, 1, content, kbar,
                    Kdig=kdig, Kexp=kexp)
    return kexp


@pytest.mark.parametrize("content,stride,H,H_kv,L_q,topT,n_sel", [
    (1024, 1088, 4, 4, 64, 256, 2),   # the benchmark's chunk shape: 64 rows
    (1000, 1024, 4, 2, 16, 100, 2),   # G = 2, 32 rows, ragged last tile
    (200, 256, 2, 2, 20, 0, 1),       # T = 0: the BOS only
    (200, 256, 2, 2, 20, 200, 3),     # T = the whole chunk
    (64, 128, 3, 3, 48, 1, 2),        # one tile, 48 rows
    (300, 301, 2, 2, 32, 37, 2),      # stride off the page grid
])
@pytest.mark.parametrize("simt,certified", [(False, True), (False, False), (True, False)])
def test_token_select_matches_oracle(content, stride, H, H_kv, L_q, topT, n_sel, simt, certified,
                                     cuda_device, kernel_flags):
    if simt:
        kernel_flags(dl.DL_FLAG_TOKEN_SIMT)
    batch, d, page, n_chunks = 2, 128, 64, 3
    G = H // H_kv
    L_ctx = n_chunks * stride
    n_pages = -(-L_ctx // page)
    n_slots = batch * n_pages
    sid = 12000 + content + 7 * L_q + topT
    q = (synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d)).to(
        torch.bfloat16)
    kp = (synth.normals(SEED, sid + 1, 0, n_slots * H_kv * page * d).reshape(
        n_slots, H_kv, page, d)).to(torch.bfloat16)
    perm = torch.argsort(synth.uniforms(SEED, sid + 2, 0, n_slots)).to(torch.int32)
    page_table = perm.reshape(batch, n_pages)
    sel_keys = synth.uniforms(SEED, sid + 3, 0, batch * H_kv * n_chunks).reshape(
        batch * H_kv, n_chunks)
    chunk_idx = torch.sort(torch.argsort(sel_keys, dim=1)[:, :n_sel], dim=1).values.to(
        torch.int32).reshape(batch, H_kv, n_sel)
    desc = dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=L_q, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    per = topT + 1
    tok_pos = torch.full((batch, H_kv, n_sel * per), -7, dtype=torch.int32, device=cuda_device)
    tok_cnt = torch.full((batch, H_kv), -7, dtype=torch.int32, device=cuda_device)
    Kexp = _chunk_exps(desc, kp, page_table, n_chunks, stride, content, cuda_device) \
        if certified else None
    dl.dl_token_select(desc, q.to(cuda_device), kp.to(cuda_device), page_table.to(cuda_device),
                       chunk_idx.to(cuda_device), stride, content, topT, tok_pos, tok_cnt, ws,
                       Kexp=Kexp)
    torch.cuda.synchronize()
    exact = certified and stride % page == 0  # the tensor-core kernel takes page-aligned chunks
    assert dl.dl_get_status() == dl.DL_OK
    got, cnt = np_(tok_pos), np_(tok_cnt)
    assert (cnt == n_sel * per).all()
    scale = oracle.scale_for(d)
    Q, K = S.f64(q), S.f64(kp)
    pt = np.asarray(page_table, dtype=np.int64)
    for b in range(batch):
        for g in range(H_kv):
            rows = Q[b, g * G:(g + 1) * G].reshape(-1, d)
            for j in range(n_sel):
                c = int(chunk_idx[b, g, j])
                base = c * stride
                keys = S.gather_context(K, pt[b], g, base + 1 + np.arange(content), page)
                off, tau = S.token_select(rows, keys, topT, scale)
                out = got[b, g, j * per:(j + 1) * per]
                assert out[0] == base, (b, g, j)
                kept = out[1:]
                assert (kept[len(off):] == -1).all() if topT else True
                mine = kept[: len(off)] - base - 1
                assert np.all(np.diff(mine) > 0), (b, g, j)
                tol = 1e-5 * tau.max()
                if exact:
                    assert mine.tolist() == off.tolist(), (b, g, j)
                elif cut_margin(tau, off) > tol:
                    assert mine.tolist() == off.tolist(), (b, g, j)
                else:
                    assert (tau[mine] >= np.sort(tau)[-topT] - tol).all(), (b, g, j)


@pytest.mark.parametrize("exact_tie", [False, True])
def test_token_select_near_tie_at_the_cut(exact_tie, cuda_device):
    """Two content tokens of one chunk built to have (nearly or exactly) the
    same mass and to straddle the top-T cut: token a's key is raised so that
    it ranks T-th, token b is a copy of it (a tie: the lower position is
    kept), or the copy with one value moved by a bf16 ulp (masses apart by
    less than the certification bound, so the fp64 recheck decides).  The
    certified cut equals the oracle's."""
    batch, H, H_kv, d, L_q, page = 1, 2, 2, 128, 32, 64
    content, stride, n_chunks, topT = 1024, 1088, 2, 64
    L_ctx = n_chunks * stride
    n_pages = -(-L_ctx // page)
    n_slots = batch * n_pages
    q = synth.normals(SEED, 12990, 0, batch * H * L_q * d).reshape(batch, H, L_q, d).to(
        torch.bfloat16)
    kp = synth.normals(SEED, 12991, 0, n_slots * H_kv * page * d).reshape(
        n_slots, H_kv, page, d).to(torch.bfloat16)
    page_table = torch.arange(n_slots, dtype=torch.int32).reshape(batch, n_pages)
    chunk_idx = torch.tensor([[[1], [1]]], dtype=torch.int32)
    base = 1 * stride
    desc = dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=L_q, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    scale = oracle.scale_for(d)
    bpos = 900  # content offsets (positions base + 1 + offset)
    pt0 = page_table[0].numpy()

    def taus(g):
        keys = S.gather_context(S.f64(kp), pt0, g, base + 1 + np.arange(content), page)
        return S.token_select(S.f64(q[0, g]), keys, topT, scale)[1]

    def row(off, g):
        pos = base + 1 + off
        return (int(page_table[0, pos // page]), g, pos % page)

    chosen_a = []
    for g in range(H_kv):
        qbar = q[0, g].to(torch.float32).mean(dim=0)
        rb = row(bpos, g)
        for a in range(100, 120):  # a token whose boosted copy lands exactly on the cut
            ra = row(a, g)
            orig_a, orig_b = kp[ra].clone(), kp[rb].clone()

            def put(boost):
                kp[ra] = (orig_a.to(torch.float32) + boost * qbar).to(torch.bfloat16)
                kp[rb] = kp[ra]

            lo, hi = 0.0, 20.0  # smallest boost with a among the top T (both keys raised)
            for _ in range(30):
                mid = (lo + hi) / 2
                put(mid)
                rank_a = int((np.argsort(-taus(g), kind="stable") == a).nonzero()[0][0])
                if rank_a <= topT - 1:
                    hi = mid
                else:
                    lo = mid
            put(hi)
            order = np.argsort(-taus(g), kind="stable")
            if order[topT - 1] == a and order[topT] == bpos:
                chosen_a.append(a)
                break
            kp[ra], kp[rb] = orig_a, orig_b
        else:
            pytest.fail("no token could be placed on the cut")
        if not exact_tie:
            rw = kp[rb].clone()
            rw[7] = (rw[7].view(torch.int16) + 1).view(torch.bfloat16)
            kp[rb] = rw
    dev = cuda_device
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=dev)
    per = topT + 1
    tok_pos = torch.full((batch, H_kv, per), -7, dtype=torch.int32, device=dev)
    tok_cnt = torch.full((batch, H_kv), -7, dtype=torch.int32, device=dev)
    Kexp = _chunk_exps(desc, kp, page_table, n_chunks, stride, content, dev)
    dl.dl_token_select(desc, q.to(dev), kp.to(dev), page_table.to(dev), chunk_idx.to(dev),
                       stride, content, topT, tok_pos, tok_cnt, ws, Kexp=Kexp)
    assert dl.dl_get_status() == dl.DL_OK
    got = np_(tok_pos)
    for g in range(H_kv):
        a = chosen_a[g]
        keys = S.gather_context(S.f64(kp), pt0, g, base + 1 + np.arange(content), page)
        off, tau = S.token_select(S.f64(q[0, g]), keys, topT, scale)
        order = np.argsort(-tau, kind="stable")
        assert set(order[topT - 1:topT + 1].tolist()) == {a, bpos}, g  # straddling the cut
        gap = abs(tau[a] - tau[bpos]) / tau[a]
        assert (0.0 < gap < 1e-3) if not exact_tie else gap == 0.0
        mine = got[0, g, 1:] - base - 1
        assert mine.tolist() == off.tolist(), g


@pytest.mark.parametrize("certified", [False, True])
def test_token_select_more_items_than_sms_with_bad_chunks(certified, cuda_device):
    """192 (b, g, chunk) items: the persistent kernel gives some CTAs two of
    them.  Three chunk indices are bad (-1 twice, one chunk past the context),
    one of them a CTA's second item and one a CTA's first: those items are
    written as -1 and reported (DL_ERR_BAD_INDEX); every other item equals
    the oracle's selection."""
    batch, H, H_kv, L_q, d, page = 2, 16, 16, 32, 128, 64
    content, stride, n_chunks, topT, n_sel = 256, 320, 8, 40, 6
    L_ctx = n_chunks * stride
    n_pages = L_ctx // page
    n_slots = batch * n_pages
    sid = 12900
    q = (synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d)).to(
        torch.bfloat16)
    kp = (synth.normals(SEED, sid + 1, 0, n_slots * H_kv * page * d).reshape(
        n_slots, H_kv, page, d)).to(torch.bfloat16)
    perm = torch.argsort(synth.uniforms(SEED, sid + 2, 0, n_slots)).to(torch.int32)
    page_table = perm.reshape(batch, n_pages)
    sel_keys = synth.uniforms(SEED, sid + 3, 0, batch * H_kv * n_chunks).reshape(
        batch * H_kv, n_chunks)
    chunk_idx = torch.sort(torch.argsort(sel_keys, dim=1)[:, :n_sel], dim=1).values.to(
        torch.int32).reshape(batch, H_kv, n_sel)
    # items are (b * H_kv + g) * n_sel + sel; with 148 CTAs, CTA c takes c and c + 148
    bad = {(0, 3, 2): -1,          # item 20: CTA 20, first of two
           (1, 9, 0): -1,          # item 150: CTA 2, second of two
           (1, 7, 0): n_chunks}    # item 138: a chunk past the context
    for (b, g, j), v in bad.items():
        chunk_idx[b, g, j] = v
    desc = dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=L_q, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    ws = torch.empty(max(dl.dl_workspace_size(desc), 256), dtype=torch.uint8, device=cuda_device)
    per = topT + 1
    tok_pos = torch.full((batch, H_kv, n_sel * per), -7, dtype=torch.int32, device=cuda_device)
    tok_cnt = torch.full((batch, H_kv), -7, dtype=torch.int32, device=cuda_device)
    Kexp = _chunk_exps(desc, kp, page_table, n_chunks, stride, content, cuda_device) \
        if certified else None
    dl.dl_token_select(desc, q.to(cuda_device), kp.to(cuda_device), page_table.to(cuda_device),
                       chunk_idx.to(cuda_device), stride, content, topT, tok_pos, tok_cnt, ws,
                       Kexp=Kexp)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_ERR_BAD_INDEX
    got = np_(tok_pos)
    assert (np_(tok_cnt) == n_sel * per).all()
    scale = oracle.scale_for(d)
    Q, K = S.f64(q), S.f64(kp)
    pt = np.asarray(page_table, dtype=np.int64)
    for b in range(batch):
        for g in range(H_kv):
            rows = Q[b, g].reshape(-1, d)
            for j in range(n_sel):
                out = got[b, g, j * per:(j + 1) * per]
                if (b, g, j) in bad:
                    assert (out == -1).all(), (b, g, j)
                    continue
                c = int(chunk_idx[b, g, j])
                base = c * stride
                keys = S.gather_context(K, pt[b], g, base + 1 + np.arange(content), page)
                off, tau = S.token_select(rows, keys, topT, scale)
                assert out[0] == base, (b, g, j)
                mine = out[1:1 + len(off)] - base - 1
                tol = 1e-5 * tau.max()
                if certified or cut_margin(tau, off) > tol:
                    assert mine.tolist() == off.tolist(), (b, g, j)
                else:
                    assert (tau[mine] >= np.sort(tau)[-topT] - tol).all(), (b, g, j)
