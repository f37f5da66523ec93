"""GPU parity of the cache refresh with fused pooling (dl_cache_write) against
the oracle: writes aligned to a block, straddling two and three blocks, up to
the ragged end of the context, bf16 and fp32 at d 64 and 128 (every compiled
variant), GQA descriptors, permuted pages.  The pools must equal the oracle's
bit for bit; the touched blocks' pooled keys exactly for bf16 (fp64 sums of
the block are exact, rounded once to fp32) and within one fp32 ulp for fp32
keys (an fp64 sum of fp32 values is exact only while their exponents are
close); every other pooled key must be left as it was.  A start out of range,
also one near the int32 limit, is reported and leaves that sequence
untouched."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from tests.helpers import np_

pytestmark = pytest.mark.gpu

SEED = 20261204


@pytest.mark.parametrize("dtype,d,H_kv,G,L_ctx,n_new,starts", [
    ("bf16", 128, 4, 1, 1000, 32, [64, 950]),      # one block half written; the last full block
    ("bf16", 128, 2, 1, 1000, 100, [10, 900]),     # three blocks; up to the ragged end
    ("fp32", 64, 3, 1, 700, 64, [0, 200]),         # one whole block; two halves
    ("bf16", 64, 2, 4, 900, 40, [0, 500, 860]),    # d 64 (two rows per thread), GQA, batch 3
    ("fp32", 128, 2, 7, 1100, 70, [30, 1030, 640, 128]),  # fp32 d 128, G 7, batch 4
])
def test_cache_write_matches_oracle(dtype, d, H_kv, G, L_ctx, n_new, starts, cuda_device):
    batch, page = len(starts), 64
    n_pages = -(-L_ctx // page)
    n_slots = batch * n_pages
    n_blk = n_pages
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    sid = 14000 + d + n_new
    shape = (n_slots, H_kv, page, d)
    kp = synth.normals(SEED, sid, 0, int(np.prod(shape))).reshape(shape).to(tdt)
    vp = synth.normals(SEED, sid + 1, 0, int(np.prod(shape))).reshape(shape).to(tdt)
    kn = synth.normals(SEED, sid + 2, 0, batch * H_kv * n_new * d).reshape(
        batch, H_kv, n_new, d).to(tdt)
    vn = synth.normals(SEED, sid + 3, 0, batch * H_kv * n_new * d).reshape(
        batch, H_kv, n_new, d).to(tdt)
    perm = torch.argsort(synth.uniforms(SEED, sid + 4, 0, n_slots)).to(torch.int32)
    page_table = perm.reshape(batch, n_pages)
    desc = dl.make_desc(batch=batch, H=H_kv * G, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=32, page=page,
                        n_pages=n_pages, n_slots=n_slots,
                        dtype=dl.DL_BF16 if dtype == "bf16" else dl.DL_FP32)
    K_dev, V_dev = kp.to(cuda_device), vp.to(cuda_device)
    kbar = torch.full((batch, H_kv, n_blk, d), -123.0, dtype=torch.float32, device=cuda_device)
    start = torch.tensor(starts, dtype=torch.int32)
    dl.dl_cache_write(desc, kn.to(cuda_device), vn.to(cuda_device), start.to(cuda_device),
                      page_table.to(cuda_device), K_dev, V_dev, kbar)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_OK
    K_got, V_got, kbar_got = np_(K_dev), np_(V_dev), np_(kbar)
    K_ref, V_ref = oracle.steps.f64(kp), oracle.steps.f64(vp)
    touched = {}
    for b in range(batch):
        K_ref, V_ref, kb = oracle.cache_write(K_ref, V_ref, np.asarray(page_table[b]), kn[b], vn[b],
                                              starts[b], L_ctx, page)
        touched[b] = kb
    assert np.array_equal(K_got, K_ref) and np.array_equal(V_got, V_ref)
    for b in range(batch):
        for j in range(n_blk):
            if j in touched[b]:
                ref = np.asarray(touched[b][j], dtype=np.float32)
                got = kbar_got[b, :, j].astype(np.float32)
                if dtype == "bf16":
                    assert np.array_equal(got, ref), (b, j)
                else:  # one fp32 ulp at most
                    ulp = np.abs(np.nextafter(ref, np.float32(np.inf)) - ref)
                    assert (np.abs(got - ref) <= ulp).all(), (b, j)
            else:
                assert (kbar_got[b, :, j] == -123.0).all(), (b, j)


@pytest.mark.parametrize("bad_start", ["past_end", "near_int32_max"])
def test_cache_write_start_out_of_range_is_reported(bad_start, cuda_device):
    batch, H_kv, d, page, L_ctx, n_new = 2, 2, 128, 64, 512, 32
    n_pages = L_ctx // page
    n_slots = batch * n_pages
    shape = (n_slots, H_kv, page, d)
    kp = synth.normals(SEED, 14900, 0, int(np.prod(shape))).reshape(shape).to(torch.bfloat16)
    kn = synth.normals(SEED, 14901, 0, batch * H_kv * n_new * d).reshape(
        batch, H_kv, n_new, d).to(torch.bfloat16)
    page_table = torch.arange(n_slots, dtype=torch.int32).reshape(batch, n_pages)
    desc = dl.make_desc(batch=batch, H=H_kv, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=32, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    K_dev, V_dev = kp.to(cuda_device), kp.to(cuda_device).clone()
    kbar = torch.zeros((batch, H_kv, n_pages, d), dtype=torch.float32, device=cuda_device)
    st0 = L_ctx - n_new + 1 if bad_start == "past_end" else 2**31 - 8
    start = torch.tensor([st0, 0], dtype=torch.int32, device=cuda_device)
    dl.dl_cache_write(desc, kn.to(cuda_device), kn.to(cuda_device), start,
                      page_table.to(cuda_device), K_dev, V_dev, kbar)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_ERR_BAD_INDEX
    got = np_(K_dev)
    assert np.array_equal(got[:n_pages], np_(kp)[:n_pages])      # sequence 0 untouched
    assert np.array_equal(got[n_pages, :, :n_new], np_(kn)[1])    # sequence 1 written
