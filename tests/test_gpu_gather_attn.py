"""GPU parity of attention over gathered cached tokens (the chunked-prefix
path's attention) called directly through the C ABI, against the oracle's
attention over the same explicit positions: every row configuration of the
tensor-core kernel (32 rows in four replicas, 64 in two, 96 in one M-tile,
160 in two), head dim 64 and 128, ragged per-(b, g) token counts (empty,
one token, not a multiple of 64, several tiles), permuted pages; and the
same cases through the CUDA-core kernel."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from oracle import steps as S
from tests.helpers import check_attention, np_

pytestmark = pytest.mark.gpu

SEED = 20261203


@pytest.mark.parametrize("H,H_kv,L_q,d,cnts", [
    (4, 4, 64, 128, [[2056, 1000, 64, 1], [300, 65, 0, 2056]]),   # 64 rows
    (8, 4, 16, 128, [[200, 0, 129, 63]]),                           # 32 rows
    (6, 2, 32, 128, [[700, 1]]),                                    # 96 rows
    (8, 1, 20, 128, [[513], [40]]),                                 # 160 rows
    (4, 4, 32, 64, [[777, 64, 5, 128]]),                            # head dim 64
    # 32 KV heads: several tiles per CTA, partial last tiles followed by the
    # decode tile inside one CTA's run
    (32, 32, 64, 128, [[2056] * 16 + [1000, 1, 0, 65] * 4]),
])
@pytest.mark.parametrize("simt", [False, True])
def test_gather_attention_matches_oracle(H, H_kv, L_q, d, cnts, simt, cuda_device, kernel_flags):
    if simt:
        kernel_flags(dl.DL_FLAG_GATHER_SIMT)
    batch, page, L_ctx = len(cnts), 64, 4096
    n_pages = L_ctx // page
    n_slots = batch * n_pages
    max_tok = max(max(c) for c in cnts)
    sid = 13000 + H * 100 + L_q + d
    q = synth.normals(SEED, sid, 0, batch * H * L_q * d).reshape(batch, H, L_q, d).to(
        torch.bfloat16)
    kp = synth.normals(SEED, sid + 1, 0, n_slots * H_kv * page * d).reshape(
        n_slots, H_kv, page, d).to(torch.bfloat16)
    vp = synth.normals(SEED, sid + 2, 0, n_slots * H_kv * page * d).reshape(
        n_slots, H_kv, page, d).to(torch.bfloat16)
    kd = synth.normals(SEED, sid + 3, 0, batch * H_kv * L_q * d).reshape(
        batch, H_kv, L_q, d).to(torch.bfloat16)
    vd = synth.normals(SEED, sid + 4, 0, batch * H_kv * L_q * d).reshape(
        batch, H_kv, L_q, d).to(torch.bfloat16)
    perm = torch.argsort(synth.uniforms(SEED, sid + 5, 0, n_slots)).to(torch.int32)
    page_table = perm.reshape(batch, n_pages)
    tok_pos = torch.full((batch, H_kv, max_tok), -1, dtype=torch.int32)
    positions = []
    for b in range(batch):
        row = []
        for g in range(H_kv):
            c = cnts[b][g]
            keys = synth.uniforms(SEED, sid + 10 + b * H_kv + g, 0, L_ctx)
            pos = torch.sort(torch.argsort(keys)[:c]).values.to(torch.int32)
            tok_pos[b, g, :c] = pos
            row.append(pos.numpy().astype(np.int64))
        positions.append(row)
    tok_cnt = torch.tensor(cnts, dtype=torch.int32)
    desc = dl.make_desc(batch=batch, H=H, H_kv=H_kv, d=d, L_ctx=L_ctx, L_q=L_q, page=page,
                        n_pages=n_pages, n_slots=n_slots, dtype=dl.DL_BF16)
    ws = torch.empty(dl.dl_workspace_size(desc), dtype=torch.uint8, device=cuda_device)
    O = torch.full((batch, L_q, H, d), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    lse = torch.full((batch, H, L_q), float("nan"), dtype=torch.float32, device=cuda_device)
    dev = lambda x: x.to(cuda_device)  # noqa: E731
    dl.dl_sparse_attn_gather(desc, dev(q), dev(kp), dev(vp), dev(page_table), dev(tok_pos),
                             dev(tok_cnt), dev(kd), dev(vd), O, lse, ws)
    torch.cuda.synchronize()
    assert dl.dl_get_status() == dl.DL_OK
    scale = oracle.scale_for(d)
    pt = np.asarray(page_table, dtype=np.int64)
    for b in range(batch):
        O_ref, lse_ref = S.chunk_attention(q[b], kp, vp, pt[b], positions[b], page, kd[b], vd[b],
                                           scale)
        check_attention(O[b], lse[b], O_ref, lse_ref, False, f"b={b}")
