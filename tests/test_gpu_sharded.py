"""GPU parity for the split sink search and for sinks kept across the steps
of a decode block.

Head shards run here one after the other on one GPU: each shard's heads are
copied into tensors of their own (as a rank of a head-sharded run holds
them), dl_sink_mass computes that shard's part of the mass, the parts are
summed (the all-reduce of a multi-GPU run) and dl_sink_topn picks the sinks.
No kernel waits on another."""
import numpy as np
import pytest
import torch

import long_context_diffusion_b200 as dl
import oracle
import synth
from long_context_diffusion_b200 import pipeline, sharded
from oracle import steps as S
from tests.helpers import check_attention, cut_margin, desc_for, np_

pytestmark = pytest.mark.gpu


def _predicted(wl, inp, dev):
    q_idx = torch.empty((wl.batch, wl.L_q), dtype=torch.int32, device=dev)
    q_cnt = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
    dl.dl_predict_queries(inp.conf_prev, inp.still_masked, wl.k, wl.w, q_idx, q_cnt)
    return q_idx, q_cnt


def _oracle_mass(wl, inp, q_idx, q_cnt, n, g0=0, g1=None):
    g1 = wl.H_kv if g1 is None else g1
    G = wl.G
    qi, qc = np_(q_idx), np_(q_cnt)
    tops, masses = [], []
    for b in range(wl.batch):
        Kc = np.stack([S.gather_context(np_(inp.k_pool), np_(inp.page_table)[b], g,
                                        np.arange(wl.L_ctx), wl.B) for g in range(g0, g1)])
        top, mass = S.find_sinks(np_(inp.q_dec)[b, g0 * G:g1 * G], Kc,
                                 np_(inp.k_dec)[b, g0:g1], qi[b, : qc[b]], n,
                                 S.scale_for(wl.d))
        tops.append(top)
        masses.append(mass)
    return np.stack(tops), np.stack(masses)


@pytest.mark.parametrize("name,world", [("llada8k", 2), ("llada8k", 3), ("dream16k", 2),
                                        ("tiny", 4)])
def test_shard_masses_sum_to_the_sinks(name, world, cuda_device):
    wl = synth.workload(name)
    inp = synth.make_step_inputs(wl, device=cuda_device)
    desc = desc_for(wl)
    q_idx, q_cnt = _predicted(wl, inp, cuda_device)
    n = 4
    total = torch.zeros((wl.batch, wl.L_ctx), dtype=torch.float32, device=cuda_device)
    for r in range(world):
        sh = sharded.HeadShard.of(desc, r, world)
        h0, h1 = sh.heads
        q = inp.q_dec[:, h0:h1].contiguous()
        kp = inp.k_pool[:, sh.g0:sh.g1].contiguous()
        kd = inp.k_dec[:, sh.g0:sh.g1].contiguous()
        mass = torch.full((wl.batch, wl.L_ctx), float("nan"), dtype=torch.float32,
                          device=cuda_device)
        ws = pipeline.workspace(sh.desc, cuda_device)
        dl.dl_sink_mass(sh.desc, q, q_idx, q_cnt, kp, inp.page_table, kd, mass, ws)
        assert dl.dl_get_status() == dl.DL_OK
        _, want = _oracle_mass(wl, inp, q_idx, q_cnt, n, sh.g0, sh.g1)
        got = np_(mass)
        # fp32 sums of exponentials: relative to the largest column mass
        assert np.abs(got - want).max() <= 1e-5 * want.max(), f"shard {r}"
        total += mass
    sinks = torch.empty((wl.batch, n), dtype=torch.int32, device=cuda_device)
    dl.dl_sink_topn(total, sinks)
    top, mass = _oracle_mass(wl, inp, q_idx, q_cnt, n)
    for b in range(wl.batch):
        if cut_margin(mass[b], top[b]) > 1e-5 * mass[b].max():
            assert np_(sinks)[b].tolist() == top[b].tolist()
    if wl.G == 1 and inp.sinks_planted.shape[-1] == n:
        assert np_(sinks).tolist() == np_(inp.sinks_planted).tolist()


@pytest.mark.parametrize("n", [4, 12])
def test_split_calls_equal_find_sinks(n, cuda_device):
    """One shard of every head: dl_sink_mass then dl_sink_topn give exactly
    what dl_find_sinks without exponent words gives (the same kernels), and
    both top-n kernels leave the mass as it is."""
    wl = synth.workload("llada8k")
    inp = synth.make_step_inputs(wl, device=cuda_device)
    desc = desc_for(wl)
    q_idx, q_cnt = _predicted(wl, inp, cuda_device)
    ws = pipeline.workspace(desc, cuda_device)
    ref = torch.empty((wl.batch, n), dtype=torch.int32, device=cuda_device)
    dl.dl_find_sinks(desc, inp.q_dec, q_idx, q_cnt, inp.k_pool, inp.page_table, inp.k_dec, n,
                     ref, ws)
    mass = torch.empty((wl.batch, wl.L_ctx), dtype=torch.float32, device=cuda_device)
    dl.dl_sink_mass(desc, inp.q_dec, q_idx, q_cnt, inp.k_pool, inp.page_table, inp.k_dec, mass,
                    ws)
    before = mass.clone()
    sinks = torch.empty_like(ref)
    dl.dl_sink_topn(mass, sinks)
    assert dl.dl_get_status() == dl.DL_OK
    assert torch.equal(sinks, ref)
    assert torch.equal(mass, before)


def test_sink_group_of_one_rank_takes_the_split_path(cuda_device):
    """DenoiseStep with a sink group runs dl_sink_mass, the reduction (none
    for a group of one rank) and dl_sink_topn; the sinks and every output
    equal those of the unsharded step."""
    import os
    import socket

    import torch.distributed as dist
    wl = synth.workload("llada32k_step", batch=2, L_ctx=4096, n_layers=3, topK=16)
    desc = desc_for(wl)
    layers = [synth.make_step_inputs(wl, layer=l, device=cuda_device) for l in range(3)]
    x0 = layers[0]
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    group_owner = not dist.is_initialized()
    if group_owner:
        dist.init_process_group("gloo", store=store, rank=0, world_size=1)
    try:
        outs = []
        for grp in (None, dist.group.WORLD):
            step = pipeline.DenoiseStep(desc, 3, wl.first_sparse_layer, wl.topK, wl.detect_sinks,
                                        wl.k, wl.w, torch.bfloat16, cuda_device, sink_group=grp)
            kcs = [step.key_cache() for _ in range(3)]
            for l in range(3):
                step.refresh_pooled_keys(l, layers[l].k_pool, layers[l].page_table, kcs[l])
            step.run(x0.conf_prev, x0.still_masked, [x.q_dec for x in layers],
                     [x.k_pool for x in layers], [x.v_pool for x in layers], x0.page_table,
                     [x.k_dec for x in layers], [x.v_dec for x in layers], kcs)
            torch.cuda.synchronize()
            assert dl.dl_get_status() == dl.DL_OK
            outs.append(step)
        a, b = outs
        assert b.mass is not None and a.mass is None
        assert torch.equal(a.sink_pos, b.sink_pos)
        assert np_(a.sink_pos).tolist() == np_(x0.sinks_planted).tolist()
        for l in range(3):
            if l >= wl.first_sparse_layer:  # dense layers select nothing
                assert torch.equal(a.blk_idx[l], b.blk_idx[l])
            assert torch.equal(a.O[l], b.O[l])
    finally:
        if group_owner:
            dist.destroy_process_group()


def test_decode_block_keeps_the_first_steps_sinks(cuda_device):
    """Two steps of one decode block (reading: sinks found at the first step
    are kept until the block is committed): the second step runs with
    find_sinks=False and matches oracle.denoise_block, whose second step
    keeps the first step's sinks although its own queries would pick
    others."""
    wl = synth.workload("llada32k_step", batch=2, L_ctx=4096, n_layers=3, topK=16)
    desc = desc_for(wl)
    n_layers = 3
    ctx = [synth.make_step_inputs(wl, layer=l, device=cuda_device) for l in range(n_layers)]
    steps = []
    for sd in (wl.seed, wl.seed + 11):
        xs = [synth.make_step_inputs(wl.replace(seed=sd), layer=l, device=cuda_device)
              for l in range(n_layers)]
        steps.append(dict(conf_prev=xs[0].conf_prev, still_masked=xs[0].still_masked,
                          q_dec=[x.q_dec for x in xs], k_dec=[x.k_dec for x in xs],
                          v_dec=[x.v_dec for x in xs]))
    step = pipeline.DenoiseStep(desc, n_layers, wl.first_sparse_layer, wl.topK, wl.detect_sinks,
                                wl.k, wl.w, torch.bfloat16, cuda_device)
    kcs = [step.key_cache() for _ in range(n_layers)]
    for l in range(n_layers):
        step.refresh_pooled_keys(l, ctx[l].k_pool, ctx[l].page_table, kcs[l])
    got = []
    for t, st in enumerate(steps):
        step.run(st["conf_prev"], st["still_masked"], st["q_dec"], [x.k_pool for x in ctx],
                 [x.v_pool for x in ctx], ctx[0].page_table, st["k_dec"], st["v_dec"], kcs,
                 find_sinks=(t == 0))
        torch.cuda.synchronize()
        assert dl.dl_get_status() == dl.DL_OK
        got.append(dict(sink_pos=np_(step.sink_pos), q_idx=np_(step.q_idx),
                        blk_idx=[np_(b) for b in step.blk_idx],
                        blk_cnt=[np_(b) for b in step.blk_cnt],
                        O=[o.clone() for o in step.O], lse=[x.clone() for x in step.lse]))
    cpu = lambda xs: [x.cpu() for x in xs]  # noqa: E731
    ref = oracle.denoise_block(cpu([x.k_pool for x in ctx]), cpu([x.v_pool for x in ctx]),
                               ctx[0].page_table.cpu(),
                               [dict(conf_prev=s["conf_prev"].cpu(),
                                     still_masked=s["still_masked"].cpu(),
                                     q_dec=cpu(s["q_dec"]), k_dec=cpu(s["k_dec"]),
                                     v_dec=cpu(s["v_dec"])) for s in steps],
                               wl.L_ctx, wl.B, wl.topK, first_sparse=wl.first_sparse_layer,
                               n_sinks=wl.detect_sinks, k=wl.k, w=wl.w)
    fs = wl.first_sparse_layer
    for t in range(2):
        assert np.array_equal(got[t]["q_idx"], ref[t][fs].q_idx), f"step {t} q_idx"
        assert np.array_equal(got[t]["sink_pos"], ref[t][fs].sink_pos), f"step {t} sinks"
        for l in range(n_layers):
            if l >= fs:
                assert np.array_equal(got[t]["blk_idx"][l], ref[t][l].blk_idx), f"{t}/{l}"
                assert np.array_equal(got[t]["blk_cnt"][l], ref[t][l].blk_cnt), f"{t}/{l}"
            check_attention(got[t]["O"][l], got[t]["lse"][l], ref[t][l].O, ref[t][l].lse, False,
                            f"step {t} layer {l}")
