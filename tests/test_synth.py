"""The seeded generator: published splitmix64 answers, ranges, structure."""
import numpy as np
import pytest
import torch

import synth


def test_splitmix64_known_answers():
    # published first outputs of splitmix64 started from state 0
    assert synth.mix64_int(synth.GAMMA) == 0xE220A8397B1DCDAF
    state0 = 0
    outs = []
    for _ in range(3):
        state0 = (state0 + synth.GAMMA) & ((1 << 64) - 1)
        outs.append(synth.mix64_int(state0))
    assert outs == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_draws_match_python_ints_and_slices():
    seed, sid = 7, 0x1234
    x = synth.splitmix64_draws(seed, sid, 0, 50)
    st = synth.mix64_int((seed << 32) ^ sid)
    ref = [synth.mix64_int(st + (i + 1) * synth.GAMMA) for i in range(50)]
    assert [int(v) & ((1 << 64) - 1) for v in x] == ref
    # any slice is drawn without the draws before it
    assert torch.equal(synth.splitmix64_draws(seed, sid, 20, 10), x[20:30])


def test_uniform_and_normal_ranges():
    u = synth.uniforms(0, 1, 0, 200000)
    assert float(u.min()) > 0.0 and float(u.max()) < 1.0
    n = synth.normals(0, 2, 0, 200000)
    assert abs(float(n.mean())) < 0.01 and abs(float(n.std()) - 1.0) < 0.01


def test_workload_structure():
    wl = synth.workload("llada8k")
    for b in range(2):
        s = synth.sink_positions(wl.replace(batch=2), b)
        assert s[0] == 0 and len(set(s)) == 4 and s == sorted(s) and max(s) < wl.L_ctx
    conf, masked = synth.confidence(wl, 0)
    assert conf.dtype == torch.float32 and float(conf.min()) >= 0 and float(conf.max()) <= 1
    assert int((masked == 0).sum()) == wl.n_unmasked
    wc = synth.workload("chunked32k")
    pt = synth.page_permutation(wc)
    assert sorted(pt.view(-1).tolist()) == list(range(wc.n_slots))


def test_planted_sink_keys():
    wl = synth.workload("tiny")
    q = synth.make_q_dec(wl, 0)
    k, _ = synth.make_logical_kv(wl, 0, 0, 0, 1, q)
    k_plain, _ = synth.make_logical_kv(wl.replace(n_planted=0), 0, 0, 0, 1, None)
    sinks = synth.sink_positions(wl, 0)
    diff = (k - k_plain).abs().sum(-1)[0]
    assert set(torch.nonzero(diff).view(-1).tolist()) == set(sinks)


@pytest.mark.gpu
def test_generator_same_bits_on_cuda(cuda_device):
    a = synth.splitmix64_draws(3, 99, 1000, 4096)
    b = synth.splitmix64_draws(3, 99, 1000, 4096, device=cuda_device).cpu()
    assert torch.equal(a, b)
    wl = synth.workload("tiny")
    qa = synth.make_q_dec(wl, 0)
    qb = synth.make_q_dec(wl, 0, device=cuda_device).cpu()
    assert torch.equal(qa, qb)
