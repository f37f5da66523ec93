"""Head-sharded sink search (long_context_diffusion_b200/sharded.py) on CPU:
the KV-head ranges, the per-shard descriptors, and two or three gloo ranks
that each hold only their heads, compute their part of the sink mass (the
oracle's find_sinks over those heads stands in for dl_sink_mass, which needs
a GPU), sum the parts with the all-reduce of reduce_and_pick and pick the
sinks.  Every rank must end with the whole model's mass and the sinks the
oracle finds over all heads."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import long_context_diffusion_b200 as dl
from long_context_diffusion_b200 import runtime, sharded


@pytest.mark.parametrize("H_kv,world", [(4, 1), (4, 2), (3, 2), (32, 8), (5, 3), (8, 8)])
def test_kv_head_ranges_partition_the_heads(H_kv, world):
    spans = [sharded.kv_head_range(H_kv, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == H_kv
    for (_, hi), (lo, _) in zip(spans, spans[1:]):
        assert hi == lo
    sizes = [hi - lo for lo, hi in spans]
    assert min(sizes) >= 1 and max(sizes) - min(sizes) <= 1


def test_kv_head_range_rejects_bad_splits():
    with pytest.raises(ValueError):
        sharded.kv_head_range(2, 0, 3)
    with pytest.raises(ValueError):
        sharded.kv_head_range(4, 2, 2)


def test_shard_desc_keeps_every_other_size():
    d = dl.make_desc(2, 28, 4, 128, 16384, 32, 64, 256, 512, dl.DL_BF16)
    shards = [sharded.HeadShard.of(d, r, 3) for r in range(3)]
    assert [s.desc.H_kv for s in shards] == [2, 1, 1]
    assert [s.desc.H for s in shards] == [14, 7, 7]
    assert [s.heads for s in shards] == [(0, 14), (14, 21), (21, 28)]
    for s in shards:
        for name, _ in d._fields_:
            if name not in ("H", "H_kv"):
                assert getattr(s.desc, name) == getattr(d, name), name


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed=3):
    """A GQA sink search: H=6 query heads over H_kv=3 KV heads, two
    sequences, with a planted column of large mass in each."""
    r = np.random.default_rng(seed)
    B, H, H_kv, L_ctx, L_q, d = 2, 6, 3, 96, 8, 16
    Q = r.standard_normal((B, H, L_q, d)) / 4
    Kc = r.standard_normal((B, H_kv, L_ctx, d)) / 4
    Kd = r.standard_normal((B, H_kv, L_q, d)) / 4
    for b in range(B):
        v = r.standard_normal(d)
        v /= np.linalg.norm(v)
        Q[b] += v                       # a direction every query shares ...
        Kc[b, :, 17 + 40 * b] += 6 * v  # ... and one column that follows it
    rows = [np.array([0, 1, 2, 5]), np.array([3, 4, 6, 7])]
    return Q, Kc, Kd, rows


def _oracle_topn(n):
    from oracle import steps as S

    def topn(mass, sink_pos, stream=None):
        for b in range(mass.shape[0]):
            top = np.sort(S.topk_lower_index(mass[b].numpy(), n))
            sink_pos[b] = torch.from_numpy(top.astype(np.int32))
    return topn


def _rank_main(rank, world, port, n_sinks, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from oracle import steps as S
    r, w, _, _ = runtime.init(backend="gloo", timeout_s=60)
    Q, Kc, Kd, rows = _problem()
    B, H, L_q, d = Q.shape
    H_kv, L_ctx = Kc.shape[1], Kc.shape[2]
    desc = dl.make_desc(B, H, H_kv, d, L_ctx, L_q, 16, L_ctx // 16, L_ctx // 16, dl.DL_FP32)
    shard = sharded.HeadShard.of(desc, r, w)
    h0, h1 = shard.heads
    # this rank holds only its heads: its part of the mass
    mass = torch.zeros((B, L_ctx), dtype=torch.float64)
    for b in range(B):
        _, m = S.find_sinks(Q[b, h0:h1], Kc[b, shard.g0:shard.g1], Kd[b, shard.g0:shard.g1],
                            rows[b], n_sinks, S.scale_for(d))
        mass[b] = torch.from_numpy(m)
    sink_pos = torch.full((B, n_sinks), -1, dtype=torch.int32)
    sharded.reduce_and_pick(mass, sink_pos, topn=_oracle_topn(n_sinks))
    out[r] = (shard.g0, shard.g1, mass.numpy().tolist(), sink_pos.numpy().tolist())
    runtime.finalize()


@pytest.mark.parametrize("world,n_sinks", [(2, 4), (3, 2)])
def test_gloo_ranks_sum_the_shard_masses(world, n_sinks):
    from oracle import steps as S
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, n_sinks, out), nprocs=world,
                           join=True, start_method="spawn")
        res = dict(out)
    assert sorted(res) == list(range(world))
    Q, Kc, Kd, rows = _problem()
    d = Q.shape[-1]
    want_mass, want_sinks = [], []
    for b in range(Q.shape[0]):
        top, m = S.find_sinks(Q[b], Kc[b], Kd[b], rows[b], n_sinks, S.scale_for(d))
        want_mass.append(m)
        want_sinks.append(top.tolist())
    assert sorted((v[0], v[1]) for v in res.values())[0][0] == 0
    for g0, g1, mass, sinks in res.values():
        assert np.allclose(np.array(mass), np.array(want_mass), rtol=1e-12, atol=0)
        assert sinks == want_sinks
    # the planted columns lead in both sequences
    assert all(17 + 40 * b in want_sinks[b] for b in range(2))


def test_reduce_and_pick_without_a_group_only_picks():
    mass = torch.tensor([[0.5, 3.0, 3.0, 1.0]], dtype=torch.float64)
    sink_pos = torch.empty((1, 2), dtype=torch.int32)
    sharded.reduce_and_pick(mass, sink_pos, topn=_oracle_topn(2))
    assert sink_pos.tolist() == [[1, 2]]
    assert mass.tolist() == [[0.5, 3.0, 3.0, 1.0]]
