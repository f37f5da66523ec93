"""The N > 1 plumbing of the benchmark (long_context_diffusion_b200/runtime.py)
on CPU: work sharding, whole-job throughput, and two gloo ranks that run
independent shards and agree on the slowest rank's time (max over ranks) and
on the total work (sum over ranks), as bench.py does on N GPUs."""
import os
import socket

import pytest
import torch.multiprocessing as mp

from long_context_diffusion_b200 import runtime


@pytest.mark.parametrize("n,world", [(0, 2), (1, 2), (7, 2), (128, 3), (5, 8), (128, 8)])
def test_shard_partitions_the_items(n, world):
    spans = [runtime.shard(n, r, world) for r in range(world)]
    assert spans[0][0] == 0 and spans[-1][1] == n
    for (lo, hi), (lo2, _) in zip(spans, spans[1:]):
        assert hi == lo2
    sizes = [hi - lo for lo, hi in spans]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == n


def test_weak_throughput_is_total_over_slowest():
    assert runtime.weak_throughput([3, 3], 0.5) == 12.0
    assert runtime.weak_throughput([1] * 8, 2.0) == 4.0
    assert runtime.weak_throughput([4], 0.0) == 0.0


def test_single_process_collectives_are_identities():
    assert runtime.max_over_ranks(2.5, "cpu") == 2.5
    assert runtime.sum_over_ranks(2.5, "cpu") == 2.5
    runtime.barrier()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    r, w, _, device = runtime.init(backend="gloo", timeout_s=60)
    lo, hi = runtime.shard(10, r, w)
    runtime.barrier(device)
    # each rank "times" its own shard; the job's time is the slowest rank's
    t_mine = 0.1 * (r + 1)
    t_max = runtime.max_over_ranks(t_mine, device)
    units = runtime.sum_over_ranks(hi - lo, device)
    runtime.barrier(device)
    out[r] = (r, w, lo, hi, t_max, units, runtime.weak_throughput([units], t_max))
    runtime.finalize()


def test_two_gloo_ranks_agree_on_time_and_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True,
                           start_method="spawn")
        res = dict(out)
    assert sorted(res) == [0, 1]
    spans = sorted((v[2], v[3]) for v in res.values())
    assert spans == [(0, 5), (5, 10)]
    for r, w, lo, hi, t_max, units, thr in res.values():
        assert w == 2 and t_max == pytest.approx(0.2) and units == 10
        assert thr == pytest.approx(10 / 0.2)
