"""Head-sharded execution of the denoising step over several GPUs.

Every step of the path is independent per (sequence, KV head) except the
sink search: the attention mass of a context column is a sum over all heads
(Focus-dLLM abstract: the sink locations are shared by every head and reused
across layers).  Ranks hold disjoint, contiguous ranges of KV heads, each
with its G query heads and only those heads' KV.  A rank computes its heads'
part of the mass (dl_sink_mass), one all-reduce (sum) of mass[b][L_ctx] over
the ranks gives the whole mass, and every rank picks the same sinks from it
(dl_sink_topn).  Nothing else crosses GPUs: no peer memory is read.

The reduction sums fp32 partial masses in the collective's order, so near
ties the chosen sinks can differ from a single-GPU run by the rounding of
that sum; an exact tie still goes to the lower position.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional, Tuple

import torch
import torch.distributed as dist

from . import _abi as A


def kv_head_range(H_kv: int, rank: int, world: int) -> Tuple[int, int]:
    """[g0, g1): the KV heads of `rank`, contiguous, sizes differing by at
    most one (the lower ranks take the extra heads)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if H_kv < world:
        raise ValueError(f"{H_kv} KV heads cannot be spread over {world} ranks")
    base, extra = divmod(H_kv, world)
    g0 = rank * base + min(rank, extra)
    return g0, g0 + base + (1 if rank < extra else 0)


def shard_desc(desc: A.dl_attn_desc, rank: int, world: int) -> A.dl_attn_desc:
    """The descriptor of one rank's heads: H_kv and H = G * H_kv of its
    range, every other size unchanged."""
    G = desc.H // desc.H_kv
    g0, g1 = kv_head_range(desc.H_kv, rank, world)
    out = A.dl_attn_desc()
    for name, _ in A.dl_attn_desc._fields_:
        setattr(out, name, getattr(desc, name))
    out.H_kv = g1 - g0
    out.H = G * (g1 - g0)
    return out


def reduce_and_pick(mass: torch.Tensor, sink_pos: torch.Tensor, group=None,
                    topn: Optional[Callable] = None, stream=None) -> torch.Tensor:
    """Sum the ranks' partial masses in place (all-reduce over `group`; no
    collective without an initialised process group of more than one rank),
    then pick the sinks into sink_pos with `topn` (default dl_sink_topn)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        if stream is not None and mass.is_cuda:
            if not isinstance(stream, torch.cuda.Stream):
                stream = torch.cuda.ExternalStream(int(stream))
            with torch.cuda.stream(stream):
                dist.all_reduce(mass, op=dist.ReduceOp.SUM, group=group)
        else:
            dist.all_reduce(mass, op=dist.ReduceOp.SUM, group=group)
    (topn or A.dl_sink_topn)(mass, sink_pos, stream)
    return sink_pos


@dataclasses.dataclass
class HeadShard:
    """One rank's share of a head-sharded layer: its descriptor and the
    KV-head range it holds."""
    rank: int
    world: int
    desc: A.dl_attn_desc
    g0: int
    g1: int

    @classmethod
    def of(cls, desc: A.dl_attn_desc, rank: int, world: int) -> "HeadShard":
        g0, g1 = kv_head_range(desc.H_kv, rank, world)
        return cls(rank, world, shard_desc(desc, rank, world), g0, g1)

    @property
    def heads(self) -> Tuple[int, int]:
        """[h0, h1): the query heads of this rank."""
        G = self.desc.H // self.desc.H_kv
        return self.g0 * G, self.g1 * G


def find_sinks_sharded(shard: HeadShard, q_dec, q_idx, q_cnt, k_pool, page_table, k_dec,
                       mass: torch.Tensor, sink_pos: torch.Tensor, ws, group=None,
                       stream=None) -> torch.Tensor:
    """Sinks of the whole model from one rank's heads: q_dec / k_pool / k_dec
    hold only this rank's heads (shard.desc); mass fp32 [batch][L_ctx] is
    scratch.  Every rank gets the same sink_pos."""
    A.dl_sink_mass(shard.desc, q_dec, q_idx, q_cnt, k_pool, page_table, k_dec, mass, ws, stream)
    return reduce_and_pick(mass, sink_pos, group, stream=stream)
