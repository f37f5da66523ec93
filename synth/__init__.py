"""Seeded synthetic inputs for the sparse-attention denoising step.

This module only draws numbers.  It holds none of the method's arithmetic
(no prediction, pooling, scoring, selection or attention): both the fp64
oracle and the CUDA path receive the tensors it returns, so the two sides
share nothing but their inputs.

Generator
---------
Every value comes from splitmix64 used as a counter-based generator.  The
published splitmix64 (Steele, Lea, Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) advances a 64-bit state by the golden gamma
0x9E3779B97F4A7C15 and returns mix64(state).  Here stream (seed, sid) starts
at state0 = mix64((seed << 32) ^ sid); its i-th draw (i = 0, 1, ...) is
mix64(state0 + (i + 1) * gamma), so any slice of a tensor can be drawn
without drawing what precedes it.  All arithmetic is mod 2**64 on torch int64
tensors, so the same code runs on CPU and on CUDA and gives the same bits.

Uniforms are u = ((x >> 11) + 0.5) * 2**-53, in (0, 1).  Normals use
Box-Muller on draws 2j and 2j+1: sqrt(-2 ln u1) * cos(2 pi u2), in fp64.
Values are rounded to nearest-even into bf16 (or fp32) only at the end.

Workloads
---------
The five named workloads follow the shapes of the pages' long-context dLLM
runs (LLaDA-8B / Dream-7B attention shapes at 8K-32K context; Prefilling-dLLM
chunked prefix).  No benchmark item or model weight is used: every tensor is
drawn here from the recipe stated in each workload's docstring.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

__all__ = [
    "GAMMA", "mix64_int", "splitmix64_draws", "uniforms", "normals",
    "Workload", "WORKLOADS", "workload", "StepInputs", "make_step_inputs",
    "make_layer_kv", "sink_positions", "confidence", "page_permutation",
]

GAMMA = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB
_MASK64 = (1 << 64) - 1


def _i64(u: int) -> int:
    """Reinterpret an unsigned 64-bit integer as two's-complement int64."""
    u &= _MASK64
    return u - (1 << 64) if u >= (1 << 63) else u


def mix64_int(z: int) -> int:
    """splitmix64's output mix on a Python int (unsigned 64-bit)."""
    z &= _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def _srl(x: torch.Tensor, s: int) -> torch.Tensor:
    """Logical right shift of an int64 tensor (torch's >> is arithmetic)."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix64(z: torch.Tensor) -> torch.Tensor:
    z = (z ^ _srl(z, 30)) * _i64(_M1)
    z = (z ^ _srl(z, 27)) * _i64(_M2)
    return z ^ _srl(z, 31)


def splitmix64_draws(seed: int, sid: int, start: int, n: int,
                     device="cpu") -> torch.Tensor:
    """Draws start .. start+n-1 of stream (seed, sid), as int64 bit patterns."""
    state0 = mix64_int(((seed & 0xFFFFFFFF) << 32) ^ (sid & 0xFFFFFFFF))
    idx = torch.arange(start + 1, start + n + 1, dtype=torch.int64, device=device)
    z = idx * _i64(GAMMA) + _i64(state0)
    return _mix64(z)


def uniforms(seed: int, sid: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """fp64 uniforms in (0, 1) from draws start .. start+n-1."""
    x = splitmix64_draws(seed, sid, start, n, device)
    return (_srl(x, 11).to(torch.float64) + 0.5) * (2.0 ** -53)


def normals(seed: int, sid: int, start: int, n: int, device="cpu") -> torch.Tensor:
    """fp64 standard normals number start .. start+n-1 of stream (seed, sid).

    Normal j uses draws 2j and 2j+1 (Box-Muller, cosine branch)."""
    u = uniforms(seed, sid, 2 * start, 2 * n, device).view(n, 2)
    r = torch.sqrt(-2.0 * torch.log(u[:, 0]))
    return r * torch.cos((2.0 * math.pi) * u[:, 1])


# ----------------------------------------------------------------------------
# stream ids
# ----------------------------------------------------------------------------
_T_Q, _T_K, _T_V, _T_KDEC, _T_VDEC = 1, 2, 3, 4, 5
_T_CONF_NOISE, _T_CONF_BETA, _T_UNMASK, _T_SINKPOS, _T_PERM = 6, 7, 8, 9, 10
_STEP_LAYER = 0xFFF  # per-step quantities (shared by all layers)


def _sid(wid: int, layer: int, kind: int) -> int:
    return ((wid & 0xFF) << 24) | ((layer & 0xFFF) << 12) | (kind & 0xFFF)


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape, structure and method knobs of one synthetic workload."""
    name: str
    wid: int                 # stream-id namespace of this workload
    dtype: str               # "fp32" or "bf16"
    batch: int
    H: int
    H_kv: int
    d: int
    L_ctx: int               # cached context tokens per sequence
    L_q: int                 # decode-block length
    B: int = 64              # key-block size (= page size)
    topK: int = 4
    k: int = 4               # predicted positions (previous-step top-k)
    w: int = 2               # half-width of the window around each prediction
    n_layers: int = 1
    first_sparse_layer: int = 0   # layers below it are dense
    n_planted: int = 1       # planted sink positions: 0 plus n_planted-1 random
    sinks_given: int = 0     # >0: the first sinks_given planted positions are
                             # handed to selection as the sink list
    detect_sinks: int = 0    # >0: sinks found by attention mass at the first
                             # sparse layer (that many columns)
    n_unmasked: int = 8      # decode positions already unmasked
    conf_kind: str = "beta"  # "uniform" or "beta"
    scale_qkv: float = 1.0   # inputs are N(0,1) * scale_qkv
    seed: int = 0
    # chunked (Prefilling-dLLM) layout
    chunked: bool = False
    n_chunks: int = 0
    chunk_content: int = 0   # content tokens per chunk (BOS not counted)
    topK_chunks: int = 0
    topT_tokens: int = 0
    permute_pages: bool = False
    nan_padding: bool = False  # fill unused pool rows with NaN (edge tests)

    @property
    def G(self) -> int:
        return self.H // self.H_kv

    @property
    def chunk_tokens(self) -> int:          # BOS + content
        return self.chunk_content + 1

    @property
    def chunk_pages(self) -> int:
        return -(-self.chunk_tokens // self.B)

    @property
    def chunk_stride(self) -> int:          # logical tokens between chunk starts
        return self.chunk_pages * self.B

    @property
    def n_pages(self) -> int:               # logical pages per sequence
        if self.chunked:
            return self.n_chunks * self.chunk_pages
        return -(-self.L_ctx // self.B)

    @property
    def n_blk(self) -> int:
        return -(-self.L_ctx // self.B)

    @property
    def n_slots(self) -> int:
        return self.batch * self.n_pages

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == "fp32" else torch.bfloat16

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # Tiny single-layer step: fp32, MHA, d=64, 1K context, sink block 0 given.
    "tiny": Workload(name="tiny", wid=1, dtype="fp32", batch=1, H=4, H_kv=4, d=64,
                     L_ctx=1024, L_q=32, topK=4, n_planted=2, sinks_given=1,
                     conf_kind="uniform", scale_qkv=1.0 / 8.0),
    # LLaDA-8B-shaped single layer at 8K.
    "llada8k": Workload(name="llada8k", wid=2, dtype="bf16", batch=1, H=32, H_kv=32,
                        d=128, L_ctx=8192, L_q=32, topK=32, n_planted=4, sinks_given=4),
    # Dream-7B-shaped GQA layer at 16K, batch 2.
    "dream16k": Workload(name="dream16k", wid=3, dtype="bf16", batch=2, H=28, H_kv=4,
                         d=128, L_ctx=16384, L_q=32, topK=64, n_planted=4, sinks_given=4),
    # Full 32-layer step at 32K, batch 4: layers 0-1 dense, sinks found at layer 2.
    "llada32k_step": Workload(name="llada32k_step", wid=4, dtype="bf16", batch=4, H=32,
                              H_kv=32, d=128, L_ctx=32768, L_q=32, topK=128,
                              n_layers=32, first_sparse_layer=2, n_planted=4,
                              detect_sinks=4),
    # Chunked non-contiguous prefix: 32 chunks of BOS + 1024 tokens, permuted pages.
    "chunked32k": Workload(name="chunked32k", wid=5, dtype="bf16", batch=1, H=32, H_kv=32,
                           d=128, L_ctx=32 * 1088, L_q=64, n_planted=0, chunked=True,
                           n_chunks=32, chunk_content=1024, topK_chunks=8,
                           topT_tokens=256, permute_pages=True),
}


def workload(name: str, **overrides) -> Workload:
    return WORKLOADS[name].replace(**overrides) if overrides else WORKLOADS[name]


# ----------------------------------------------------------------------------
# per-step quantities
# ----------------------------------------------------------------------------
def _argsort_keys(wl: Workload, kind: int, b: int, n: int) -> torch.Tensor:
    """A seeded random permutation of range(n): order of n uniform keys."""
    u = uniforms(wl.seed, _sid(wl.wid, _STEP_LAYER, kind), b * n, n)
    return torch.argsort(u, stable=True)


def sink_positions(wl: Workload, b: int) -> list:
    """Planted sink positions of sequence b: 0 plus n_planted-1 distinct random
    positions in [1, L_ctx), ascending.  Shared by every layer."""
    if wl.n_planted <= 0:
        return []
    perm = _argsort_keys(wl, _T_SINKPOS, b, wl.L_ctx - 1)
    extra = sorted(int(p) + 1 for p in perm[: wl.n_planted - 1])
    return [0] + extra


def confidence(wl: Workload, b: int):
    """Previous-step confidence (fp32) and still-masked flags (uint8) of
    sequence b.  n_unmasked random positions are already decoded."""
    L = wl.L_q
    if wl.conf_kind == "uniform":
        c = uniforms(wl.seed, _sid(wl.wid, _STEP_LAYER, _T_CONF_BETA), b * L, L)
    else:
        # Beta(2,5) as the 2nd smallest of 6 uniforms, plus N(0, 0.05), clipped.
        u = uniforms(wl.seed, _sid(wl.wid, _STEP_LAYER, _T_CONF_BETA), b * L * 6, L * 6)
        beta = torch.sort(u.view(L, 6), dim=1).values[:, 1]
        noise = normals(wl.seed, _sid(wl.wid, _STEP_LAYER, _T_CONF_NOISE), b * L, L)
        c = torch.clamp(beta + 0.05 * noise, 0.0, 1.0)
    conf = c.to(torch.float32)
    masked = torch.ones(L, dtype=torch.uint8)
    perm = _argsort_keys(wl, _T_UNMASK, b, L)
    masked[perm[: min(wl.n_unmasked, L)]] = 0
    return conf, masked


def page_permutation(wl: Workload) -> torch.Tensor:
    """Logical page (b, p) -> pool slot.  Identity unless permute_pages."""
    n = wl.n_slots
    if not wl.permute_pages:
        return torch.arange(n, dtype=torch.int32).view(wl.batch, wl.n_pages)
    perm = _argsort_keys(wl, _T_PERM, 0, n)
    return perm.to(torch.int32).view(wl.batch, wl.n_pages)


# ----------------------------------------------------------------------------
# per-layer tensors
# ----------------------------------------------------------------------------
def _round(x: torch.Tensor, wl: Workload) -> torch.Tensor:
    return x.to(wl.torch_dtype)


def make_q_dec(wl: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Q of the decode block, [batch][H][L_q][d]."""
    n = wl.batch * wl.H * wl.L_q * wl.d
    x = normals(wl.seed, _sid(wl.wid, layer, _T_Q), 0, n, device) * wl.scale_qkv
    return _round(x, wl).view(wl.batch, wl.H, wl.L_q, wl.d)


def make_kv_dec(wl: Workload, layer: int, device="cpu"):
    """K and V of the decode block, [batch][H_kv][L_q][d] each."""
    n = wl.batch * wl.H_kv * wl.L_q * wl.d
    shape = (wl.batch, wl.H_kv, wl.L_q, wl.d)
    k = normals(wl.seed, _sid(wl.wid, layer, _T_KDEC), 0, n, device) * wl.scale_qkv
    v = normals(wl.seed, _sid(wl.wid, layer, _T_VDEC), 0, n, device) * wl.scale_qkv
    return _round(k, wl).view(shape), _round(v, wl).view(shape)


def _logical_tokens(wl: Workload) -> int:
    """Tokens per sequence in the logical (unpaged) context stream."""
    return wl.n_chunks * wl.chunk_tokens if wl.chunked else wl.L_ctx


def make_logical_kv(wl: Workload, layer: int, b: int, g0: int, g1: int,
                    q_dec: Optional[torch.Tensor], device="cpu"):
    """Context K and V of sequence b, KV heads g0..g1-1, in logical token order:
    [g1-g0][tokens][d] in the workload dtype.  For chunked workloads the token
    order is chunk-major (BOS first in each chunk).  Planted sink positions get
    3 * mean(Q of the group's heads over the decode block) added to K before
    rounding."""
    T = _logical_tokens(wl)
    d = wl.d
    per_head = T * d
    start = (b * wl.H_kv + g0) * per_head
    n = (g1 - g0) * per_head
    k = normals(wl.seed, _sid(wl.wid, layer, _T_K), start, n, device) * wl.scale_qkv
    v = normals(wl.seed, _sid(wl.wid, layer, _T_V), start, n, device) * wl.scale_qkv
    k = k.view(g1 - g0, T, d)
    v = v.view(g1 - g0, T, d)
    sinks = sink_positions(wl, b)
    if sinks:
        assert q_dec is not None
        G = wl.G
        for gi, g in enumerate(range(g0, g1)):
            qg = q_dec[b, g * G:(g + 1) * G].to(device=device, dtype=torch.float64)
            qbar = qg.reshape(-1, d).mean(dim=0)
            for p in sinks:
                k[gi, p] += 3.0 * qbar
    return _round(k, wl), _round(v, wl)


def make_layer_kv(wl: Workload, layer: int, q_dec: Optional[torch.Tensor],
                  device="cpu", page_table: Optional[torch.Tensor] = None):
    """Paged K and V pools of one layer: [n_slots][H_kv][B][d] each.

    Logical page p of sequence b lives in slot page_table[b][p].  Rows of a
    page past the end of the context (or of a chunk) are zero, or NaN when
    wl.nan_padding is set, and must never be read as keys."""
    if page_table is None:
        page_table = page_permutation(wl)
    B, d = wl.B, wl.d
    fill = float("nan") if wl.nan_padding else 0.0
    kp = torch.full((wl.n_slots, wl.H_kv, B, d), fill, dtype=wl.torch_dtype, device=device)
    vp = torch.full_like(kp, fill)
    pt = page_table.to(device=device, dtype=torch.int64)
    for b in range(wl.batch):
        k, v = make_logical_kv(wl, layer, b, 0, wl.H_kv, q_dec, device)
        if wl.chunked:
            # chunk c: tokens 0..chunk_tokens-1 -> logical pages c*chunk_pages + t//B
            ct, cp = wl.chunk_tokens, wl.chunk_pages
            padded = torch.full((wl.H_kv, wl.n_chunks, cp * B, d), fill,
                                dtype=wl.torch_dtype, device=device)
            padded_v = padded.clone()
            padded[:, :, :ct] = k.view(wl.H_kv, wl.n_chunks, ct, d)
            padded_v[:, :, :ct] = v.view(wl.H_kv, wl.n_chunks, ct, d)
            kk = padded.view(wl.H_kv, wl.n_pages, B, d)
            vv = padded_v.view(wl.H_kv, wl.n_pages, B, d)
        else:
            n_full = wl.L_ctx
            padded = torch.full((wl.H_kv, wl.n_pages * B, d), fill,
                                dtype=wl.torch_dtype, device=device)
            padded_v = padded.clone()
            padded[:, :n_full] = k
            padded_v[:, :n_full] = v
            kk = padded.view(wl.H_kv, wl.n_pages, B, d)
            vv = padded_v.view(wl.H_kv, wl.n_pages, B, d)
        slots = pt[b]
        kp[slots] = kk.permute(1, 0, 2, 3)
        vp[slots] = vv.permute(1, 0, 2, 3)
    return kp, vp


@dataclasses.dataclass
class StepInputs:
    """Everything one layer of one denoising step reads (CPU tensors unless a
    device was requested)."""
    wl: Workload
    layer: int
    q_dec: torch.Tensor        # [batch][H][L_q][d]
    k_dec: torch.Tensor        # [batch][H_kv][L_q][d]
    v_dec: torch.Tensor
    k_pool: torch.Tensor       # [n_slots][H_kv][B][d]
    v_pool: torch.Tensor
    page_table: torch.Tensor   # int32 [batch][n_pages]
    conf_prev: torch.Tensor    # fp32 [batch][L_q]
    still_masked: torch.Tensor  # uint8 [batch][L_q]
    sinks_planted: torch.Tensor  # int32 [batch][n_planted]


def make_step_inputs(wl: Workload, layer: int = 0, device="cpu") -> StepInputs:
    q = make_q_dec(wl, layer, device)
    kd, vd = make_kv_dec(wl, layer, device)
    pt = page_permutation(wl)
    kp, vp = make_layer_kv(wl, layer, q, device, pt)
    confs, masks = zip(*(confidence(wl, b) for b in range(wl.batch)))
    sinks = torch.tensor([sink_positions(wl, b) for b in range(wl.batch)],
                         dtype=torch.int32).view(wl.batch, max(wl.n_planted, 0))
    return StepInputs(wl=wl, layer=layer, q_dec=q, k_dec=kd, v_dec=vd, k_pool=kp,
                      v_pool=vp, page_table=pt.to(device), conf_prev=torch.stack(confs).to(device),
                      still_masked=torch.stack(masks).to(device), sinks_planted=sinks.to(device))
