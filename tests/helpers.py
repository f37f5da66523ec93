"""Shared test helpers: descriptors for the synthetic workloads and the
tolerance checks of the parity bar."""
import numpy as np
import torch

import long_context_diffusion_b200 as dl

# Parity bar: bf16 attention outputs within max-abs 2e-2 and mean-abs 2e-3
# of the fp64 oracle; fp32 inputs within 1e-5.  The LSE is accumulated in
# fp32 from exactly converted inputs; 1e-3 (bf16) / 1e-5 (fp32) absolute.
BF16_MAX_ABS, BF16_MEAN_ABS, FP32_MAX_ABS = 2e-2, 2e-3, 1e-5
BF16_LSE_ABS, FP32_LSE_ABS = 1e-3, 1e-5


def desc_for(wl, L_ctx=None):
    return dl.make_desc(batch=wl.batch, H=wl.H, H_kv=wl.H_kv, d=wl.d,
                        L_ctx=wl.L_ctx if L_ctx is None else L_ctx, L_q=wl.L_q, page=wl.B,
                        n_pages=wl.n_pages, n_slots=wl.n_slots,
                        dtype=dl.DL_BF16 if wl.dtype == "bf16" else dl.DL_FP32)


def np_(t):
    return t.detach().to("cpu").to(torch.float64).numpy() if t.is_floating_point() \
        else t.detach().to("cpu").numpy().astype(np.int64)


def check_attention(O_gpu, lse_gpu, O_ref, lse_ref, fp32: bool, what=""):
    O = np_(O_gpu)
    err = np.abs(O - O_ref)
    lerr = np.abs(np_(lse_gpu) - lse_ref)
    if fp32:
        assert err.max() <= FP32_MAX_ABS, f"{what} fp32 max-abs {err.max():.3g}"
        assert lerr.max() <= FP32_LSE_ABS, f"{what} fp32 lse max-abs {lerr.max():.3g}"
    else:
        assert err.max() <= BF16_MAX_ABS, f"{what} bf16 max-abs {err.max():.3g}"
        assert err.mean() <= BF16_MEAN_ABS, f"{what} bf16 mean-abs {err.mean():.3g}"
        assert lerr.max() <= BF16_LSE_ABS, f"{what} lse max-abs {lerr.max():.3g}"
    return float(err.max()), float(err.mean())


def cut_margin(values, kept, excluded=()):
    """Oracle gap at a top-k cut: smallest kept value minus largest dropped
    value (candidates only)."""
    v = np.asarray(values, dtype=np.float64)
    mask = np.ones(len(v), dtype=bool)
    mask[list(excluded)] = False
    keep = np.zeros(len(v), dtype=bool)
    keep[list(kept)] = True
    a = v[mask & keep]
    b = v[mask & ~keep]
    if len(a) == 0 or len(b) == 0:
        return float("inf")
    return float(a.min() - b.max())


def key_digits_np(kbar):
    """The integer-digit form of fp32 pooled keys [..., d] that dl_pool_keys
    documents (include/dl.h): per row the largest exponent field E (at least
    1), every value as V = trunc(m * 2^(11 - (E - e))), negated when negative,
    written base 128 with a signed top digit.  Returns (Kdig [..., 5, d] moved
    to the plane axis by the caller, Kexp [...]) as int8 / int32 arrays with
    the digit plane as the second-to-last axis."""
    x = np.ascontiguousarray(np.asarray(kbar, dtype=np.float32))
    u = x.view(np.uint32).astype(np.int64)
    sign = (u >> 31) & 1
    e = (u >> 23) & 0xFF
    mant = u & 0x7FFFFF
    m = np.where(e == 0, mant, mant | 0x800000)
    ee = np.maximum(e, 1)
    E = ee.max(axis=-1, keepdims=True)
    sh = E - ee
    v0 = m << 11
    v = np.where(sh < 63, v0 >> np.minimum(sh, 62), 0)
    inexact = (m != 0) & ((sh >= 63) | ((v << np.minimum(sh, 62)) != v0))
    sv = np.where(sign == 1, -v, v)
    digs = [sv >> 28] + [(sv >> (7 * (4 - t))) & 127 for t in range(1, 5)]
    kdig = np.stack(digs, axis=-2).astype(np.int8)   # [..., 5, d]
    kexp = (E[..., 0] | (inexact.sum(axis=-1) << 8)).astype(np.int32)
    return kdig, kexp


def check_norm_field(kexp, k_pool, page_table, L_ctx, B):
    """The norm field (bits 16-31, bf16) of every Kexp word: at least the
    largest Euclidean norm of the block's key rows (fp64 on the host), and at
    most the documented quantity sqrt(sum over 16-byte column chunks of the
    largest sum of squares in the chunk) by more than bf16 rounding plus the
    stated fp32 allowance."""
    kexp = np.asarray(kexp)
    bits = ((kexp.astype(np.int64) >> 16) & 0xFFFF).astype(np.uint32) << 16
    bound = bits.view(np.float32).astype(np.float64)
    K = np.asarray(torch.as_tensor(k_pool).to(torch.float64))
    pt = np.asarray(page_table).astype(np.int64)
    batch, H_kv, n_blk = kexp.shape
    d = K.shape[-1]
    ept = 8 if torch.as_tensor(k_pool).dtype == torch.bfloat16 else 4
    for b in range(batch):
        for g in range(H_kv):
            for j in range(n_blk):
                n = min(B, L_ctx - j * B)
                rows = K[pt[b, j], g, :n]
                true = np.sqrt((rows ** 2).sum(axis=1)).max()
                chunk = (rows ** 2).reshape(n, d // ept, ept).sum(axis=2).max(axis=0).sum()
                assert bound[b, g, j] >= true, (b, g, j)
                assert bound[b, g, j] <= np.sqrt(chunk) * (1 + 2 ** -6), (b, g, j)
