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
