"""ctypes binding of the C ABI declared in include/dl.h.

Argument marshalling only: each function has the C entry point's name and
arguments, takes torch tensors for the device buffers (their data pointers
are passed through) and the current torch CUDA stream unless one is given.
Every step runs in the library's CUDA kernels; there is no other code path.
A failing call raises DLError with the library's message.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libdlsparse.so")

DL_OK, DL_ERR_INVALID_ARG, DL_ERR_UNSUPPORTED, DL_ERR_WORKSPACE = 0, 1, 2, 3
DL_ERR_CUDA, DL_ERR_BAD_INDEX, DL_ERR_TIMEOUT = 4, 5, 6
DL_BF16, DL_FP32 = 0, 1
DL_FLAG_TOKEN_SIMT, DL_FLAG_GATHER_SIMT, DL_FLAG_PDL, DL_FLAG_SCORE_FP64 = 1, 2, 4, 8
STATUS_NAMES = {0: "DL_OK", 1: "DL_ERR_INVALID_ARG", 2: "DL_ERR_UNSUPPORTED",
                3: "DL_ERR_WORKSPACE", 4: "DL_ERR_CUDA", 5: "DL_ERR_BAD_INDEX",
                6: "DL_ERR_TIMEOUT"}


class DLError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class dl_attn_desc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("batch", "H", "H_kv", "d", "L_ctx", "L_q", "page", "n_pages", "n_slots",
                 "dtype")]


_c_int, _vp, _i32p = ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p
_SIGS = {
    "dl_version": ([], ctypes.c_int),
    "dl_set_kernel_flags": ([ctypes.c_uint], ctypes.c_uint),
    "dl_last_error_message": ([], ctypes.c_char_p),
    "dl_get_status": ([_vp], _c_int),
    "dl_workspace_size": ([ctypes.POINTER(dl_attn_desc), ctypes.POINTER(ctypes.c_size_t)], _c_int),
    "dl_predict_queries": ([_vp, _vp, _c_int, _c_int, _c_int, _c_int, _vp, _vp, _vp], _c_int),
    "dl_pool_keys": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _c_int, _c_int, _c_int, _c_int,
                      _vp, _vp, _vp, _vp], _c_int),
    "dl_cache_write": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _c_int, _vp, _vp, _vp, _vp, _vp,
                        _vp, _vp, _vp], _c_int),
    "dl_block_scores": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _c_int, _vp, _vp,
                         ctypes.c_size_t, _vp], _c_int),
    "dl_find_sinks": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                       _vp, _vp, ctypes.c_size_t, _vp], _c_int),
    "dl_select": ([_vp, _c_int, _c_int, _c_int, _c_int, _c_int, _vp, _c_int, _vp, _vp, _c_int,
                   _vp], _c_int),
    "dl_sink_mass": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                      ctypes.c_size_t, _vp], _c_int),
    "dl_sink_topn": ([_vp, _c_int, _c_int, _c_int, _vp, _vp], _c_int),
    "dl_block_select": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _vp, _vp, _c_int,
                         _c_int, _c_int, _vp, _c_int, _vp, _vp, _vp, _c_int, _c_int, _vp,
                         ctypes.c_size_t, _vp], _c_int),
    "dl_read_counters": ([_vp, _vp], _c_int),
    "dl_sparse_attn": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _vp, _vp, _c_int, _vp,
                        _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp], _c_int),
    "dl_token_select": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _c_int, _c_int,
                         _c_int, _c_int, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp], _c_int),
    "dl_block_scores_noalloc": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _c_int, _vp,
                                 _vp], _c_int),
    "dl_sparse_attn_gather": ([ctypes.POINTER(dl_attn_desc), _vp, _vp, _vp, _vp, _vp, _vp,
                               _c_int, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp], _c_int),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m long_context_diffusion_b200.build`"
            " (the library has no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (args, res) in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    return lib


lib = _load()


def _check(status: int):
    if status != DL_OK:
        raise DLError(status, lib.dl_last_error_message().decode(errors="replace"))


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to the library must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_desc(batch, H, H_kv, d, L_ctx, L_q, page, n_pages, n_slots, dtype) -> dl_attn_desc:
    if isinstance(dtype, torch.dtype):
        dtype = DL_BF16 if dtype == torch.bfloat16 else DL_FP32
    return dl_attn_desc(batch, H, H_kv, d, L_ctx, L_q, page, n_pages, n_slots, dtype)


def dl_version() -> int:
    return lib.dl_version()


def dl_set_kernel_flags(flags: int) -> int:
    """Kernel-choice switches for the tests (DL_FLAG_*); returns the previous
    flags."""
    return int(lib.dl_set_kernel_flags(int(flags)))


def dl_get_status(stream=None) -> int:
    """Synchronises the stream; returns the status (does not raise)."""
    return lib.dl_get_status(_s(stream))


def dl_workspace_size(desc: dl_attn_desc) -> int:
    n = ctypes.c_size_t(0)
    _check(lib.dl_workspace_size(ctypes.byref(desc), ctypes.byref(n)))
    return int(n.value)


def dl_predict_queries(conf_prev, still_masked, k, w, q_idx, q_cnt, stream=None):
    batch, L_q = conf_prev.shape
    _check(lib.dl_predict_queries(_p(conf_prev), _p(still_masked), batch, L_q, k, w, _p(q_idx),
                                  _p(q_cnt), _s(stream)))


def dl_pool_keys(desc, K_pool, page_table, n_units, unit_stride, unit_offset, unit_len, Kbar,
                 stream=None, Kdig=None, Kexp=None):
    _check(lib.dl_pool_keys(ctypes.byref(desc), _p(K_pool), _p(page_table), n_units, unit_stride,
                            unit_offset, unit_len, _p(Kbar), _p(Kdig), _p(Kexp), _s(stream)))


def dl_cache_write(desc, K_new, V_new, start, page_table, K_pool, V_pool, Kbar, stream=None,
                   Kdig=None, Kexp=None):
    _check(lib.dl_cache_write(ctypes.byref(desc), _p(K_new), _p(V_new), K_new.shape[-2],
                              _p(start), _p(page_table), _p(K_pool), _p(V_pool), _p(Kbar),
                              _p(Kdig), _p(Kexp), _s(stream)))


def key_digit_buffers(batch, H_kv, n_units, d, device):
    """Allocates the Kdig / Kexp buffers of dl_pool_keys' digit output."""
    return (torch.empty((batch, H_kv, 5, n_units, d), dtype=torch.int8, device=device),
            torch.empty((batch, H_kv, n_units), dtype=torch.int32, device=device))


def dl_read_counters():
    """(fast, fallback) selections of dl_block_select's int8 kernel since the
    last read."""
    f, b = ctypes.c_ulonglong(0), ctypes.c_ulonglong(0)
    _check(lib.dl_read_counters(ctypes.byref(f), ctypes.byref(b)))
    return int(f.value), int(b.value)


def dl_block_scores(desc, Q_dec, q_idx, q_cnt, Kbar, n_units, score, ws, stream=None):
    _check(lib.dl_block_scores(ctypes.byref(desc), _p(Q_dec), _p(q_idx), _p(q_cnt), _p(Kbar),
                               n_units, _p(score), _p(ws), ws.numel() * ws.element_size(),
                               _s(stream)))


def dl_find_sinks(desc, Q_dec, q_idx, q_cnt, K_pool, page_table, K_dec, n_sinks, sink_pos, ws,
                  stream=None, Kexp=None):
    """Kexp: the layer's key exponent words (key_digit_buffers, filled by
    dl_pool_keys / dl_cache_write); given, the sink cut is certified."""
    _check(lib.dl_find_sinks(ctypes.byref(desc), _p(Q_dec), _p(q_idx), _p(q_cnt), _p(K_pool),
                             _p(page_table), _p(K_dec), _p(Kexp), n_sinks, _p(sink_pos), _p(ws),
                             ws.numel() * ws.element_size(), _s(stream)))


def dl_sink_mass(desc, Q_dec, q_idx, q_cnt, K_pool, page_table, K_dec, mass, ws, stream=None):
    """This shard's part of the sink mass, mass fp32 [batch][L_ctx]."""
    _check(lib.dl_sink_mass(ctypes.byref(desc), _p(Q_dec), _p(q_idx), _p(q_cnt), _p(K_pool),
                            _p(page_table), _p(K_dec), _p(mass), _p(ws),
                            ws.numel() * ws.element_size(), _s(stream)))


def dl_sink_topn(mass, sink_pos, stream=None):
    """sink_pos [batch][n_sinks] from the summed mass [batch][L_ctx]."""
    batch, L_ctx = mass.shape
    _check(lib.dl_sink_topn(_p(mass), batch, L_ctx, sink_pos.shape[-1], _p(sink_pos),
                            _s(stream)))


def dl_select(score, unit_size, topK, sink_pos, blk_idx, blk_cnt, stream=None):
    batch, H_kv, n_units = score.shape
    n_sinks = 0 if sink_pos is None else sink_pos.shape[-1]
    _check(lib.dl_select(_p(score), batch, H_kv, n_units, unit_size, topK, _p(sink_pos), n_sinks,
                         _p(blk_idx), _p(blk_cnt), blk_idx.shape[-1], _s(stream)))


def dl_block_select(desc, Q_dec, q_idx, q_cnt, Kbar, n_units, unit_size, topK, sink_pos, score,
                    blk_idx, blk_cnt, ws, stream=None, max_q=0, Kdig=None, Kexp=None):
    n_sinks = 0 if sink_pos is None else sink_pos.shape[-1]
    _check(lib.dl_block_select(ctypes.byref(desc), _p(Q_dec), _p(q_idx), _p(q_cnt), _p(Kbar),
                               _p(Kdig), _p(Kexp), n_units, unit_size, topK, _p(sink_pos),
                               n_sinks, _p(score),
                               _p(blk_idx), _p(blk_cnt), blk_idx.shape[-1], max_q, _p(ws),
                               ws.numel() * ws.element_size(), _s(stream)))


def dl_sparse_attn(desc, Q_dec, K_pool, V_pool, page_table, blk_idx, blk_cnt, K_dec, V_dec, O,
                   lse, ws, stream=None):
    max_sel = 0 if blk_idx is None else blk_idx.shape[-1]
    _check(lib.dl_sparse_attn(ctypes.byref(desc), _p(Q_dec), _p(K_pool), _p(V_pool),
                              _p(page_table), _p(blk_idx), _p(blk_cnt), max_sel, _p(K_dec),
                              _p(V_dec), _p(O), _p(lse), _p(ws), ws.numel() * ws.element_size(),
                              _s(stream)))


def dl_token_select(desc, Q_dec, K_pool, page_table, chunk_idx, chunk_stride, chunk_content, topT,
                    tok_pos, tok_cnt, ws=None, stream=None, Kexp=None):
    """Kexp: the chunk keys' exponent words (dl_pool_keys over the chunks);
    given, the top-T cut is certified."""
    n_sel = chunk_idx.shape[-1]
    wsz = 0 if ws is None else ws.numel() * ws.element_size()
    _check(lib.dl_token_select(ctypes.byref(desc), _p(Q_dec), _p(K_pool), _p(page_table),
                               _p(chunk_idx), n_sel, chunk_stride, chunk_content, topT, _p(Kexp),
                               _p(tok_pos), _p(tok_cnt), _p(ws), wsz, _s(stream)))


def dl_sparse_attn_gather(desc, Q_dec, K_pool, V_pool, page_table, tok_pos, tok_cnt, K_dec, V_dec,
                          O, lse, ws, stream=None):
    _check(lib.dl_sparse_attn_gather(ctypes.byref(desc), _p(Q_dec), _p(K_pool), _p(V_pool),
                                     _p(page_table), _p(tok_pos), _p(tok_cnt), tok_pos.shape[-1],
                                     _p(K_dec), _p(V_dec), _p(O), _p(lse), _p(ws),
                                     ws.numel() * ws.element_size(), _s(stream)))


def dl_block_scores_noalloc(desc, Q_dec, q_idx, q_cnt, Kbar, n_units, score, stream=None):
    """dl_block_scores without a workspace: for callers that cannot allocate
    device memory; the library's built-in 32 MiB scratch array is used."""
    _check(lib.dl_block_scores_noalloc(ctypes.byref(desc), _p(Q_dec), _p(q_idx), _p(q_cnt),
                                       _p(Kbar), n_units, _p(score), _s(stream)))
