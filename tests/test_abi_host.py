"""The C-ABI library on a host without a GPU: it loads, exports every entry
point include/dl.h declares, and rejects bad arguments before launching."""
import ctypes
import os
import re

import pytest

import long_context_diffusion_b200 as dl
from long_context_diffusion_b200 import _abi

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "dl.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dl_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_path():
    names = _declared()
    for n in ("dl_predict_queries", "dl_pool_keys", "dl_block_scores", "dl_find_sinks",
              "dl_select", "dl_block_select", "dl_sparse_attn", "dl_token_select",
              "dl_sparse_attn_gather", "dl_cache_write", "dl_workspace_size", "dl_get_status",
              "dl_sink_mass", "dl_sink_topn"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_abi.LIB_PATH)
    for n in _declared():
        assert hasattr(lib, n), n


def test_version():
    assert dl.dl_version() >= 100


def _desc(**kw):
    base = dict(batch=2, H=28, H_kv=4, d=128, L_ctx=16384, L_q=32, page=64, n_pages=256,
                n_slots=512, dtype=dl.DL_BF16)
    base.update(kw)
    return dl.make_desc(**base)


def test_workspace_size_and_validation():
    n = dl.dl_workspace_size(_desc())
    assert n > 0 and n % 256 == 0
    bad = [dict(d=96), dict(page=32), dict(H=30), dict(L_q=0), dict(L_q=300), dict(n_pages=10),
           dict(dtype=7), dict(batch=0)]
    for kw in bad:
        with pytest.raises(dl.DLError) as e:
            dl.dl_workspace_size(_desc(**kw))
        assert e.value.status in (dl.DL_ERR_INVALID_ARG, dl.DL_ERR_UNSUPPORTED), kw


def test_null_and_range_arguments_rejected_before_launch():
    lib = _abi.lib
    d = _desc()
    assert lib.dl_predict_queries(None, None, 1, 32, 4, 2, None, None, None) == dl.DL_ERR_INVALID_ARG
    fake = ctypes.c_void_p(0x1000)
    assert lib.dl_predict_queries(fake, fake, 1, 2000, 4, 2, fake, fake, None) == \
        dl.DL_ERR_INVALID_ARG
    assert lib.dl_select(None, 1, 1, 8, 64, 2, None, 0, fake, fake, 4, None) == \
        dl.DL_ERR_INVALID_ARG
    # max_sel too small for topK + sinks
    assert lib.dl_select(fake, 1, 1, 8, 64, 4, fake, 2, fake, fake, 5, None) == \
        dl.DL_ERR_INVALID_ARG
    assert "max_sel" in lib.dl_last_error_message().decode()
    # fused scores + selection: the same checks before any launch
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, None, None, None, 256, 64, 4,
                               None, 0, fake, fake, fake, 4, 0, fake, 1 << 40,
                               None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, fake, None, None, 256, 64, 4,
                               fake, 2, fake, fake, fake, 5, 0, fake, 1 << 40,
                               None) == dl.DL_ERR_INVALID_ARG
    assert "max_sel" in lib.dl_last_error_message().decode()
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, fake, None, None, 256, 64, 4,
                               None, 0, fake, fake, fake, 4, -1, fake, 1 << 40,
                               None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, fake, None, None, 256, 64, 4,
                               None, 0, fake, fake, fake, 4, 0, fake, 256,
                               None) == dl.DL_ERR_WORKSPACE
    # key digits: both or neither, 16-byte aligned
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, fake, fake, None, 256, 64, 4,
                               None, 0, fake, fake, fake, 4, 0, fake, 1 << 40,
                               None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_block_select(ctypes.byref(d), fake, None, None, fake, ctypes.c_void_p(0x1008),
                               fake, 256, 64, 4, None, 0, fake, fake, fake, 4, 0, fake, 1 << 40,
                               None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_pool_keys(ctypes.byref(d), fake, fake, 256, 64, 0, 64, fake, None, fake,
                            None) == dl.DL_ERR_INVALID_ARG
    assert "Kdig" in lib.dl_last_error_message().decode()
    # misaligned attention pointers
    odd = ctypes.c_void_p(0x1008)
    st = lib.dl_sparse_attn(ctypes.byref(d), odd, fake, fake, fake, None, None, 0, fake, fake,
                            fake, None, fake, 1 << 40, None)
    assert st == dl.DL_ERR_INVALID_ARG
    # workspace too small
    st = lib.dl_sparse_attn(ctypes.byref(d), fake, fake, fake, fake, None, None, 0, fake, fake,
                            fake, None, ctypes.c_void_p(0x10000), 256, None)
    assert st == dl.DL_ERR_WORKSPACE
    # unsupported token-select sizes
    st = lib.dl_token_select(ctypes.byref(d), fake, fake, fake, fake, 8, 1088, 2048, 256, None,
                             fake, fake, None, 0, None)
    assert st == dl.DL_ERR_INVALID_ARG



def test_split_sink_calls_rejected_before_launch():
    lib = _abi.lib
    d = _desc()
    fake = ctypes.c_void_p(0x1000)
    # the mass half: NULL mass, misaligned keys, workspace too small
    assert lib.dl_sink_mass(ctypes.byref(d), fake, fake, fake, fake, fake, fake, None, fake,
                            1 << 40, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_sink_mass(ctypes.byref(d), fake, fake, fake, ctypes.c_void_p(0x1008), fake,
                            fake, fake, fake, 1 << 40, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_sink_mass(ctypes.byref(d), fake, fake, fake, fake, fake, fake, fake, fake,
                            256, None) == dl.DL_ERR_WORKSPACE
    # the top-n half: sizes and pointers
    assert lib.dl_sink_topn(None, 1, 1024, 4, fake, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_sink_topn(fake, 1, 1024, 4, None, None) == dl.DL_ERR_INVALID_ARG
    for n_sinks in (0, 65):
        assert lib.dl_sink_topn(fake, 1, 1024, n_sinks, fake, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_sink_topn(fake, 0, 1024, 4, fake, None) == dl.DL_ERR_INVALID_ARG
    assert lib.dl_sink_topn(fake, 1, 0, 4, fake, None) == dl.DL_ERR_INVALID_ARG


def test_cache_write_arguments_rejected_before_launch():
    lib = _abi.lib
    d = _desc()
    fake = ctypes.c_void_p(0x1000)
    args = [fake, fake, 32, fake, fake, fake, fake, fake, None, None, None]
    assert lib.dl_cache_write(ctypes.byref(d), *args[:1], None, *args[2:]) == dl.DL_ERR_INVALID_ARG
    for n_new in (0, 16385):  # 1 .. L_ctx
        a = list(args)
        a[2] = n_new
        assert lib.dl_cache_write(ctypes.byref(d), *a) == dl.DL_ERR_INVALID_ARG
    a = list(args)
    a[0] = ctypes.c_void_p(0x1008)  # K_new off the 16-byte grid
    assert lib.dl_cache_write(ctypes.byref(d), *a) == dl.DL_ERR_INVALID_ARG
    assert "aligned" in lib.dl_last_error_message().decode()
    a = list(args)
    a[8] = fake  # Kdig without Kexp
    assert lib.dl_cache_write(ctypes.byref(d), *a) == dl.DL_ERR_INVALID_ARG


def test_kernel_flags_round_trip():
    prev = dl.dl_set_kernel_flags(dl.DL_FLAG_TOKEN_SIMT | dl.DL_FLAG_GATHER_SIMT)
    try:
        assert dl.dl_set_kernel_flags(0) == dl.DL_FLAG_TOKEN_SIMT | dl.DL_FLAG_GATHER_SIMT
        assert dl.dl_set_kernel_flags(0) == 0
    finally:
        dl.dl_set_kernel_flags(prev)


def test_read_counters_is_exported():
    lib = ctypes.CDLL(_abi.LIB_PATH)
    assert hasattr(lib, "dl_read_counters")
