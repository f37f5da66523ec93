"""B200 (sm_100a) library for one denoising step of sink-aware,
query-predicted, block-sparse bidirectional attention over a cached
long-context KV (Focus-dLLM; chunked prefix as in Prefilling-dLLM).

The compute path is the C-ABI shared library lib/libdlsparse.so (CUDA
kernels); `_abi` binds its entry points by name, and `pipeline` sequences
them into a layer or a multi-layer step.  Importing fails if the library has
not been built: there is no other implementation to fall back to.
"""
from ._abi import (  # noqa: F401
    DLError, dl_attn_desc, make_desc, dl_version, dl_set_kernel_flags, dl_get_status, dl_workspace_size,
    dl_predict_queries, dl_pool_keys, dl_cache_write, dl_block_scores, dl_find_sinks, dl_sink_mass,
    dl_sink_topn, dl_select,
    dl_block_select, dl_read_counters, key_digit_buffers,
    dl_sparse_attn, dl_token_select, dl_sparse_attn_gather, dl_block_scores_noalloc, LIB_PATH,
    DL_OK, DL_ERR_INVALID_ARG, DL_ERR_UNSUPPORTED, DL_ERR_WORKSPACE, DL_ERR_CUDA,
    DL_ERR_BAD_INDEX, DL_ERR_TIMEOUT, DL_BF16, DL_FP32,
    DL_FLAG_TOKEN_SIMT, DL_FLAG_GATHER_SIMT, DL_FLAG_PDL, DL_FLAG_SCORE_FP64,
)
