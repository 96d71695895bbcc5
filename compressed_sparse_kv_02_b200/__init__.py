"""CSA / HCA hybrid compressed attention on NVIDIA B200 (sm_100a).

The hot path -- KV compression, the state-cache append, the Lightning-indexer
scores with top-k selection, and CSA / HCA attention -- runs in hand-written
CUDA kernels behind the C ABI of include/cskv.h (libcskv.so). This package is
the thin Python binding over that ABI; see `_binding` for the entry points.
"""
from ._binding import (  # noqa: F401
    BF16, F32, FP8_E4M3, FP4_E2M1, LAYER_CSA, LAYER_HCA,
    OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_OUT_OF_RANGE,
    SYMBOLS, CskvError, Layer, lib, status_string,
    csa_compress_kv, hca_compress_kv, cskv_cache_append,
    csa_index_ws_bytes, csa_index_score_topk, csa_index_score_topk_static,
    cskv_attend_ws_bytes, csa_attend, hca_attend,
    cskv_get_status, cskv_selftest_wait, cskv_version,
)
