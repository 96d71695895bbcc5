"""C-ABI checks that need no GPU: every symbol the header declares is exported,
buffer sizes, and host-side argument validation (which returns before any
CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "cskv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:cskv_status|const char\*|int32_t)\s+(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for want in ("csa_compress_kv", "hca_compress_kv", "cskv_cache_append", "csa_index_score_topk",
                 "csa_attend", "hca_attend", "cskv_get_status"):
        assert want in names


def test_library_exports_every_declared_symbol(cskv_built):
    lib = ctypes.CDLL(cskv_built)
    for name in _declared_functions():
        assert hasattr(lib, name), name
    import compressed_sparse_kv_02_b200 as ck
    assert set(ck.SYMBOLS) == set(_declared_functions())


def test_version_and_status_strings(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    assert ck.cskv_version() >= 100
    assert ck.status_string(ck.OK) == "ok"
    assert "out of range" in ck.status_string(ck.ERR_OUT_OF_RANGE)
    assert ck.status_string(12345) == "unknown status"


def _layer(**kw):
    import compressed_sparse_kv_02_b200 as ck
    base = dict(kind=ck.LAYER_CSA, m=4, n_win=128, d_qk=576, d_v=512, d_idx=128, page_size=64, kv_dtype=ck.BF16,
                idx_dtype=ck.BF16, gate_cols=576, gate_cols_idx=128, n_seqs=8, max_pages_per_seq=4096, n_pages=32768)
    base.update(kw)
    return ck.Layer(**base)


def test_layer_buffer_bytes(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    sz = _layer().buffer_bytes()
    rows = 32768 * 64
    assert sz["kv_pool"] == rows * 576 * 2 and sz["kv_scale"] == 0
    assert sz["idx_pool"] == rows * 128 * 2 and sz["idx_scale"] == 0
    assert sz["ring_x"] == 8 * 128 * 576 * 2 and sz["ring_zi"] == 8 * 128 * 128 * 2
    sz = _layer(kv_dtype=ck.FP8_E4M3, idx_dtype=ck.FP4_E2M1, gate_cols=1).buffer_bytes()
    assert sz["kv_pool"] == rows * 576 and sz["kv_scale"] == rows * 4
    assert sz["idx_pool"] == rows * 64 and sz["idx_scale"] == rows * 8
    assert sz["ring_z"] == 8 * 128 * 2
    sz = _layer(kind=ck.LAYER_HCA, m=128).buffer_bytes()
    assert sz["idx_pool"] == 0 and sz["ring_xi"] == 0


@pytest.mark.parametrize("bad", [dict(m=3), dict(m=256), dict(d_qk=100), dict(d_v=640), dict(page_size=24),
                                 dict(gate_cols=7), dict(kind=5), dict(d_idx=48), dict(n_pages=0)])
def test_layer_shape_rejected(cskv_built, bad):
    import compressed_sparse_kv_02_b200 as ck
    with pytest.raises(ck.CskvError) as e:
        _layer(**bad).buffer_bytes()
    assert e.value.code in (ck.ERR_INVALID_ARG, ck.ERR_UNSUPPORTED)


def test_unsupported_dtype_rejected(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    with pytest.raises(ck.CskvError) as e:
        _layer(kv_dtype=ck.FP4_E2M1).buffer_bytes()
    assert e.value.code == ck.ERR_UNSUPPORTED


def test_null_and_short_args_rejected_on_host(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    from compressed_sparse_kv_02_b200 import _binding as b
    L = ck.lib()
    assert L.csa_compress_kv(None, None) == ck.ERR_INVALID_ARG
    assert L.cskv_cache_append(None, None) == ck.ERR_INVALID_ARG
    assert L.csa_index_score_topk(None, None, 0, None) == ck.ERR_INVALID_ARG
    assert L.csa_attend(None, None, 0, None) == ck.ERR_INVALID_ARG
    assert L.hca_attend(None, None, 0, None) == ck.ERR_INVALID_ARG
    h = ctypes.c_int32()
    assert L.cskv_get_status(None, None, ctypes.byref(h)) == ck.ERR_INVALID_ARG
    layer = _layer()
    s = layer.struct  # pointers are null: shape checks pass, pointer checks fail
    a = b.CompressArgs(ctypes.sizeof(b.CompressArgs) - 8, ctypes.pointer(s), 1, None, 0, 4, None, None, None, None,
                       None)
    assert L.csa_compress_kv(ctypes.byref(a), None) == ck.ERR_INVALID_ARG  # struct_size too small
    a.struct_size = ctypes.sizeof(b.CompressArgs)
    assert L.csa_compress_kv(ctypes.byref(a), None) == ck.ERR_INVALID_ARG  # null pools
    assert L.hca_compress_kv(ctypes.byref(a), None) == ck.ERR_INVALID_ARG  # kind mismatch
    ia = b.IndexArgs(ctypes.sizeof(b.IndexArgs), ctypes.pointer(s), 4, 8, None, None, 1 << 20, None, None, None,
                     0, None, None, None, None)
    assert L.csa_index_score_topk(ctypes.byref(ia), None, 0, None) == ck.ERR_INVALID_ARG  # k = 0
    ia.k = 1024
    ia.n_heads_idx = 17
    assert L.csa_index_score_topk(ctypes.byref(ia), None, 0, None) == ck.ERR_INVALID_ARG


def test_workspace_queries_are_host_only(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    layer = _layer()
    n = ck.csa_index_ws_bytes(layer, n_q=8, n_heads_idx=8, max_pos=(1 << 20) - 1, k=1024)
    assert n >= 8 * 262112 * 4
    with pytest.raises(ck.CskvError):
        ck.csa_index_ws_bytes(layer, n_q=8, n_heads_idx=8, max_pos=-1, k=1024)


def test_wait_selftest_rejects_bad_arguments_on_host(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    L = ck.lib()
    assert L.cskv_selftest_wait(0, 1000, None, None) == ck.ERR_INVALID_ARG  # no status word
    st = ctypes.c_int32(0)  # never dereferenced: the limit check returns first
    assert L.cskv_selftest_wait(0, 0, ctypes.addressof(st), None) == ck.ERR_INVALID_ARG
