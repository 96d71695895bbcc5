"""Thin ctypes binding of libcskv.so (include/cskv.h).

Argument marshalling only: torch tensors are checked for dtype, shape,
device and contiguity, then passed as raw device pointers with the current
CUDA stream. Every step of the computation runs in the library's kernels;
there is no fallback: if the library is missing, importing the entry points
raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass, field
from typing import Optional

import torch

from .build import LIB

# ------------------------------------------------------------- constants
OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4
ERR_TIMEOUT = -5
ERR_OUT_OF_RANGE = -6

BF16, F32, FP8_E4M3, FP4_E2M1 = 0, 1, 2, 3
LAYER_CSA, LAYER_HCA = 0, 1


class CskvError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__("%s failed: %s (%d)" % (where, status_string(code), code))
        self.code = code


# ------------------------------------------------------------- structs
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64


class LayerStruct(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("kind", _I32), ("m", _I32), ("n_win", _I32),
        ("d_qk", _I32), ("d_v", _I32), ("d_idx", _I32), ("page_size", _I32),
        ("kv_dtype", _I32), ("idx_dtype", _I32), ("gate_cols", _I32), ("gate_cols_idx", _I32),
        ("n_seqs", _I32), ("max_pages_per_seq", _I32), ("n_pages", _I64),
        ("page_table", _P), ("kv_pool", _P), ("kv_scale", _P), ("idx_pool", _P), ("idx_scale", _P),
        ("ring_x", _P), ("ring_z", _P), ("ring_xi", _P), ("ring_zi", _P),
        ("pos_bias", _P), ("pos_bias_idx", _P), ("overlap", _I32),
    ]


class CompressArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("layer", ctypes.POINTER(LayerStruct)), ("n_seq", _I32),
        ("seq_ids", _P), ("tok0", _I64), ("n_tok", _I64), ("x", _P), ("z", _P), ("xi", _P), ("zi", _P),
        ("d_status", _P),
    ]


class AppendArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("layer", ctypes.POINTER(LayerStruct)), ("n_seq", _I32),
        ("n_new", _I32), ("seq_ids", _P), ("pos", _P), ("x", _P), ("z", _P), ("xi", _P), ("zi", _P),
        ("ring_only", _I32), ("d_status", _P), ("emit_only", _I32),
    ]


class IndexArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("layer", ctypes.POINTER(LayerStruct)), ("n_q", _I32),
        ("n_heads_idx", _I32), ("q_seq", _P), ("q_pos", _P), ("max_pos", _I64), ("q_idx", _P),
        ("q_idx_scale", _P), ("w", _P), ("k", _I32), ("out_idx", _P), ("out_cnt", _P),
        ("out_scores", _P), ("d_status", _P), ("score_bf16", _I32),
    ]


class AttendArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", ctypes.c_uint32), ("layer", ctypes.POINTER(LayerStruct)), ("n_q", _I32),
        ("n_heads", _I32), ("q_seq", _P), ("q_pos", _P), ("max_pos", _I64), ("q", _P),
        ("sel_idx", _P), ("sel_cnt", _P), ("k", _I32), ("sm_scale", ctypes.c_float), ("out", _P),
        ("lse", _P), ("x_chunk", _P), ("chunk_pos0", _I64), ("chunk_len", _I64), ("d_status", _P),
        ("rope_dims", _I32), ("rope_base", ctypes.c_float), ("chunk_desc", _P),
    ]


SYMBOLS = {
    "cskv_layer_bytes": (_I32, [ctypes.POINTER(LayerStruct)] + [ctypes.POINTER(ctypes.c_size_t)] * 8),
    "csa_compress_kv": (_I32, [ctypes.POINTER(CompressArgs), _P]),
    "hca_compress_kv": (_I32, [ctypes.POINTER(CompressArgs), _P]),
    "cskv_cache_append": (_I32, [ctypes.POINTER(AppendArgs), _P]),
    "csa_index_ws_bytes": (_I32, [ctypes.POINTER(IndexArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "csa_index_score_topk": (_I32, [ctypes.POINTER(IndexArgs), _P, ctypes.c_size_t, _P]),
    "csa_index_score_topk_static": (_I32, [ctypes.POINTER(IndexArgs), _P]),
    "cskv_attend_ws_bytes": (_I32, [ctypes.POINTER(AttendArgs), ctypes.POINTER(ctypes.c_size_t)]),
    "csa_attend": (_I32, [ctypes.POINTER(AttendArgs), _P, ctypes.c_size_t, _P]),
    "hca_attend": (_I32, [ctypes.POINTER(AttendArgs), _P, ctypes.c_size_t, _P]),
    "cskv_get_status": (_I32, [_P, _P, ctypes.POINTER(_I32)]),
    "cskv_selftest_wait": (_I32, [_I32, ctypes.c_uint32, _P, _P]),
    "cskv_status_string": (ctypes.c_char_p, [_I32]),
    "cskv_version": (_I32, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libcskv.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise ImportError("libcskv.so is not built (%s); run `python -m compressed_sparse_kv_02_b200.build`"
                              % LIB)
        L = ctypes.CDLL(LIB)
        for name, (res, args) in SYMBOLS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().cskv_status_string(int(code)).decode()


def _check(code: int, where: str):
    if code != OK:
        raise CskvError(code, where)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _need(t: Optional[torch.Tensor], name: str, dtype, shape=None, optional=False):
    if t is None:
        if optional:
            return
        raise ValueError("%s is required" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


# ------------------------------------------------------------- layer state
_TORCH_STORE = {BF16: torch.bfloat16, FP8_E4M3: torch.uint8, FP4_E2M1: torch.uint8}


@dataclass
class Layer:
    """One layer's caches: the paged compressed cache and the state-cache rings.

    All buffers are torch tensors owned by this object; `struct` is the
    cskv_layer view passed to the library.
    """
    kind: int
    m: int
    n_win: int
    d_qk: int
    d_v: int
    d_idx: int
    page_size: int
    kv_dtype: int
    idx_dtype: int
    gate_cols: int
    gate_cols_idx: int
    n_seqs: int
    max_pages_per_seq: int
    n_pages: int
    page_table: torch.Tensor = None
    kv_pool: torch.Tensor = None
    kv_scale: torch.Tensor = None
    idx_pool: torch.Tensor = None
    idx_scale: torch.Tensor = None
    ring_x: torch.Tensor = None
    ring_z: torch.Tensor = None
    ring_xi: torch.Tensor = None
    ring_zi: torch.Tensor = None
    pos_bias: torch.Tensor = None
    pos_bias_idx: torch.Tensor = None
    overlap: int = 0  # block overlap: an entry also folds the last `overlap` tokens of the block before it
    _struct: LayerStruct = field(default=None, repr=False)

    @property
    def is_csa(self) -> bool:
        return self.kind == LAYER_CSA

    def shape_struct(self) -> LayerStruct:
        s = LayerStruct()
        s.struct_size = ctypes.sizeof(LayerStruct)
        for f in ("kind", "m", "n_win", "d_qk", "d_v", "d_idx", "page_size", "kv_dtype", "idx_dtype",
                  "gate_cols", "gate_cols_idx", "n_seqs", "max_pages_per_seq", "n_pages", "overlap"):
            setattr(s, f, int(getattr(self, f)))
        return s

    def buffer_bytes(self) -> dict:
        sizes = [ctypes.c_size_t() for _ in range(8)]
        s = self.shape_struct()
        _check(lib().cskv_layer_bytes(ctypes.byref(s), *[ctypes.byref(v) for v in sizes]), "cskv_layer_bytes")
        names = ("kv_pool", "kv_scale", "idx_pool", "idx_scale", "ring_x", "ring_z", "ring_xi", "ring_zi")
        return {n: v.value for n, v in zip(names, sizes)}

    @classmethod
    def allocate(cls, kind: int, m: int, d_qk: int, d_v: int, n_seqs: int, n_pages: int,
                 max_pages_per_seq: int, page_size: int = 64, n_win: int = 128, d_idx: int = 0,
                 kv_dtype: int = BF16, idx_dtype: int = BF16, gate_cols: Optional[int] = None,
                 gate_cols_idx: Optional[int] = None, device="cuda", overlap: int = 0) -> "Layer":
        L = cls(kind=kind, m=m, n_win=n_win, d_qk=d_qk, d_v=d_v, d_idx=d_idx if kind == LAYER_CSA else 0,
                page_size=page_size, kv_dtype=kv_dtype, idx_dtype=idx_dtype if kind == LAYER_CSA else BF16,
                gate_cols=d_qk if gate_cols is None else gate_cols,
                gate_cols_idx=(d_idx if gate_cols_idx is None else gate_cols_idx) if kind == LAYER_CSA else 1,
                n_seqs=n_seqs, max_pages_per_seq=max_pages_per_seq, n_pages=n_pages, overlap=overlap)
        sz = L.buffer_bytes()
        rows = n_pages * page_size
        u8 = dict(dtype=torch.uint8, device=device)
        bf = dict(dtype=torch.bfloat16, device=device)
        L.page_table = torch.full((n_seqs, max_pages_per_seq), -1, dtype=torch.int32, device=device)
        if kv_dtype == BF16:
            L.kv_pool = torch.zeros(rows, d_qk, **bf)
        else:
            L.kv_pool = torch.zeros(rows, d_qk, **u8)
            L.kv_scale = torch.ones(rows, dtype=torch.float32, device=device)
        if L.is_csa:
            if L.idx_dtype == BF16:
                L.idx_pool = torch.zeros(rows, L.d_idx, **bf)
            else:
                L.idx_pool = torch.zeros(rows, L.d_idx // 2, **u8)
                L.idx_scale = torch.zeros(rows, L.d_idx // 16, **u8)
            L.ring_xi = torch.zeros(n_seqs, n_win, L.d_idx, **bf)
            L.ring_zi = torch.zeros(n_seqs, n_win, L.gate_cols_idx, **bf)
        L.ring_x = torch.zeros(n_seqs, n_win, d_qk, **bf)
        L.ring_z = torch.zeros(n_seqs, n_win, L.gate_cols, **bf)
        for name, want in sz.items():
            t = getattr(L, name)
            have = 0 if t is None else t.numel() * t.element_size()
            if have != want:
                raise RuntimeError("buffer %s: %d bytes allocated, library wants %d" % (name, have, want))
        return L

    # -------- paging helpers (storage layout only: which pool row holds entry j)
    def set_pages(self, seq: int, pages: torch.Tensor):
        """Give sequence `seq` the pool pages `pages` (int32) for its entries 0, P, 2P, ..."""
        self.page_table[seq, : pages.numel()] = pages.to(torch.int32).to(self.page_table.device)

    def rows_of(self, seq: int, j0: int, n: int) -> torch.Tensor:
        """Pool row ids (int64) of entries j0 .. j0+n-1 of sequence `seq`."""
        j = torch.arange(j0, j0 + n, device=self.page_table.device, dtype=torch.int64)
        page = self.page_table[seq].long()[j // self.page_size]
        if n and int(page.min()) < 0:
            raise ValueError("entries %d..%d of sequence %d have no page" % (j0, j0 + n - 1, seq))
        return page * self.page_size + j % self.page_size

    def write_entries(self, seq: int, j0: int, kv=None, kv_scale=None, idx=None, idx_scale=None):
        """Store already-encoded entries (rows in the pool's dtype) at entries j0.. of `seq`."""
        n = next(t.shape[0] for t in (kv, idx) if t is not None)
        rows = self.rows_of(seq, j0, n)
        if kv is not None:
            self.kv_pool[rows] = kv.to(self.kv_pool.dtype)
        if kv_scale is not None:
            self.kv_scale[rows] = kv_scale.float()
        if idx is not None:
            self.idx_pool[rows] = idx.to(self.idx_pool.dtype)
        if idx_scale is not None:
            self.idx_scale[rows] = idx_scale
        return rows

    def read_entries(self, seq: int, n: int, j0: int = 0) -> dict:
        """Stored rows (and scales) of entries j0 .. j0+n-1 of `seq`, in entry order."""
        rows = self.rows_of(seq, j0, n)
        out = {"kv": self.kv_pool[rows]}
        if self.kv_scale is not None:
            out["kv_scale"] = self.kv_scale[rows]
        if self.is_csa:
            out["idx"] = self.idx_pool[rows]
            if self.idx_scale is not None:
                out["idx_scale"] = self.idx_scale[rows]
        return out

    @property
    def struct(self) -> LayerStruct:
        s = self.shape_struct()
        for f in ("page_table", "kv_pool", "kv_scale", "idx_pool", "idx_scale", "ring_x", "ring_z",
                  "ring_xi", "ring_zi", "pos_bias", "pos_bias_idx"):
            t = getattr(self, f)
            setattr(s, f, None if t is None else t.data_ptr())
        self._struct = s  # keep alive while the call runs
        return s


# ------------------------------------------------------------- entry points
def _compress(fn, where, layer: Layer, seq_ids, tok0, x, z, xi=None, zi=None, status=None, stream=None):
    n_seq, n_tok = x.shape[0], x.shape[1]
    _need(seq_ids, "seq_ids", torch.int32, (n_seq,))
    _need(x, "x", torch.bfloat16, (n_seq, n_tok, layer.d_qk))
    _need(z, "z", torch.bfloat16, (n_seq, n_tok, layer.gate_cols))
    if layer.is_csa:
        _need(xi, "xi", torch.bfloat16, (n_seq, n_tok, layer.d_idx))
        _need(zi, "zi", torch.bfloat16, (n_seq, n_tok, layer.gate_cols_idx))
    _need(status, "status", torch.int32, optional=True)
    a = CompressArgs(ctypes.sizeof(CompressArgs), ctypes.pointer(layer.struct), n_seq, _ptr(seq_ids), int(tok0),
                     n_tok, _ptr(x), _ptr(z), _ptr(xi), _ptr(zi), _ptr(status))
    _check(fn(ctypes.byref(a), _stream(stream)), where)


def csa_compress_kv(layer: Layer, seq_ids, tok0: int, x, z, xi, zi, status=None, stream=None):
    """Fold raw tokens tok0 .. tok0+n_tok-1 of each sequence into the CSA cache (KV and indexer keys)."""
    if not layer.is_csa:
        raise ValueError("csa_compress_kv needs a CSA layer")
    _compress(lib().csa_compress_kv, "csa_compress_kv", layer, seq_ids, tok0, x, z, xi, zi, status, stream)


def hca_compress_kv(layer: Layer, seq_ids, tok0: int, x, z, status=None, stream=None):
    """Fold raw tokens tok0 .. tok0+n_tok-1 of each sequence into the HCA cache."""
    if layer.is_csa:
        raise ValueError("hca_compress_kv needs an HCA layer")
    _compress(lib().hca_compress_kv, "hca_compress_kv", layer, seq_ids, tok0, x, z, None, None, status, stream)


def cskv_cache_append(layer: Layer, seq_ids, pos, x, z, xi=None, zi=None, ring_only=False, status=None,
                      stream=None, emit_only=False):
    """Append n_new tokens per sequence to the state-cache rings; fold completed blocks into the cache
    (ring_only: the rings only; emit_only: the completed blocks only, the rings holding the tokens already)."""
    n_seq, n_new = x.shape[0], x.shape[1]
    _need(seq_ids, "seq_ids", torch.int32, (n_seq,))
    _need(pos, "pos", torch.int64, (n_seq,))
    _need(x, "x", torch.bfloat16, (n_seq, n_new, layer.d_qk))
    _need(z, "z", torch.bfloat16, (n_seq, n_new, layer.gate_cols))
    if layer.is_csa:
        _need(xi, "xi", torch.bfloat16, (n_seq, n_new, layer.d_idx))
        _need(zi, "zi", torch.bfloat16, (n_seq, n_new, layer.gate_cols_idx))
    _need(status, "status", torch.int32, optional=True)
    a = AppendArgs(ctypes.sizeof(AppendArgs), ctypes.pointer(layer.struct), n_seq, n_new, _ptr(seq_ids), _ptr(pos),
                   _ptr(x), _ptr(z), _ptr(xi), _ptr(zi), int(bool(ring_only)), _ptr(status), int(bool(emit_only)))
    _check(lib().cskv_cache_append(ctypes.byref(a), _stream(stream)), "cskv_cache_append")


def _index_args(layer, q_seq, q_pos, max_pos, q_idx, w, k, out_idx, out_cnt, out_scores, q_idx_scale, status,
                score_bf16=False):
    n_q, h_i = w.shape
    return IndexArgs(ctypes.sizeof(IndexArgs), ctypes.pointer(layer.struct), n_q, h_i, _ptr(q_seq), _ptr(q_pos),
                     int(max_pos), _ptr(q_idx), _ptr(q_idx_scale), _ptr(w), int(k), _ptr(out_idx), _ptr(out_cnt),
                     _ptr(out_scores), _ptr(status), 1 if score_bf16 else 0)


def csa_index_ws_bytes(layer: Layer, n_q: int, n_heads_idx: int, max_pos: int, k: int) -> int:
    a = IndexArgs(ctypes.sizeof(IndexArgs), ctypes.pointer(layer.struct), n_q, n_heads_idx, None, None,
                  int(max_pos), None, None, None, int(k), None, None, None, None)
    n = ctypes.c_size_t()
    _check(lib().csa_index_ws_bytes(ctypes.byref(a), ctypes.byref(n)), "csa_index_ws_bytes")
    return n.value


def csa_index_score_topk(layer: Layer, q_seq, q_pos, max_pos: int, q_idx, w, k: int, out_idx, out_cnt,
                         out_scores=None, q_idx_scale=None, workspace=None, status=None, stream=None,
                         score_bf16=False):
    """Indexer scores of every visible CSA entry and the ascending top-k ids per query (score_bf16: select
    on the scores rounded to bf16)."""
    if not layer.is_csa:
        raise ValueError("csa_index_score_topk needs a CSA layer")
    _need(w, "w", torch.float32)
    n_q, h_i = w.shape
    _need(q_seq, "q_seq", torch.int32, (n_q,))
    _need(q_pos, "q_pos", torch.int64, (n_q,))
    if layer.idx_dtype == BF16:
        _need(q_idx, "q_idx", torch.bfloat16, (n_q, h_i, layer.d_idx))
    else:
        _need(q_idx, "q_idx", torch.uint8, (n_q, h_i, layer.d_idx // 2))
        _need(q_idx_scale, "q_idx_scale", torch.uint8, (n_q, h_i, layer.d_idx // 16))
    _need(out_idx, "out_idx", torch.int32, (n_q, k))
    _need(out_cnt, "out_cnt", torch.int32, (n_q,))
    _need(out_scores, "out_scores", torch.float32, (n_q, k), optional=True)
    _need(status, "status", torch.int32, optional=True)
    if workspace is None:
        workspace = torch.empty(csa_index_ws_bytes(layer, n_q, h_i, max_pos, k), dtype=torch.uint8,
                                device=w.device)
    a = _index_args(layer, q_seq, q_pos, max_pos, q_idx, w, k, out_idx, out_cnt, out_scores, q_idx_scale, status,
                    score_bf16)
    _check(lib().csa_index_score_topk(ctypes.byref(a), _ptr(workspace), workspace.numel(), _stream(stream)),
           "csa_index_score_topk")


def csa_index_score_topk_static(layer: Layer, q_seq, q_pos, max_pos: int, q_idx, w, k: int, out_idx, out_cnt,
                                out_scores=None, q_idx_scale=None, status=None, stream=None):
    """csa_index_score_topk without a workspace: the library's fixed device scratch is used instead.

    For callers that cannot allocate device memory where they call the indexer; the scratch
    holds CSKV_STATIC_INDEX_SCRATCH_FLOATS scores, is shared by every call (overlapping calls
    race), and is set up by the first call on each device, which should precede any stream capture.
    """
    if not layer.is_csa:
        raise ValueError("csa_index_score_topk_static needs a CSA layer")
    _need(w, "w", torch.float32)
    n_q, h_i = w.shape
    _need(q_seq, "q_seq", torch.int32, (n_q,))
    _need(q_pos, "q_pos", torch.int64, (n_q,))
    _need(out_idx, "out_idx", torch.int32, (n_q, k))
    _need(out_cnt, "out_cnt", torch.int32, (n_q,))
    _need(out_scores, "out_scores", torch.float32, (n_q, k), optional=True)
    a = _index_args(layer, q_seq, q_pos, max_pos, q_idx, w, k, out_idx, out_cnt, out_scores, q_idx_scale, status)
    _check(lib().csa_index_score_topk_static(ctypes.byref(a), _stream(stream)), "csa_index_score_topk_static")


def _attend_args(layer, q_seq, q_pos, max_pos, q, sel_idx, sel_cnt, k, sm_scale, out, lse, x_chunk, chunk_pos0,
                 status, n_q=None, n_heads=None, rope_dims=0, rope_base=10000.0, chunk_desc=None):
    if q is not None:
        n_q, n_heads = q.shape[0], q.shape[1]
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(layer.d_qk)
    return AttendArgs(ctypes.sizeof(AttendArgs), ctypes.pointer(layer.struct), n_q, n_heads, _ptr(q_seq),
                      _ptr(q_pos), int(max_pos), _ptr(q), _ptr(sel_idx), _ptr(sel_cnt), int(k), float(sm_scale),
                      _ptr(out), _ptr(lse), _ptr(x_chunk), int(chunk_pos0),
                      0 if x_chunk is None else int(x_chunk.shape[0]), _ptr(status), int(rope_dims),
                      float(rope_base), _ptr(chunk_desc))


def cskv_attend_ws_bytes(layer: Layer, n_q: int, n_heads: int, max_pos: int, k: int = 0) -> int:
    a = _attend_args(layer, None, None, max_pos, None, None, None, k, None, None, None, None, 0, None, n_q, n_heads)
    n = ctypes.c_size_t()
    _check(lib().cskv_attend_ws_bytes(ctypes.byref(a), ctypes.byref(n)), "cskv_attend_ws_bytes")
    return n.value


def _attend(fn, where, layer, q_seq, q_pos, max_pos, q, sel_idx, sel_cnt, k, out, lse, sm_scale, workspace,
            x_chunk, chunk_pos0, status, stream, rope_dims=0, rope_base=10000.0):
    n_q, n_heads = q.shape[0], q.shape[1]
    _need(q_seq, "q_seq", torch.int32, (n_q,))
    _need(q_pos, "q_pos", torch.int64, (n_q,))
    _need(q, "q", torch.bfloat16, (n_q, n_heads, layer.d_qk))
    _need(out, "out", torch.bfloat16, (n_q, n_heads, layer.d_v))
    _need(lse, "lse", torch.float32, (n_q, n_heads), optional=True)
    _need(x_chunk, "x_chunk", torch.bfloat16, optional=True)
    _need(status, "status", torch.int32, optional=True)
    if workspace is None:
        workspace = torch.empty(cskv_attend_ws_bytes(layer, n_q, n_heads, max_pos, k), dtype=torch.uint8,
                                device=q.device)
    a = _attend_args(layer, q_seq, q_pos, max_pos, q, sel_idx, sel_cnt, k, sm_scale, out, lse, x_chunk, chunk_pos0,
                     status, rope_dims=rope_dims, rope_base=rope_base)
    _check(fn(ctypes.byref(a), _ptr(workspace), workspace.numel(), _stream(stream)), where)


def csa_attend(layer: Layer, q_seq, q_pos, max_pos: int, q, sel_idx, sel_cnt, out, lse=None, sm_scale=None,
               workspace=None, x_chunk=None, chunk_pos0: int = 0, status=None, stream=None, rope_dims: int = 0,
               rope_base: float = 10000.0):
    """One softmax over the window and the selected CSA entries, every head sharing the latent KV
    (rope_dims > 0: inverse RoPE on the output's last rope_dims channels at each query's position)."""
    if not layer.is_csa:
        raise ValueError("csa_attend needs a CSA layer")
    k = sel_idx.shape[1]
    _need(sel_idx, "sel_idx", torch.int32, (q.shape[0], k))
    _need(sel_cnt, "sel_cnt", torch.int32, (q.shape[0],))
    _attend(lib().csa_attend, "csa_attend", layer, q_seq, q_pos, max_pos, q, sel_idx, sel_cnt, k, out, lse,
            sm_scale, workspace, x_chunk, chunk_pos0, status, stream, rope_dims, rope_base)


def hca_attend(layer: Layer, q_seq, q_pos, max_pos: int, q, out, lse=None, sm_scale=None, workspace=None,
               x_chunk=None, chunk_pos0: int = 0, status=None, stream=None, rope_dims: int = 0,
               rope_base: float = 10000.0):
    """One softmax over the window and every visible HCA entry (rope_dims > 0: inverse RoPE on the
    output's last rope_dims channels at each query's position)."""
    if layer.is_csa:
        raise ValueError("hca_attend needs an HCA layer")
    _attend(lib().hca_attend, "hca_attend", layer, q_seq, q_pos, max_pos, q, None, None, 0, out, lse, sm_scale,
            workspace, x_chunk, chunk_pos0, status, stream, rope_dims, rope_base)


def cskv_get_status(status: torch.Tensor, stream=None) -> int:
    """Read and clear a device status word (synchronises the stream)."""
    _need(status, "status", torch.int32)
    h = ctypes.c_int32()
    _check(lib().cskv_get_status(_ptr(status), _stream(stream), ctypes.byref(h)), "cskv_get_status")
    return h.value


def cskv_selftest_wait(arrive: bool, spin_limit: int, status: torch.Tensor, stream=None):
    """Launch the library's bounded-wait check: one warp waits on an mbarrier for at most spin_limit
    polls; with arrive=False nothing arrives and the wait reports CSKV_ERR_TIMEOUT in `status`."""
    _need(status, "status", torch.int32)
    _check(lib().cskv_selftest_wait(1 if arrive else 0, int(spin_limit), _ptr(status), _stream(stream)),
           "cskv_selftest_wait")


def cskv_version() -> int:
    return lib().cskv_version()
