"""Plain fp64 CPU oracle for CSA / HCA hybrid compressed attention.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / reference leg of ``bench.py`` may import this package. It
shares no code with the GPU library (``compressed_sparse_kv_02_b200``) and
imports nothing from it; the arithmetic lives in ``cskv_oracle.c`` (plain C,
fp64) and this module only marshals numpy arrays into it.

Method sources (page title, section):
  * DeepSeek-V4 report digest (gitcode.csdn.net/69eb1ea0...), section 3:
    CSA folds every m tokens into one entry, a Lightning Indexer picks the
    top-k entries (k = 512 Flash, 1024 Pro); HCA folds every m' = 128 tokens
    and attends densely; both add the last n_win = 128 raw tokens.
  * DeepSeek-V4-book ch.1, section 4: m = 4, top-k = 1024 -> 4096 effective
    tokens, m' = 128 -> n/m' = 8K entries at 1M, dense HCA.
  * 10100.com DeepSeek-V4 article, sections 2.1-2.3 and 5.

Every function states the reading it follows where the pages are silent;
``cskv_oracle.c`` lists the readings in its header.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(closed forms, invariants, library routines, brute force); the
whole-method output has no printed worked example on the pages, so the
end-to-end numbers are pinned only through those invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cskv_oracle.c")
_LIB_DIR = os.path.join(_HERE, "build")
_LIB = os.path.join(_LIB_DIR, "libcskv_oracle.so")

# storage dtypes (must match cskv_oracle.c)
F64, F32, BF16, E4M3, E2M1 = 0, 1, 2, 3, 4


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(_LIB_DIR, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(tmp, _LIB)
    return _LIB


class _Mat(ctypes.Structure):
    _fields_ = [("dtype", ctypes.c_int32), ("pad_", ctypes.c_int32),
                ("data", ctypes.c_void_p), ("scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


_lib = None


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        D = ctypes.c_double
        MP = ctypes.POINTER(_Mat)
        sig = {
            "orc_bf16_to_f64": (D, [ctypes.c_uint16]),
            "orc_e4m3_to_f64": (D, [ctypes.c_uint8]),
            "orc_e2m1_to_f64": (D, [ctypes.c_uint8]),
            "orc_f32_to_bf16_bits": (ctypes.c_uint16, [ctypes.c_float]),
            "orc_f32_to_e4m3": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_f32_to_e2m1": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_mat_decode": (ctypes.c_int, [MP, P]),
            "orc_store_rows": (ctypes.c_int, [P, I64, I64, ctypes.c_int32, P, P]),
            "orc_compress": (ctypes.c_int, [MP, MP, P, I64, P]),
            "orc_compress_overlap": (ctypes.c_int, [MP, MP, P, I64, I64, P]),
            "orc_round_scores_bf16": (ctypes.c_int, [P, I64, P]),
            "orc_inverse_rope": (ctypes.c_int, [P, I64, I64, I64, I64, I64, D]),
            "orc_visible_entries": (I64, [I64, I64, I64]),
            "orc_window_start": (I64, [I64, I64]),
            "orc_index_scores": (ctypes.c_int, [MP, P, MP, I64, P]),
            "orc_topk": (I64, [P, I64, I64, P]),
            "orc_attend": (ctypes.c_int, [MP, MP, I64, D, P, P]),
            "orc_csa_query": (ctypes.c_int, [I64, I64, I64, I64, MP, MP, P, MP, MP, MP, I64, D,
                                             P, P, P, P]),
            "orc_hca_query": (ctypes.c_int, [I64, I64, I64, MP, MP, MP, I64, D, P, P]),
            "orc_num_threads": (ctypes.c_int, []),
            "orc_set_num_threads": (None, [ctypes.c_int]),
        }
        for name, (res, args) in sig.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


@dataclass
class Stored:
    """A matrix as it sits in memory: `rows` x `cols` elements of `dtype`.

    data:  F64 float64 / F32 float32 / BF16 uint16 / E4M3 uint8 [rows, cols];
           E2M1 uint8 [rows, cols // 2] (element 2i in the low nibble of byte i).
    scale: E4M3 float32 [rows]; E2M1 uint8 e4m3 codes [rows, cols // 16].
    """
    dtype: int
    data: np.ndarray
    rows: int
    cols: int
    scale: Optional[np.ndarray] = None

    def __post_init__(self):
        self.data = np.ascontiguousarray(self.data)
        if self.scale is not None:
            self.scale = np.ascontiguousarray(self.scale)
        want = {F64: np.float64, F32: np.float32, BF16: np.uint16, E4M3: np.uint8,
                E2M1: np.uint8}[self.dtype]
        if self.data.dtype != want:
            raise TypeError("data dtype %s does not match storage dtype %d" % (self.data.dtype, self.dtype))
        per_row = self.cols // 2 if self.dtype == E2M1 else self.cols
        if self.data.size != self.rows * per_row:
            raise ValueError("data size %d != %d x %d" % (self.data.size, self.rows, per_row))
        if self.dtype == E4M3 and (self.scale is None or self.scale.dtype != np.float32
                                   or self.scale.size != self.rows):
            raise ValueError("E4M3 needs one float32 scale per row")
        if self.dtype == E2M1 and (self.cols % 16 or self.scale is None or self.scale.dtype != np.uint8
                                   or self.scale.size != self.rows * self.cols // 16):
            raise ValueError("E2M1 needs one e4m3 scale byte per 16 elements")

    def mat(self) -> _Mat:
        return _Mat(self.dtype, 0, _ptr(self.data), _ptr(self.scale), self.rows, self.cols)

    def rows_subset(self, lo: int, hi: int) -> "Stored":
        """Rows lo..hi-1 (a view-like copy)."""
        per_row = self.cols // 2 if self.dtype == E2M1 else self.cols
        d = self.data.reshape(self.rows, per_row)[lo:hi]
        s = None
        if self.dtype == E4M3:
            s = self.scale.reshape(-1)[lo:hi]
        elif self.dtype == E2M1:
            s = self.scale.reshape(self.rows, self.cols // 16)[lo:hi]
        return Stored(self.dtype, d, hi - lo, self.cols, s)

    def take_rows(self, idx: np.ndarray) -> "Stored":
        """Rows at the given indices, in that order (used to undo paging)."""
        per_row = self.cols // 2 if self.dtype == E2M1 else self.cols
        d = self.data.reshape(self.rows, per_row)[idx]
        s = None
        if self.dtype == E4M3:
            s = self.scale.reshape(-1)[idx]
        elif self.dtype == E2M1:
            s = self.scale.reshape(self.rows, self.cols // 16)[idx]
        return Stored(self.dtype, d, len(idx), self.cols, s)


def f64(a: np.ndarray) -> Stored:
    a = np.ascontiguousarray(a, dtype=np.float64)
    if a.ndim == 1:
        a = a[None, :]
    return Stored(F64, a, a.shape[0], a.shape[1])


# ---------------------------------------------------------------- formats
def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    f = _L().orc_bf16_to_f64
    return np.array([f(int(b)) for b in np.asarray(bits, np.uint16).ravel()]).reshape(np.shape(bits))


def e4m3_to_f64(codes: np.ndarray) -> np.ndarray:
    f = _L().orc_e4m3_to_f64
    return np.array([f(int(b)) for b in np.asarray(codes, np.uint8).ravel()]).reshape(np.shape(codes))


def e2m1_to_f64(nibbles: np.ndarray) -> np.ndarray:
    f = _L().orc_e2m1_to_f64
    return np.array([f(int(b)) for b in np.asarray(nibbles, np.uint8).ravel()]).reshape(np.shape(nibbles))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    f = _L().orc_f32_to_bf16_bits
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint16).reshape(np.shape(x))


def f32_to_e4m3(x: np.ndarray) -> np.ndarray:
    f = _L().orc_f32_to_e4m3
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint8).reshape(np.shape(x))


def f32_to_e2m1(x: np.ndarray) -> np.ndarray:
    f = _L().orc_f32_to_e2m1
    return np.array([f(float(v)) for v in np.asarray(x, np.float32).ravel()],
                    dtype=np.uint8).reshape(np.shape(x))


def decode(s: Stored) -> np.ndarray:
    out = np.empty((s.rows, s.cols), np.float64)
    m = s.mat()
    rc = _L().orc_mat_decode(ctypes.byref(m), out.ctypes.data)
    if rc:
        raise ValueError("orc_mat_decode failed (%d)" % rc)
    return out


def store(values: np.ndarray, dtype: int) -> Stored:
    """Round fp64 rows to a storage dtype (BF16, F32, E4M3 + row scale, E2M1 + block scales)."""
    v = np.ascontiguousarray(values, np.float64)
    if v.ndim == 1:
        v = v[None, :]
    rows, cols = v.shape
    if dtype == BF16:
        data, scale = np.empty((rows, cols), np.uint16), None
    elif dtype == F32:
        data, scale = np.empty((rows, cols), np.float32), None
    elif dtype == E4M3:
        data, scale = np.empty((rows, cols), np.uint8), np.empty(rows, np.float32)
    elif dtype == E2M1:
        if cols % 16:
            raise ValueError("E2M1 rows must be a multiple of 16 wide")
        data, scale = np.empty((rows, cols // 2), np.uint8), np.empty((rows, cols // 16), np.uint8)
    else:
        raise ValueError("unsupported storage dtype %d" % dtype)
    rc = _L().orc_store_rows(v.ctypes.data, rows, cols, dtype, data.ctypes.data, _ptr(scale))
    if rc:
        raise ValueError("orc_store_rows failed (%d)" % rc)
    return Stored(dtype, data, rows, cols, scale)


# ---------------------------------------------------------------- method
def compress(x: Stored, z: Stored, m: int, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Softmax-gated fold of every m consecutive rows of x -> fp64 [n/m, d]."""
    if x.rows % m:
        raise ValueError("token count %d is not a multiple of m=%d" % (x.rows, m))
    out = np.empty((x.rows // m, x.cols), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float64).reshape(m, x.cols)
    xm, zm = x.mat(), z.mat()
    rc = _L().orc_compress(ctypes.byref(xm), ctypes.byref(zm), _ptr(b), m, out.ctypes.data)
    if rc:
        raise ValueError("orc_compress failed (%d)" % rc)
    return out


def compress_overlap(x: Stored, z: Stored, m: int, ov: int, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """Fold of every block of m rows plus the ov rows before it (x, z: the stream from position 0;
    bias: [m + ov, d] or None) -> fp64 [n/m, d]. ov = 0 is `compress`."""
    if x.rows % m:
        raise ValueError("token count %d is not a multiple of m=%d" % (x.rows, m))
    out = np.empty((x.rows // m, x.cols), np.float64)
    b = None if bias is None else np.ascontiguousarray(bias, np.float64).reshape(m + ov, x.cols)
    xm, zm = x.mat(), z.mat()
    rc = _L().orc_compress_overlap(ctypes.byref(xm), ctypes.byref(zm), _ptr(b), m, ov, out.ctypes.data)
    if rc:
        raise ValueError("orc_compress_overlap failed (%d)" % rc)
    return out


def round_scores_bf16(scores: np.ndarray) -> np.ndarray:
    """Index scores as the BF16-score selection sees them: fp64 -> fp32 -> bf16 (RNE), back to fp64."""
    s = np.ascontiguousarray(scores, np.float64).ravel()
    out = np.empty_like(s)
    _L().orc_round_scores_bf16(s.ctypes.data, s.size, out.ctypes.data)
    return out


def topk_bf16(scores: np.ndarray, k: int):
    """Top-k of the bf16-rounded scores (order: rounded score desc, index asc) -> (idx, k_eff)."""
    return topk(round_scores_bf16(scores), k)


def inverse_rope(o: np.ndarray, r0: int, d_rope: int, t: int, base: float = 10000.0) -> np.ndarray:
    """Channels [r0, r0 + d_rope) of every row of o rotated by -t theta_i (pairs 2i, 2i+1) -> new array."""
    out = np.array(o, np.float64, copy=True, order="C")
    rows, cols = out.shape
    rc = _L().orc_inverse_rope(out.ctypes.data, rows, cols, r0, d_rope, t, float(base))
    if rc:
        raise ValueError("orc_inverse_rope failed (%d)" % rc)
    return out


def visible_entries(t: int, m: int, n_win: int = 128) -> int:
    return int(_L().orc_visible_entries(t, m, n_win))


def window_start(t: int, n_win: int = 128) -> int:
    return int(_L().orc_window_start(t, n_win))


def index_scores(qI: Stored, w: np.ndarray, kI: Stored, n_vis: int) -> np.ndarray:
    w = np.ascontiguousarray(w, np.float64).ravel()
    if w.size != qI.rows:
        raise ValueError("w needs one weight per indexer head")
    out = np.empty(max(n_vis, 1), np.float64)
    qm, km = qI.mat(), kI.mat()
    rc = _L().orc_index_scores(ctypes.byref(qm), w.ctypes.data, ctypes.byref(km), n_vis, out.ctypes.data)
    if rc:
        raise ValueError("orc_index_scores failed (%d)" % rc)
    return out[:n_vis]


def topk(scores: np.ndarray, k: int):
    """-> (idx int32 [k] ascending, -1 padded; k_eff)."""
    s = np.ascontiguousarray(scores, np.float64).ravel()
    idx = np.empty(k, np.int32)
    keff = _L().orc_topk(s.ctypes.data, s.size, k, idx.ctypes.data)
    return idx, int(keff)


def attend(q: Stored, keys: Stored, dv: int, sm_scale: float):
    """One softmax over all rows of `keys` for every head (row) of q -> (o [H, dv], lse [H])."""
    o = np.empty((q.rows, dv), np.float64)
    lse = np.empty(q.rows, np.float64)
    qm, km = q.mat(), keys.mat()
    rc = _L().orc_attend(ctypes.byref(qm), ctypes.byref(km), dv, sm_scale, o.ctypes.data, lse.ctypes.data)
    if rc:
        raise ValueError("orc_attend failed (%d)" % rc)
    return o, lse


def csa_query(t: int, m: int, n_win: int, k: int, q: Stored, qI: Stored, w: np.ndarray,
              win: Stored, kv: Stored, kI: Stored, dv: int, sm_scale: float):
    """One query through a CSA layer -> (idx [k], scores [n_vis], o [H, dv], lse [H])."""
    n_vis = visible_entries(t, m, n_win)
    w = np.ascontiguousarray(w, np.float64).ravel()
    idx = np.empty(k, np.int32)
    scores = np.empty(max(n_vis, 1), np.float64)
    o = np.empty((q.rows, dv), np.float64)
    lse = np.empty(q.rows, np.float64)
    ms = [a.mat() for a in (q, qI, win, kv, kI)]
    rc = _L().orc_csa_query(t, m, n_win, k, ctypes.byref(ms[0]), ctypes.byref(ms[1]), w.ctypes.data,
                            ctypes.byref(ms[2]), ctypes.byref(ms[3]), ctypes.byref(ms[4]), dv, sm_scale,
                            idx.ctypes.data, scores.ctypes.data, o.ctypes.data, lse.ctypes.data)
    if rc:
        raise ValueError("orc_csa_query failed (%d)" % rc)
    return idx, scores[:n_vis], o, lse


def hca_query(t: int, m: int, n_win: int, q: Stored, win: Stored, kv: Stored, dv: int,
              sm_scale: float):
    """One query through an HCA layer -> (o [H, dv], lse [H])."""
    o = np.empty((q.rows, dv), np.float64)
    lse = np.empty(q.rows, np.float64)
    ms = [a.mat() for a in (q, win, kv)]
    rc = _L().orc_hca_query(t, m, n_win, ctypes.byref(ms[0]), ctypes.byref(ms[1]), ctypes.byref(ms[2]),
                            dv, sm_scale, o.ctypes.data, lse.ctypes.data)
    if rc:
        raise ValueError("orc_hca_query failed (%d)" % rc)
    return o, lse


def num_threads() -> int:
    return int(_L().orc_num_threads())


def set_threads(n: int) -> None:
    _L().orc_set_num_threads(int(n))
