"""Helpers for the GPU parity tests: moving device tensors into the oracle's
storage view, building paged layers, and the tolerance checks.

Tolerances (stated in the spec contract for this path):
  * floating outputs: max |d| <= 1e-2 and ||d||_2 / ||ref||_2 <= 2e-2 for
    bf16 (5e-2 for both with FP8 / FP4 storage);
  * top-k: the GPU and oracle index sets have the same size and every id in
    their symmetric difference has an fp64 oracle score within 1e-3 relative
    of the oracle's k-th score (any zero-score choice when that score is 0);
  * compressed entries: within one unit in the last place of the storage
    format (a different summation order can flip one rounding), plus the
    fp32 summation error of the fold where the weighted sum cancels.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

ATOL_BF16, REL_BF16 = 1e-2, 2e-2
ATOL_LP, REL_LP = 5e-2, 5e-2
TIE_REL = 1e-3


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def stored_bf16(t: torch.Tensor) -> oracle.Stored:
    t2 = t.reshape(-1, t.shape[-1])
    return oracle.Stored(oracle.BF16, bf16_bits(t2), t2.shape[0], t2.shape[1])


def stored_fp8(codes: torch.Tensor, scale: torch.Tensor) -> oracle.Stored:
    c = codes.detach().cpu().contiguous().numpy()
    return oracle.Stored(oracle.E4M3, c, c.shape[0], c.shape[1], scale.detach().cpu().float().numpy())


def stored_fp4(codes: torch.Tensor, scales: torch.Tensor) -> oracle.Stored:
    c = codes.detach().cpu().contiguous().numpy()
    return oracle.Stored(oracle.E2M1, c, c.shape[0], c.shape[1] * 2, scales.detach().cpu().contiguous().numpy())


def layer_entries(layer, seq: int, n: int) -> dict:
    """The layer's stored entries 0..n-1 of `seq` as oracle storage views."""
    import compressed_sparse_kv_02_b200 as ck
    e = layer.read_entries(seq, n)
    out = {}
    out["kv"] = stored_bf16(e["kv"]) if layer.kv_dtype == ck.BF16 else stored_fp8(e["kv"], e["kv_scale"])
    if layer.is_csa:
        out["idx"] = stored_bf16(e["idx"]) if layer.idx_dtype == ck.BF16 else stored_fp4(e["idx"], e["idx_scale"])
    return out


def ring_window(layer, seq: int, t: int) -> oracle.Stored:
    """Raw window rows of positions max(0, t-n_win+1) .. t, read from the layer's ring (position order)."""
    ws = max(0, t - layer.n_win + 1)
    slots = [p % layer.n_win for p in range(ws, t + 1)]
    return stored_bf16(layer.ring_x[seq][slots])


def assert_close(got: np.ndarray, ref: np.ndarray, atol: float, rel: float, what: str = ""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what + ": non-finite output"
    d = np.abs(got - ref)
    nrm = np.linalg.norm(ref)
    r = np.linalg.norm(got - ref) / nrm if nrm > 0 else np.linalg.norm(got - ref)
    assert d.max() <= atol, "%s: max |d| = %.3g > %.3g" % (what, d.max(), atol)
    assert r <= rel, "%s: rel l2 = %.3g > %.3g" % (what, r, rel)
    return float(d.max()), float(r)


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    a = np.maximum(np.abs(np.asarray(x, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def assert_fold_close(got: np.ndarray, ref: np.ndarray, x_raw: np.ndarray, m: int, what: str = ""):
    """Stored compressed entries vs the oracle's: one unit in the last place of bf16 plus the fp32
    summation error of an m-term weighted sum, 2 * m * 2^-24 * max_i |x_i| per (entry, channel).

    The second term matters only where the weighted sum cancels to far below its terms (results of
    1e-8 from inputs of 1e-1), where one bf16 ulp of the result is smaller than fp32 rounding of the terms.
    x_raw: the decoded raw rows [n, d] the entries were folded from (rows in entry order).
    """
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    nb, d = ref.shape
    amax = np.abs(np.asarray(x_raw, np.float64)[: nb * m]).reshape(nb, m, d).max(axis=1)
    tol = bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 * m * 2.0 ** -24 * amax
    bad = np.abs(got - ref) > tol * 1.0000001
    assert not bad.any(), "%s: %d elements beyond tolerance, e.g. got %r ref %r" % (
        what, int(bad.sum()), got[bad][:4], ref[bad][:4])


def check_topk(gpu_idx: np.ndarray, gpu_cnt: int, scores: np.ndarray, k: int, rel: float = TIE_REL) -> int:
    """Tie-band check of one query's GPU selection against fp64 oracle scores; returns #swaps."""
    n = scores.size
    keff = min(k, n)
    assert gpu_cnt == keff, (gpu_cnt, keff)
    g = np.asarray(gpu_idx[:keff], np.int64)
    assert np.all(np.asarray(gpu_idx[keff:]) == -1)
    assert np.all(np.diff(g) > 0), "selection not strictly ascending"
    assert keff == 0 or (g.min() >= 0 and g.max() < n)
    ref, _ = oracle.topk(scores, k)
    sym = set(g.tolist()) ^ set(ref[:keff].tolist())
    if sym and keff > 0:
        s_k = np.sort(scores)[::-1][keff - 1]
        for j in sym:
            if s_k == 0.0:
                assert scores[j] == 0.0, (j, scores[j])
            else:
                assert abs(scores[j] - s_k) <= rel * abs(s_k), (j, scores[j], s_k)
    return len(sym) // 2


def make_layer(kind: int, m: int, d_qk: int, d_v: int, n_seqs: int, entries_per_seq: int, d_idx: int = 0,
               page_size: int = 64, kv_dtype=None, idx_dtype=None, gate_cols=None, gate_cols_idx=None,
               seed: int = 0, spare_pages: int = 3):
    """A layer whose sequences own `entries_per_seq` entries on a seeded random permutation of pages."""
    import compressed_sparse_kv_02_b200 as ck
    from compressed_sparse_kv_02_b200 import synth
    pps = max(1, -(-entries_per_seq // page_size))
    n_pages = n_seqs * pps + spare_pages
    layer = ck.Layer.allocate(kind, m, d_qk, d_v, n_seqs=n_seqs, n_pages=n_pages, max_pages_per_seq=pps,
                              page_size=page_size, d_idx=d_idx,
                              kv_dtype=ck.BF16 if kv_dtype is None else kv_dtype,
                              idx_dtype=ck.BF16 if idx_dtype is None else idx_dtype,
                              gate_cols=gate_cols, gate_cols_idx=gate_cols_idx)
    perm = synth.page_permutation(n_pages, seed, 999)
    for s in range(n_seqs):
        layer.set_pages(s, perm[s * pps:(s + 1) * pps])
    return layer
