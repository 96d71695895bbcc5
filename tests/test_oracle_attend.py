"""Pins for the oracle's attention over a key set (the CSA / HCA core).

DeepSeek-V4 report digest, section 3: the selected (CSA) or all (HCA)
compressed entries and the n_win raw window tokens enter one attention; the
shared latent KV serves every query head (MQA), with V the first d_v channels
of the stored vector (the MLA latent of DeepSeek-V4-book ch.1, section 4).

Pins: torch's scaled-dot-product attention (a library routine) on the same
keys; the log-sum-exp merge of two disjoint key sets (the flash-decoding
identity); a single key gives o = v and lse = the logit; constant V is a
fixed point (weights sum to 1); each head equals a one-head call; key order
does not matter; an empty key set.
"""
import numpy as np
import pytest
import torch


def _rand(orc, rng, rows, cols, scale=1.0):
    return orc.f64(rng.standard_normal((rows, cols)) * scale)


@pytest.mark.parametrize("H,N,dqk,dv", [(4, 37, 32, 32), (8, 130, 72, 64), (2, 1, 16, 8)])
def test_matches_torch_sdpa(orc, H, N, dqk, dv):
    rng = np.random.default_rng(H * 1000 + N)
    q, keys = _rand(orc, rng, H, dqk), _rand(orc, rng, N, dqk, 0.5)
    scale = 1.0 / np.sqrt(dqk)
    o, lse = orc.attend(q, keys, dv, scale)
    Q = torch.from_numpy(q.data)[None]
    K = torch.from_numpy(keys.data)[None]
    V = K[..., :dv]
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)


def test_lse_merge_identity(orc):
    rng = np.random.default_rng(1)
    H, dqk, dv = 6, 40, 32
    q = _rand(orc, rng, H, dqk)
    k1, k2 = rng.standard_normal((50, dqk)), rng.standard_normal((23, dqk))
    s = 0.3
    o1, l1 = orc.attend(q, orc.f64(k1), dv, s)
    o2, l2 = orc.attend(q, orc.f64(k2), dv, s)
    o, l = orc.attend(q, orc.f64(np.vstack([k1, k2])), dv, s)
    lm = np.logaddexp(l1, l2)
    om = (np.exp(l1 - lm)[:, None] * o1 + np.exp(l2 - lm)[:, None] * o2)
    assert np.allclose(l, lm, rtol=1e-13, atol=1e-13)
    assert np.allclose(o, om, rtol=1e-12, atol=1e-13)


def test_single_key(orc):
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((3, 8)), rng.standard_normal((1, 8))
    o, lse = orc.attend(orc.f64(q), orc.f64(k), 5, 0.7)
    assert np.allclose(o, np.tile(k[0, :5], (3, 1)), rtol=1e-15, atol=0)
    assert np.allclose(lse, 0.7 * (q @ k[0]), rtol=1e-14, atol=1e-14)


def test_constant_values_fixed_point(orc):
    rng = np.random.default_rng(3)
    H, N, dqk, dv = 4, 60, 24, 16
    keys = rng.standard_normal((N, dqk))
    const = rng.standard_normal(dv)
    keys[:, :dv] = const  # every V_u equal; keys still differ in the other channels
    o, _ = orc.attend(_rand(orc, rng, H, dqk, 3.0), orc.f64(keys), dv, 1.0)
    assert np.allclose(o, np.tile(const, (H, 1)), rtol=1e-13, atol=1e-14)


def test_each_head_is_an_independent_single_head(orc):
    rng = np.random.default_rng(4)
    q, keys = _rand(orc, rng, 5, 16), _rand(orc, rng, 33, 16)
    o, lse = orc.attend(q, keys, 12, 0.25)
    for h in range(5):
        oh, lh = orc.attend(orc.f64(q.data[h]), keys, 12, 0.25)
        assert np.array_equal(oh[0], o[h]) and lh[0] == lse[h]


def test_key_order_invariance(orc):
    rng = np.random.default_rng(5)
    q, keys = rng.standard_normal((3, 16)), rng.standard_normal((40, 16))
    perm = rng.permutation(40)
    o1, l1 = orc.attend(orc.f64(q), orc.f64(keys), 16, 0.25)
    o2, l2 = orc.attend(orc.f64(q), orc.f64(keys[perm]), 16, 0.25)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14) and np.allclose(l1, l2, rtol=1e-14)


def test_empty_key_set(orc):
    o, lse = orc.attend(orc.f64(np.ones((2, 4))), orc.Stored(orc.F64, np.zeros((0, 4)), 0, 4), 4, 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))
