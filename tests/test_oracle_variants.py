"""Pins of the oracle's variant rows: BF16 index scores, inverse RoPE on the
attention output, and the fold with block overlap.

Each function is checked against something other than itself: a library
routine (torch's fp32 -> bf16 conversion, numpy's complex exponential,
scipy's softmax), a closed form, or an invariant that a dropped term, a wrong
sign or a shifted index would break.
"""
import numpy as np
import pytest
import scipy.special
import torch

import oracle


# ----------------------------------------------------------------- BF16 index scores
def test_bf16_rounding_matches_torch():
    g = np.random.default_rng(7)
    x = np.concatenate([g.normal(0, 30, 5000), g.uniform(-1e-3, 1e-3, 500), [0.0, -0.0, 1.0, 3.0]])
    want = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).float().double().numpy()
    assert np.array_equal(oracle.round_scores_bf16(x), want)


def test_bf16_representable_scores_are_unchanged():
    x = np.array([k / 128.0 for k in range(-255, 256, 7)] + [96.0, 1024.0, -3.5])  # at most 8 significant bits
    assert np.array_equal(oracle.round_scores_bf16(x), x)
    for k in (1, 5, 40, 500):
        assert np.array_equal(oracle.topk_bf16(x, k)[0], oracle.topk(x, k)[0])


def test_bf16_selection_orders_by_rounded_score_then_index():
    g = np.random.default_rng(3)
    for trial in range(30):
        n, k = int(g.integers(5, 200)), int(g.integers(1, 60))
        s = g.normal(0, 1, n) * (1.0 + 0.002 * g.normal(0, 1, n))
        s[g.integers(0, n, n // 4)] = s[0]  # planted exact ties
        r = oracle.round_scores_bf16(s)
        idx, keff = oracle.topk_bf16(s, k)
        order = np.lexsort((np.arange(n), -r))  # rounded score desc, then index asc
        assert keff == min(k, n)
        assert np.array_equal(idx[:keff], np.sort(order[:keff]))
        assert np.all(idx[keff:] == -1)


def test_bf16_selection_equals_fp32_selection_when_scores_are_far_apart():
    g = np.random.default_rng(11)
    s = 1.02 ** np.arange(400) * np.exp(g.normal(0, 0.1))  # neighbours 2% apart, well above a bf16 step
    s = g.permutation(s)
    for k in (8, 100, 399):
        assert np.array_equal(oracle.topk_bf16(s, k)[0], oracle.topk(s, k)[0])


# ----------------------------------------------------------------- inverse RoPE
def _forward_rope(v, pos, d_rope, base):
    """Rotate pairs (2i, 2i+1) of v by +pos theta_i with complex arithmetic (independent of the oracle)."""
    i = np.arange(d_rope // 2)
    theta = base ** (-2.0 * i / d_rope)
    z = (v[..., 0::2] + 1j * v[..., 1::2]) * np.exp(1j * pos * theta)
    out = np.empty_like(v)
    out[..., 0::2], out[..., 1::2] = z.real, z.imag
    return out


def test_inverse_rope_identity_at_position_zero():
    o = np.random.default_rng(1).normal(0, 1, (5, 64))
    assert np.array_equal(oracle.inverse_rope(o, 0, 64, 0), o)


def test_inverse_rope_closed_form_unit_pair():
    d_rope, t, base = 16, 123, 10000.0
    o = np.zeros((1, d_rope))
    o[0, 0::2] = 1.0
    got = oracle.inverse_rope(o, 0, d_rope, t, base)
    theta = base ** (-2.0 * np.arange(d_rope // 2) / d_rope)
    assert np.allclose(got[0, 0::2], np.cos(t * theta), atol=1e-15)
    assert np.allclose(got[0, 1::2], -np.sin(t * theta), atol=1e-15)


def test_inverse_rope_makes_positions_relative_to_the_query():
    g = np.random.default_rng(5)
    d_rope, base = 64, 10000.0
    v = g.normal(0, 1, (3, d_rope))
    for p, t in ((0, 0), (17, 100), (100, 17), (5000, 1048575)):
        rotated = _forward_rope(v, p, d_rope, base)               # a value carrying RoPE at its key position p
        got = oracle.inverse_rope(rotated, 0, d_rope, t, base)    # corrected at the query position t
        assert np.allclose(got, _forward_rope(v, p - t, d_rope, base), atol=1e-9)


def test_inverse_rope_composes_and_keeps_norms_and_other_channels():
    g = np.random.default_rng(9)
    o = g.normal(0, 1, (4, 576))
    r0, d = 512, 64
    a = oracle.inverse_rope(oracle.inverse_rope(o, r0, d, 300), r0, d, 77)
    b = oracle.inverse_rope(o, r0, d, 377)
    assert np.allclose(a, b, atol=1e-12)
    assert np.array_equal(b[:, :r0], o[:, :r0])
    pn = lambda x: np.hypot(x[:, r0::2][:, : d // 2], x[:, r0 + 1::2][:, : d // 2])
    assert np.allclose(pn(b), pn(o), atol=1e-12)


# ----------------------------------------------------------------- fold with block overlap
def _stored(x):
    return oracle.f64(np.asarray(x, np.float64))


def test_overlap_zero_is_the_plain_fold():
    g = np.random.default_rng(2)
    x, z = g.normal(0, 1, (64, 24)), g.normal(0, 1, (64, 24))
    for m in (1, 4, 8):
        assert np.allclose(oracle.compress_overlap(_stored(x), _stored(z), m, 0), oracle.compress(_stored(x), _stored(z), m),
                           rtol=0, atol=1e-15)


@pytest.mark.parametrize("m,ov", [(4, 2), (4, 4), (8, 3), (128, 64)])
def test_overlap_constant_gate_is_the_mean_of_the_extended_block(m, ov):
    g = np.random.default_rng(m + ov)
    n, d = 4 * m, 8
    x = g.normal(0, 1, (n, d))
    z = np.full((n, 1), 0.37)
    got = oracle.compress_overlap(_stored(x), _stored(z), m, ov)
    for j in range(n // m):
        lo = max(0, j * m - ov)
        assert np.allclose(got[j], x[lo:j * m + m].mean(axis=0), atol=1e-12)


def test_overlap_dominant_logit_in_the_overlap_picks_that_token():
    m, ov, n, d = 4, 3, 32, 5
    g = np.random.default_rng(4)
    x, z = g.normal(0, 1, (n, d)), g.normal(0, 1, (n, d))
    j = 3
    p = j * m - 2  # a token of the previous block, inside the overlap
    z2 = z.copy()
    z2[p] += 60.0
    got = oracle.compress_overlap(_stored(x), _stored(z2), m, ov)
    assert np.allclose(got[j], x[p], atol=1e-20 + 1e-20 * np.abs(x[p]).max() + np.exp(-50))
    # the entry whose window does not reach position p is unchanged
    assert np.allclose(got[j + 1], oracle.compress_overlap(_stored(x), _stored(z), m, ov)[j + 1], atol=1e-15)


def test_overlap_bias_against_scipy_softmax():
    m, ov, n, d = 4, 2, 16, 3
    g = np.random.default_rng(6)
    x, z, bias = g.normal(0, 1, (n, d)), g.normal(0, 1, (n, d)), g.normal(0, 1, (m + ov, d))
    got = oracle.compress_overlap(_stored(x), _stored(z), m, ov, bias)
    for j in range(1, n // m):  # full extended windows
        lo = j * m - ov
        w = scipy.special.softmax(z[lo:j * m + m] + bias, axis=0)
        assert np.allclose(got[j], (w * x[lo:j * m + m]).sum(axis=0), atol=1e-13)
    # the first entry sees only its own block, with bias rows ov .. ov + m - 1
    w0 = scipy.special.softmax(z[0:m] + bias[ov:], axis=0)
    assert np.allclose(got[0], (w0 * x[0:m]).sum(axis=0), atol=1e-13)
