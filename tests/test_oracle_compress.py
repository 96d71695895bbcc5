"""Pins for the oracle's KV compression (CSA m = 4, HCA m' = 128).

DeepSeek-V4-book ch.1, section 4: CSA folds every m = 4 tokens into one
entry, HCA every m' = 128. DeepSeek-V4 report digest, section 3: the same.
The "constraint chain" essay (innovation 1) calls the fold a weighted fusion
of several tokens' KV; the 10100.com article (section 2.1) adds position
weighting. The fold is a softmax-gated weighted sum per channel.

Pins: m = 1 is the identity; a constant gate gives the block mean; one
dominant logit picks its token; a constant stream is a fixed point (the gate
weights sum to 1); a shared per-token gate equals the broadcast per-channel
gate; the position bias enters as an additive logit (checked against
scipy's softmax); shift invariance and order invariance within a block; the
pages' entry counts at 1M context.
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax


def _bf16(orc, a):
    a = np.asarray(a, np.float32)
    bits = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return orc.Stored(orc.BF16, bits, a.shape[0], a.shape[1])


def _stream(orc, n, d, zc, seed):
    rng = np.random.default_rng(seed)
    x = _bf16(orc, rng.standard_normal((n, d)) / np.sqrt(d))
    z = _bf16(orc, rng.standard_normal((n, zc)))
    return x, z


def test_m1_is_identity(orc):
    x, z = _stream(orc, 64, 32, 32, 0)
    c = orc.compress(x, z, 1)
    assert np.array_equal(c, orc.decode(x))


@pytest.mark.parametrize("m", [4, 128])
def test_constant_gate_gives_block_mean(orc, m):
    n, d = 2 * m, 16
    rng = np.random.default_rng(1)
    x = _bf16(orc, rng.standard_normal((n, d)))
    z = _bf16(orc, np.full((n, d), 0.75))
    c = orc.compress(x, z, m)
    mean = orc.decode(x).reshape(n // m, m, d).mean(axis=1)
    assert np.allclose(c, mean, rtol=1e-13, atol=1e-15)


def test_dominant_logit_picks_its_token(orc):
    m, d = 4, 8
    n = 3 * m
    rng = np.random.default_rng(2)
    xv = rng.standard_normal((n, d))
    zv = rng.standard_normal((n, d)) * 0.1
    pick = rng.integers(0, m, size=(n // m, d))  # per block and channel
    for j in range(n // m):
        for ch in range(d):
            zv[j * m + pick[j, ch], ch] += 60.0
    x, z = _bf16(orc, xv), _bf16(orc, zv)
    c = orc.compress(x, z, m)
    xd = orc.decode(x)
    want = np.array([[xd[j * m + pick[j, ch], ch] for ch in range(d)] for j in range(n // m)])
    assert np.allclose(c, want, rtol=0, atol=1e-20 + 4 * np.exp(-58.0))


@pytest.mark.parametrize("m", [4, 128])
def test_constant_stream_is_fixed_point(orc, m):
    # the gate weights sum to 1, so a channel that is constant over a block
    # comes out unchanged whatever the gate logits are
    n, d = 2 * m, 24
    rng = np.random.default_rng(3)
    col = rng.standard_normal(d)
    x = _bf16(orc, np.tile(col, (n, 1)))
    z = _bf16(orc, rng.standard_normal((n, d)) * 3)
    c = orc.compress(x, z, m)
    assert np.allclose(c, np.tile(orc.decode(x)[0], (n // m, 1)), rtol=1e-14, atol=0)


def test_per_token_gate_equals_broadcast_gate(orc):
    n, d, m = 32, 16, 4
    rng = np.random.default_rng(4)
    x = _bf16(orc, rng.standard_normal((n, d)))
    zt = rng.standard_normal((n, 1))
    c1 = orc.compress(x, _bf16(orc, zt), m)
    c2 = orc.compress(x, _bf16(orc, np.tile(zt, (1, d))), m)
    assert np.array_equal(c1, c2)


def test_position_bias_is_additive_logit(orc):
    n, d, m = 8, 6, 4
    rng = np.random.default_rng(5)
    x = _bf16(orc, rng.standard_normal((n, d)))
    z = _bf16(orc, np.zeros((n, d)))
    bias = rng.standard_normal((m, d)) * 2
    c = orc.compress(x, z, m, bias=bias)
    a = softmax(bias, axis=0)  # [m, d], library softmax over the block positions
    xd = orc.decode(x).reshape(n // m, m, d)
    want = (a[None] * xd).sum(axis=1)
    assert np.allclose(c, want, rtol=1e-13, atol=1e-15)


def test_gate_shift_invariance(orc):
    n, d, m = 16, 8, 4
    rng = np.random.default_rng(6)
    x = _bf16(orc, rng.standard_normal((n, d)))
    zv = np.round(rng.standard_normal((n, d)) * 4) / 4  # exact in bf16 before and after +2
    c1 = orc.compress(x, _bf16(orc, zv), m)
    c2 = orc.compress(x, _bf16(orc, zv + 2.0), m)
    assert np.allclose(c1, c2, rtol=1e-13, atol=1e-15)


def test_order_within_block_does_not_matter(orc):
    n, d, m = 8, 8, 4
    rng = np.random.default_rng(7)
    xv, zv = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    perm = np.concatenate([rng.permutation(m) + j * m for j in range(n // m)])
    c1 = orc.compress(_bf16(orc, xv), _bf16(orc, zv), m)
    c2 = orc.compress(_bf16(orc, xv[perm]), _bf16(orc, zv[perm]), m)
    assert np.allclose(c1, c2, rtol=1e-13, atol=1e-15)


def test_block_boundaries(orc):
    # entry j depends on tokens j*m .. j*m+m-1 only
    n, d, m = 16, 4, 4
    rng = np.random.default_rng(8)
    xv, zv = rng.standard_normal((n, d)), rng.standard_normal((n, d))
    c1 = orc.compress(_bf16(orc, xv), _bf16(orc, zv), m)
    xv2 = xv.copy()
    xv2[8:12] += 5.0  # block 2 only
    c2 = orc.compress(_bf16(orc, xv2), _bf16(orc, zv), m)
    changed = np.any(c1 != c2, axis=1)
    assert list(changed) == [False, False, True, False]


def test_rejects_partial_block(orc):
    x, z = _stream(orc, 10, 4, 4, 9)
    with pytest.raises(ValueError):
        orc.compress(x, z, 4)


def test_entry_counts_at_1m(orc):
    # DeepSeek-V4-book ch.1 section 4: n/m' = 8K heavy entries at n = 1M; CSA keeps
    # n/4 entries and top-k = 1024 of them cover 4096 fine-grained tokens.
    n = 1 << 20
    assert n // 128 == 8192
    assert n // 4 == 262144
    assert 1024 * 4 == 4096
