"""Pins for the oracle's whole query path: visibility, window, CSA, HCA.

DeepSeek-V4 report digest, section 3: CSA attends the top-k compressed
entries, HCA all heavy entries, and both add the last n_win = 128 raw
tokens. The pages fix no causal rule between the window and the compressed
entries; the reading taken is that entry j is visible to position t iff its
block starts before the window (j*m < t + 1 - n_win). These tests pin that
reading against the invariants it must keep:
  * context <= n_win: both layers are plain causal dense attention
    (torch's scaled-dot-product attention with a causal mask);
  * k >= |E_csa|: CSA equals dense attention over the window and all visible
    entries;
  * every position before the window is covered by a visible entry and no
    visible entry starts inside the window;
  * the pages' counts at 1M context (8K HCA entries, 4096 tokens behind
    top-1024 CSA entries);
  * a constant value stream passes through both layers unchanged.
"""
import numpy as np
import pytest
import torch


def _bf16(orc, a):
    a = np.asarray(a, np.float32)
    bits = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return orc.Stored(orc.BF16, bits, a.shape[0], a.shape[1])


def _layer_inputs(orc, n, d, H, hi, di, seed, sharp=False):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) / (1.0 if sharp else np.sqrt(d))
    return dict(
        x=_bf16(orc, x),
        z=_bf16(orc, rng.standard_normal((n, d))),
        xi=_bf16(orc, rng.standard_normal((n, di)) / 8),
        zi=_bf16(orc, rng.standard_normal((n, di))),
        q=_bf16(orc, rng.standard_normal((H, d)) * (np.sqrt(d) if sharp else 1.0)),
        qi=_bf16(orc, rng.standard_normal((hi, di))),
        w=rng.uniform(0, 1, hi),
    )


def test_visible_counts_match_pages(orc):
    t = (1 << 20) - 1
    assert orc.visible_entries(t, 128, 128) == 8191  # 8,192 stored, the last in the window
    assert orc.visible_entries(t, 4, 128) == 262112
    assert orc.visible_entries(8191, 4, 128) == 2016
    assert orc.visible_entries(8191, 128, 128) == 63
    for t in range(0, 128):
        assert orc.visible_entries(t, 4, 128) == 0 and orc.window_start(t) == 0


@pytest.mark.parametrize("m", [4, 128])
def test_visibility_covers_every_position_before_the_window(orc, m):
    for t in list(range(100, 700)) + [8191, 131071, (1 << 20) - 1]:
        nv = orc.visible_entries(t, m, 128)
        ws = orc.window_start(t)
        # the visible entries cover positions 0 .. nv*m-1, reaching at least the window
        assert nv * m >= ws
        # no visible entry starts inside the window
        assert nv == 0 or (nv - 1) * m < ws
        # every visible block is complete by position t (m <= n_win)
        assert nv == 0 or nv * m - 1 <= t
        assert t - ws + 1 == min(t + 1, 128)


@pytest.mark.parametrize("t", [0, 1, 63, 127])
def test_short_context_is_causal_dense_attention(orc, t):
    n, d, H, hi, di = 128, 32, 4, 2, 16
    inp = _layer_inputs(orc, n, d, H, hi, di, seed=t, sharp=True)
    x = orc.decode(inp["x"])
    scale = 1.0 / np.sqrt(d)
    kv_c = orc.store(orc.compress(inp["x"], inp["z"], 4), orc.BF16)
    ki_c = orc.store(orc.compress(inp["xi"], inp["zi"], 4), orc.BF16)
    kv_h = orc.store(orc.compress(inp["x"], inp["z"], 128), orc.BF16)
    win = inp["x"].rows_subset(orc.window_start(t), t + 1)
    _, _, o_csa, l_csa = orc.csa_query(t, 4, 128, 8, inp["q"], inp["qi"], inp["w"], win, kv_c, ki_c, d, scale)
    o_hca, l_hca = orc.hca_query(t, 128, 128, inp["q"], win, kv_h, d, scale)
    # textbook causal attention over raw tokens 0..t for the query row at position t
    Q = torch.from_numpy(orc.decode(inp["q"]))[:, None, :]  # [H, 1, d]
    K = torch.from_numpy(x[: t + 1])[None].expand(H, -1, -1)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, K, scale=scale)[:, 0].numpy()
    assert np.allclose(o_csa, ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(o_hca, ref, rtol=1e-12, atol=1e-13)
    assert np.allclose(l_csa, l_hca, rtol=1e-14)


def test_csa_with_k_covering_all_entries_is_dense(orc):
    n, d, H, hi, di = 1024, 32, 4, 2, 16
    t = n - 1
    inp = _layer_inputs(orc, n, d, H, hi, di, seed=11)
    kv_c = orc.store(orc.compress(inp["x"], inp["z"], 4), orc.BF16)
    ki_c = orc.store(orc.compress(inp["xi"], inp["zi"], 4), orc.BF16)
    nv = orc.visible_entries(t, 4, 128)
    win = inp["x"].rows_subset(orc.window_start(t), t + 1)
    scale = 0.2
    idx, _, o, lse = orc.csa_query(t, 4, 128, nv + 5, inp["q"], inp["qi"], inp["w"], win, kv_c, ki_c, d, scale)
    assert list(idx[:nv]) == list(range(nv)) and np.all(idx[nv:] == -1)
    # dense over window + every visible entry == an HCA-style layer over the m=4 cache
    o2, l2 = orc.hca_query(t, 4, 128, inp["q"], win, kv_c, d, scale)
    assert np.allclose(o, o2, rtol=1e-12, atol=1e-14) and np.allclose(lse, l2, rtol=1e-13)
    # and the same as attention over the explicit union
    keys = np.vstack([orc.decode(win), orc.decode(kv_c)[:nv]])
    o3, l3 = orc.attend(inp["q"], orc.f64(keys), d, scale)
    assert np.allclose(o, o3, rtol=1e-12, atol=1e-14)


def test_csa_selection_is_topk_of_scores(orc):
    n, d, H, hi, di = 2048, 32, 4, 4, 16
    t = n - 1
    inp = _layer_inputs(orc, n, d, H, hi, di, seed=12)
    kv_c = orc.store(orc.compress(inp["x"], inp["z"], 4), orc.BF16)
    ki_c = orc.store(orc.compress(inp["xi"], inp["zi"], 4), orc.BF16)
    win = inp["x"].rows_subset(orc.window_start(t), t + 1)
    idx, scores, o, _ = orc.csa_query(t, 4, 128, 64, inp["q"], inp["qi"], inp["w"], win, kv_c, ki_c, d, 0.2)
    nv = orc.visible_entries(t, 4, 128)
    assert scores.shape == (nv,)
    assert np.array_equal(scores, orc.index_scores(inp["qi"], inp["w"], ki_c, nv))
    ref_idx, _ = orc.topk(scores, 64)
    assert np.array_equal(idx, ref_idx)
    keys = np.vstack([orc.decode(win), orc.decode(kv_c)[idx]])
    o2, _ = orc.attend(inp["q"], orc.f64(keys), d, 0.2)
    assert np.allclose(o, o2, rtol=1e-12, atol=1e-14)


def test_constant_values_pass_through_both_layers(orc):
    n, d, H, hi, di = 1024, 16, 2, 2, 16
    t = n - 1
    rng = np.random.default_rng(13)
    col = rng.standard_normal(d)
    x = _bf16(orc, np.tile(col, (n, 1)))
    z = _bf16(orc, rng.standard_normal((n, d)))
    xi = _bf16(orc, rng.standard_normal((n, di)))
    zi = _bf16(orc, rng.standard_normal((n, di)))
    q = _bf16(orc, rng.standard_normal((H, d)) * 4)
    qi = _bf16(orc, rng.standard_normal((hi, di)))
    kv_c = orc.store(orc.compress(x, z, 4), orc.BF16)
    ki_c = orc.store(orc.compress(xi, zi, 4), orc.BF16)
    kv_h = orc.store(orc.compress(x, z, 128), orc.BF16)
    win = x.rows_subset(orc.window_start(t), t + 1)
    want = np.tile(orc.decode(x)[0], (H, 1))
    _, _, o, _ = orc.csa_query(t, 4, 128, 16, q, qi, np.ones(hi), win, kv_c, ki_c, d, 0.25)
    assert np.allclose(o, want, rtol=1e-13, atol=1e-14)
    o, _ = orc.hca_query(t, 128, 128, q, win, kv_h, d, 0.25)
    assert np.allclose(o, want, rtol=1e-13, atol=1e-14)


def test_dominant_key_wins(orc):
    # a key aligned with the query far above the rest takes all the weight
    n, d, H = 512, 32, 1
    t = n - 1
    rng = np.random.default_rng(14)
    xv = rng.standard_normal((n, d)) * 0.01
    qv = rng.standard_normal((H, d))
    xv[t - 5] = 3 * qv[0] / np.linalg.norm(qv[0])  # inside the window
    x = _bf16(orc, xv)
    kv_h = orc.store(orc.compress(x, _bf16(orc, np.zeros((n, d))), 128), orc.BF16)
    win = x.rows_subset(orc.window_start(t), t + 1)
    o, _ = orc.hca_query(t, 128, 128, _bf16(orc, qv * 40), win, kv_h, d, 1.0)
    assert np.allclose(o[0], orc.decode(x)[t - 5], rtol=0, atol=1e-10)
