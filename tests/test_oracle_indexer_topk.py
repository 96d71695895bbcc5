"""Pins for the oracle's Lightning-indexer score and top-k selection.

DeepSeek-V4 report digest, section 3 and DeepSeek-V4-book ch.1, section 4: a
light indexer scores every compressed entry for the query and only the
top-k entries (k = 512 Flash, k = 1024 Pro) reach core attention; the
10100.com article (section 2.1) calls it a low-rank indexer. The score is
s(j) = sum_h w_h * ReLU(q_h . K_I[j]) over the indexer heads.

Pins: hand-computed worked examples (tests/golden/indexer_hand.txt); scores
equal a library-matmul arrangement; linearity in w and ReLU clipping; top-k
against a library lexicographic sort; ties prefer the lower index; k >= n
keeps everything; the chunk-local top-k union identity the GPU merge relies
on; positive rescaling of w keeps the set; planted keys are recalled.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load_hand_cases():
    cases, cur = [], None
    with open(os.path.join(GOLDEN, "indexer_hand.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            key, _, val = line.partition(":")
            nums = [float(v) for v in val.split()]
            if key == "case":
                cur = {}
                cases.append(cur)
            else:
                cur[key] = nums
    return cases


def test_hand_examples(orc):
    for case in _load_hand_cases():
        hi, di = int(case["heads"][0]), int(case["dims"][0])
        q = orc.f64(np.array(case["q"]).reshape(hi, di))
        k = orc.f64(np.array(case["k"]).reshape(-1, di))
        s = orc.index_scores(q, np.array(case["w"]), k, k.rows)
        assert np.array_equal(s, np.array(case["scores"])), case


def test_scores_match_matmul_arrangement(orc):
    rng = np.random.default_rng(0)
    hi, di, e = 4, 64, 300
    q, k, w = rng.standard_normal((hi, di)), rng.standard_normal((e, di)), rng.uniform(0, 1, hi)
    s = orc.index_scores(orc.f64(q), w, orc.f64(k), e)
    want = np.maximum(k @ q.T, 0.0) @ w
    assert np.allclose(s, want, rtol=1e-12, atol=1e-12)


def test_linear_in_w_and_relu_clips(orc):
    rng = np.random.default_rng(1)
    hi, di, e = 3, 16, 50
    q, k = rng.standard_normal((hi, di)), rng.standard_normal((e, di))
    w1, w2 = rng.uniform(-1, 1, hi), rng.uniform(-1, 1, hi)
    f = lambda w: orc.index_scores(orc.f64(q), w, orc.f64(k), e)
    assert np.allclose(f(w1 + 2 * w2), f(w1) + 2 * f(w2), rtol=1e-12, atol=1e-12)
    # a head whose dot products are all negative contributes nothing
    qn = q.copy()
    qn[0] = -np.sign(k.sum(0)) * 0  # zero query row -> dot 0 -> ReLU 0
    s_with = orc.index_scores(orc.f64(qn), np.array([100.0, 0.0, 0.0]), orc.f64(k), e)
    assert np.all(s_with == 0.0)


def test_only_visible_prefix_is_scored(orc):
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((2, 8)), rng.standard_normal((40, 8))
    s_all = orc.index_scores(orc.f64(q), np.ones(2), orc.f64(k), 40)
    s_pre = orc.index_scores(orc.f64(q), np.ones(2), orc.f64(k), 25)
    assert np.array_equal(s_pre, s_all[:25])


def _lexsort_topk(s, k):
    order = np.lexsort((np.arange(len(s)), -s))  # score desc, index asc
    return np.sort(order[:k])


@pytest.mark.parametrize("n,k", [(64, 8), (64, 64), (100, 37), (5, 16), (0, 4), (1, 1)])
def test_topk_against_library_sort(orc, n, k):
    rng = np.random.default_rng(n * 31 + k)
    s = rng.standard_normal(n)
    idx, keff = orc.topk(s, k)
    assert keff == min(n, k)
    want = _lexsort_topk(s, k)
    assert np.array_equal(idx[:keff], want)
    assert np.all(idx[keff:] == -1)
    assert np.all(np.diff(idx[:keff]) > 0)


def test_topk_ties_prefer_lower_index(orc):
    s = np.array([1.0, 3.0, 2.0, 3.0, 3.0, 0.0, 3.0, 2.0])
    idx, keff = orc.topk(s, 3)
    assert keff == 3 and list(idx) == [1, 3, 4]
    idx, _ = orc.topk(s, 6)
    assert list(idx) == [1, 2, 3, 4, 6, 7]
    z = np.zeros(10)  # ReLU can leave many exact zeros
    idx, _ = orc.topk(z, 4)
    assert list(idx) == [0, 1, 2, 3]


def test_chunked_topk_union_identity(orc):
    # top-k(all) == top-k(union of chunk-local top-k's), the exactness argument
    # of a chunked selection followed by a merge
    rng = np.random.default_rng(3)
    n, k = 5000, 64
    s = np.round(rng.standard_normal(n), 2)  # many ties
    glob, _ = orc.topk(s, k)
    cand = []
    for lo in range(0, n, 700):
        loc, keff = orc.topk(s[lo:lo + 700], k)
        cand.extend(lo + loc[:keff])
    cand = np.array(cand)
    sel, keff = orc.topk(s[cand], k)
    assert np.array_equal(np.sort(cand[sel[:keff]]), glob)


def test_positive_rescaling_of_w_keeps_the_set(orc):
    rng = np.random.default_rng(4)
    q, k, w = rng.standard_normal((4, 32)), rng.standard_normal((500, 32)), rng.uniform(0, 1, 4)
    a, _ = orc.topk(orc.index_scores(orc.f64(q), w, orc.f64(k), 500), 50)
    b, _ = orc.topk(orc.index_scores(orc.f64(q), 7.5 * w, orc.f64(k), 500), 50)
    assert np.array_equal(a, b)


def test_planted_keys_are_recalled(orc):
    # keys pushed along sum_h w_h q_h score far above the Gaussian background
    rng = np.random.default_rng(5)
    hi, di, n, k = 8, 128, 4000, 64
    q, w = rng.standard_normal((hi, di)), rng.uniform(0, 1, hi)
    keys = rng.standard_normal((n, di))
    u = (w[:, None] * q).sum(0)
    u /= np.linalg.norm(u)
    planted = rng.choice(n, 40, replace=False)
    keys[planted] = 0.5 * keys[planted] + 2 * np.sqrt(di) * u
    idx, _ = orc.topk(orc.index_scores(orc.f64(q), w, orc.f64(keys), n), k)
    assert set(planted) <= set(idx.tolist())
    # flipping the planted direction pushes them below ReLU: none is recalled
    keys2 = keys.copy()
    keys2[planted] = -keys2[planted]
    s2 = orc.index_scores(orc.f64(q), w, orc.f64(keys2), n)
    idx2, _ = orc.topk(s2, k)
    assert not (set(planted) & set(idx2.tolist()))
