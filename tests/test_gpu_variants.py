"""GPU parity of the variant rows against the oracle: BF16 index scores (the
selection made on scores rounded to bf16; DeepSeek-V4 report digest, section
7), with their recall against the fp32 selection; and the inverse RoPE on the
attention output ("constraint chain" essay, innovation 1) on every attention
kernel that writes a final output.

BF16-mode band: the GPU rounds its fp32 score, the oracle its fp64 score, so
a score within an fp32 rounding of a bf16 midpoint may round the other way.
Every entry in the symmetric difference of the two selections must therefore
lie within one bf16 step (2^-7 relative) of the k-th rounded score.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import layer_entries, make_layer, stored_bf16, stored_fp4
from test_gpu_attend import _many, _run
from test_gpu_indexer import _oracle_scores, _setup

pytestmark = pytest.mark.gpu
BF16_BAND = 2.0 ** -7


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def check_topk_bf16(gpu_idx, gpu_cnt, gpu_sc, scores, k):
    """The GPU's bf16-mode selection against the oracle's; returns the recall of the fp32 selection."""
    n = scores.size
    keff = min(k, n)
    assert gpu_cnt == keff
    g = np.asarray(gpu_idx[:keff], np.int64)
    assert np.all(np.asarray(gpu_idx[keff:]) == -1)
    assert np.all(np.diff(g) > 0)
    r = oracle.round_scores_bf16(scores)
    ref, _ = oracle.topk(r, k)
    sym = set(g.tolist()) ^ set(ref[:keff].tolist())
    if sym and keff:
        r_k = np.sort(r)[::-1][keff - 1]
        for j in sym:
            assert abs(scores[j] - r_k) <= BF16_BAND * abs(r_k) + 1e-30, (j, scores[j], r_k)
    # the reported scores are bf16 values, within one bf16 step of the oracle's
    sc = np.asarray(gpu_sc[:keff], np.float32)
    assert np.all((sc.view(np.uint32) & 0xffff) == 0)
    if keff:
        assert np.all(np.abs(sc - scores[g]) <= BF16_BAND * np.abs(scores[g]) + 1e-30)
    if keff == 0:
        return 1.0  # nothing visible: both selections are empty
    ref32, _ = oracle.topk(scores, k)
    return len(set(g.tolist()) & set(ref32[:keff].tolist())) / keff


@pytest.mark.parametrize("hi,di,fp4", [(8, 128, False), (4, 64, False), (8, 128, True)])
def test_bf16_scores_decode(ck, orc, hi, di, fp4):
    k = 256
    positions = [50, 127 + 200 * 4, 127 + 4 * 20000 + 3, 127 + 4 * 65000 + 1]
    L, q_idx, q_sc, w, seq, pos = _setup(ck, positions, hi, di, k, fp4=fp4, seed=40 + hi + di)
    B = len(positions)
    out_idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(B, k, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc, q_idx_scale=q_sc,
                            status=status, score_bf16=True)
    assert ck.cskv_get_status(status) == ck.OK
    idx, cnt, sc = out_idx.cpu().numpy(), out_cnt.cpu().numpy(), out_sc.cpu().numpy()
    recalls = []
    for b, t in enumerate(positions):
        s = _oracle_scores(orc, L, b, t, q_idx, q_sc, w, fp4)
        recalls.append(check_topk_bf16(idx[b], int(cnt[b]), sc[b], s, k))
    assert min(recalls) >= 0.9, recalls


def test_bf16_scores_many_queries(ck, orc):
    """Grouped scan and the streaming selection (calls of >= 256 queries) in bf16 mode."""
    k, hi, di = 128, 4, 64
    positions = [127 + 4 * 6000 + (i % 4) for i in range(300)]  # one sequence's consecutive positions
    L, q_idx, _, w, _, pos = _setup(ck, positions[:1], hi, di, k, seed=77)
    n_q = len(positions)
    g = torch.Generator().manual_seed(78)
    q_idx = torch.randn(n_q, hi, di, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(n_q, hi, generator=g).cuda()
    seq = torch.zeros(n_q, dtype=torch.int32, device="cuda")
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    out_idx = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((n_q,), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(n_q, k, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc, status=status,
                            score_bf16=True)
    assert ck.cskv_get_status(status) == ck.OK
    idx, cnt, sc = out_idx.cpu().numpy(), out_cnt.cpu().numpy(), out_sc.cpu().numpy()
    nv_max = orc.visible_entries(max(positions), 4, 128)
    ent = layer_entries(L, 0, nv_max)["idx"]
    for b in (0, 1, 2, 3, 150, 299):
        t = positions[b]
        nv = orc.visible_entries(t, 4, 128)
        s = orc.index_scores(stored_bf16(q_idx[b]), w[b].cpu().double().numpy(), ent.rows_subset(0, nv), nv)
        check_topk_bf16(idx[b], int(cnt[b]), sc[b], s, k)


# ----------------------------------------------------------------- inverse RoPE on the output
@pytest.mark.parametrize("kind,rope", [("hca", 64), ("csa", 32)])
def test_inverse_rope_split_kernel(ck, orc, kind, rope):
    """d = 128 through the split kernel and its merge (positions up to 1M: angles of ~1e6 radians)."""
    _run(ck, orc, kind, 128, 128, 32, [3, 300, 128 * 300 + 5, 1048575], seed=61, rope_dims=rope)


def test_inverse_rope_latent_kernel(ck, orc):
    """The 576 / 512 tensor-core kernel and its head-minor merge."""
    _run(ck, orc, "hca", 576, 512, 128, [5, 128 * 40 + 77, 128 * 900 + 1], seed=62, rope_dims=64)


def test_inverse_rope_query_pair_kernel(ck, orc):
    """The query-pair kernel writes its bf16 output itself."""
    _many(ck, orc, "hca", 600, 2, 128 * 300, seed=63, rope_dims=64)


# ----------------------------------------------------------------- block overlap in the fold
def _assert_overlap_close(got, ref, x_raw, m, ov, what):
    """One bf16 step plus the fp32 bound of an (m + ov)-term weighted sum of the stream's values."""
    from gpu_helpers import bf16_ulp
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    tol = bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) + 2.0 * (m + ov) * 2.0 ** -24 * np.abs(x_raw).max()
    bad = np.abs(got - ref) > tol * 1.0000001
    assert not bad.any(), "%s: %d beyond tolerance, e.g. got %r ref %r" % (what, int(bad.sum()), got[bad][:3], ref[bad][:3])


@pytest.mark.parametrize("kind,m,ov,d", [("csa", 4, 2, 128), ("csa", 4, 4, 576), ("hca", 64, 64, 128)])
def test_overlap_bulk_segments_and_append(ck, orc, kind, m, ov, d):
    """The fold with block overlap (10100.com DeepSeek-V4 article, section 2.1) through three routes:
    one bulk compression of the stream, two bulk segments with the second one's overlap tokens read from
    the ring, and token-by-token decode appends. m = 64 with 64 overlap tokens takes the block-per-entry
    bulk fold."""
    from test_gpu_compress import _stream
    B, n, n1, d_idx = 2, 768, 384, 64
    is_csa = kind == "csa"
    g = torch.Generator().manual_seed(70 + m + ov)
    bias = (torch.randn(m + ov, d, generator=g) * 2).cuda()
    bias_i = torch.randn(m + ov, d_idx, generator=g).cuda() if is_csa else None
    layers = []
    for _ in range(3):
        L = make_layer(ck.LAYER_CSA if is_csa else ck.LAYER_HCA, m, d, d, B, n // m + 1,
                       d_idx=d_idx if is_csa else 0, seed=71)
        L.overlap = ov
        L.pos_bias = bias
        if is_csa:
            L.pos_bias_idx = bias_i
        layers.append(L)
    La, Lb, Lc = layers
    x, z = _stream(B, n, d, d, seed=72)
    xi, zi = _stream(B, n, d_idx, d_idx, seed=73)
    seq = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def bulk(L, t0, t1):
        sl = slice(t0, t1)
        if is_csa:
            ck.csa_compress_kv(L, seq, t0, x[:, sl].contiguous(), z[:, sl].contiguous(), xi[:, sl].contiguous(),
                               zi[:, sl].contiguous(), status=status)
        else:
            ck.hca_compress_kv(L, seq, t0, x[:, sl].contiguous(), z[:, sl].contiguous(), status=status)

    def append(L, t0, t1, ring_only=False):
        sl = slice(t0, t1)
        pos = torch.full((B,), t0, dtype=torch.int64, device="cuda")
        ck.cskv_cache_append(L, seq, pos, x[:, sl].contiguous(), z[:, sl].contiguous(),
                             xi[:, sl].contiguous() if is_csa else None, zi[:, sl].contiguous() if is_csa else None,
                             ring_only=ring_only, status=status)

    bulk(La, 0, n)
    bulk(Lb, 0, n1)
    append(Lb, n1 - 128, n1, ring_only=True)  # the state cache before the second segment
    bulk(Lb, n1, n)
    for t in range(n):
        append(Lc, t, t + 1)
    assert ck.cskv_get_status(status) == ck.OK
    for b in range(B):
        s = int(seq[b])
        ref = orc.compress_overlap(stored_bf16(x[b]), stored_bf16(z[b]), m, ov, bias.cpu().double().numpy())
        ref = orc.decode(orc.store(ref, orc.BF16))
        xd = orc.decode(stored_bf16(x[b]))
        if is_csa:
            ref_i = orc.compress_overlap(stored_bf16(xi[b]), stored_bf16(zi[b]), m, ov, bias_i.cpu().double().numpy())
            ref_i = orc.decode(orc.store(ref_i, orc.BF16))
        for L, what in ((La, "one bulk"), (Lb, "two segments"), (Lc, "appends")):
            e = layer_entries(L, s, n // m)
            _assert_overlap_close(orc.decode(e["kv"]), ref, xd, m, ov, "%s kv seq %d" % (what, s))
            if is_csa:
                _assert_overlap_close(orc.decode(e["idx"]), ref_i, orc.decode(stored_bf16(xi[b])), m, ov,
                                      "%s idx seq %d" % (what, s))


def test_overlap_bound_is_checked(ck):
    L = make_layer(ck.LAYER_CSA, 4, 128, 128, 1, 64, d_idx=64)
    L.overlap = 125  # more than n_win - m: the borrowed tokens would have left the ring
    x = torch.zeros(1, 4, 128, dtype=torch.bfloat16, device="cuda")
    xi = torch.zeros(1, 4, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ck.CskvError):
        ck.csa_compress_kv(L, torch.zeros(1, dtype=torch.int32, device="cuda"), 0, x, x, xi, xi)
