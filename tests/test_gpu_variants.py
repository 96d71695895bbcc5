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
