"""GPU parity: Lightning-indexer scores and top-k selection against the
oracle (DeepSeek-V4 report digest, section 3: the indexer scores the CSA
entries and only the top-k reach core attention; section 7: FP4 indexer QK
path). Selections are compared with the tie band; the oracle scores are
computed from the GPU's own stored indexer keys."""
import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import check_topk, layer_entries, make_layer, stored_bf16, stored_fp4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def _random_fp4(rows, d, g):
    codes = torch.randint(0, 256, (rows, d // 2), generator=g, dtype=torch.int32).to(torch.uint8)
    # e4m3 block scales between 2^-4 and 2 (codes 0x18 .. 0x40)
    scales = torch.randint(0x18, 0x41, (rows, d // 16), generator=g, dtype=torch.int32).to(torch.uint8)
    return codes, scales


def _setup(ck, positions, hi, di, k, fp4=False, seed=0, const_keys=False):
    B = len(positions)
    m, n_win = 4, 128
    n_e = max((max(positions) + 1) // m + 1, 1)
    L = make_layer(ck.LAYER_CSA, m, 128, 128, B, n_e, d_idx=di, idx_dtype=ck.FP4_E2M1 if fp4 else ck.BF16,
                   seed=seed)
    g = torch.Generator().manual_seed(100 + seed)
    q_idx_scale = None
    for b in range(B):
        if fp4:
            codes, scales = _random_fp4(n_e, di, g)
            L.write_entries(b, 0, idx=codes.cuda(), idx_scale=scales.cuda())
        else:
            keys = (torch.randn(n_e, di, generator=g)).to(torch.bfloat16)
            if const_keys:
                keys[:] = keys[0]
            L.write_entries(b, 0, idx=keys.cuda())
    if fp4:
        q_codes, q_scales = _random_fp4(B * hi, di, g)
        q_idx = q_codes.view(B, hi, di // 2).cuda()
        q_idx_scale = q_scales.view(B, hi, di // 16).cuda()
    else:
        q_idx = torch.randn(B, hi, di, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, hi, generator=g).cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    return L, q_idx, q_idx_scale, w, seq, pos


def _oracle_scores(orc, L, b, t, q_idx, q_idx_scale, w, fp4):
    nv = orc.visible_entries(t, 4, 128)
    if nv == 0:
        return np.zeros(0)
    ent = layer_entries(L, b, nv)["idx"]
    if fp4:
        q = stored_fp4(q_idx[b], q_idx_scale[b])
    else:
        q = stored_bf16(q_idx[b])
    return orc.index_scores(q, w[b].cpu().double().numpy(), ent, nv)


@pytest.mark.parametrize("hi,di", [(4, 64), (8, 128), (8, 64), (16, 128)])
def test_scores_and_topk(ck, orc, hi, di):
    k = 64
    # visible counts: 0, 5, k-1, k, k+1, ragged large
    positions = [50, 127 + 5 * 4, 127 + (k - 1) * 4, 127 + k * 4, 127 + (k + 1) * 4 - 2, 127 + 4 * 3000 + 3]
    L, q_idx, _, w, seq, pos = _setup(ck, positions, hi, di, k, seed=hi + di)
    B = len(positions)
    out_idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(B, k, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc, status=status)
    assert ck.cskv_get_status(status) == ck.OK
    idx, cnt, sc = out_idx.cpu().numpy(), out_cnt.cpu().numpy(), out_sc.cpu().numpy()
    for b, t in enumerate(positions):
        s = _oracle_scores(orc, L, b, t, q_idx, None, w, False)
        check_topk(idx[b], int(cnt[b]), s, k)
        keff = int(cnt[b])
        if keff:
            ref = s[idx[b, :keff]]
            assert np.allclose(sc[b, :keff], ref, rtol=1e-4, atol=1e-4 * np.abs(s).max())
        assert np.all(sc[b, keff:] == 0)


def test_ties_prefer_lower_index(ck, orc):
    k = 32
    positions = [127 + 4 * 500]
    L, q_idx, _, w, seq, pos = _setup(ck, positions, 4, 64, k, const_keys=True)
    out_idx = torch.zeros(1, k, dtype=torch.int32, device="cuda")
    out_cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, positions[0], q_idx, w, k, out_idx, out_cnt)
    assert out_idx.cpu().numpy()[0].tolist() == list(range(k))


def test_heavy_ties_across_ctas(ck, orc):
    # Threshold bins far larger than the selection's candidate list, split over many scanning
    # CTAs: query 0's keys are three distinct rows (every score is one of three values; the
    # top row 300 times, the second 25000 times, so 724 ties are taken at the second value),
    # query 1's keys are all equal, and query 2 is plain random in the same call. Ties go to
    # the lowest indices, so the expected selections are exact.
    k = 1024
    positions = [127 + 4 * 40000, 127 + 4 * 30000 + 1, 127 + 4 * 9000 + 2]
    hi, di = 8, 128
    B = len(positions)
    n_e = max(positions) // 4 + 2
    L = make_layer(ck.LAYER_CSA, 4, 128, 128, B, n_e, d_idx=di, seed=21)
    g = torch.Generator().manual_seed(121)
    q_idx = torch.randn(B, hi, di, generator=g).to(torch.bfloat16)
    w = torch.rand(B, hi, generator=g)
    rows = torch.randn(3, di, generator=g).to(torch.bfloat16)
    qd, wd = q_idx[0].double(), w[0].double()
    s3 = [(wd * torch.relu(qd @ rows[r].double())).sum().item() for r in range(3)]
    order = sorted(range(3), key=lambda r: -s3[r])
    assign = torch.full((n_e,), order[2], dtype=torch.long)
    perm = torch.randperm(n_e, generator=g)
    assign[perm[:25000]] = order[1]
    assign[perm[25000:25300]] = order[0]
    keys = [rows[assign], rows[0].expand(n_e, di).clone(), torch.randn(n_e, di, generator=g).to(torch.bfloat16)]
    for b in range(B):
        L.write_entries(b, 0, idx=keys[b].cuda())
    q_idx, w = q_idx.cuda(), w.cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    out_idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(B, k, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc, status=status)
    assert ck.cskv_get_status(status) == ck.OK
    idx, cnt = out_idx.cpu().numpy(), out_cnt.cpu().numpy()
    for b, t in enumerate(positions):
        s = _oracle_scores(orc, L, b, t, q_idx, None, w, False)
        assert int(cnt[b]) == k
        if b < 2:
            # distinct score values are far apart, equal ones identical: the top-k by (score desc,
            # index asc), listed in ascending index order
            want = np.sort(np.lexsort((np.arange(len(s)), -s))[:k])
            assert idx[b].tolist() == want.tolist()
        else:
            check_topk(idx[b], k, s, k)


def test_fp4_indexer(ck, orc):
    k = 128
    positions = [127 + 4 * 2000 + 1, 127 + 4 * 100, 127 + 4 * 5000]
    L, q_idx, q_sc, w, seq, pos = _setup(ck, positions, 8, 128, k, fp4=True, seed=7)
    B = len(positions)
    out_idx = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    out_cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, q_idx_scale=q_sc)
    torch.cuda.synchronize()
    for b, t in enumerate(positions):
        s = _oracle_scores(orc, L, b, t, q_idx, q_sc, w, True)
        check_topk(out_idx[b].cpu().numpy(), int(out_cnt[b]), s, k)


def test_large_selection_uses_several_ctas(ck, orc):
    # 100k visible entries per query: the selection kernel splits each query over a cluster
    k = 1024
    positions = [127 + 4 * 100000, 127 + 4 * 60000 + 2]
    L, q_idx, _, w, seq, pos = _setup(ck, positions, 8, 128, k, seed=9)
    B = len(positions)
    out_idx = torch.zeros(B, k, dtype=torch.int32, device="cuda")
    out_cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(B, k, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc)
    torch.cuda.synchronize()
    for b, t in enumerate(positions):
        s = _oracle_scores(orc, L, b, t, q_idx, None, w, False)
        check_topk(out_idx[b].cpu().numpy(), int(out_cnt[b]), s, k)


def test_position_beyond_bound_is_reported(ck):
    k = 16
    positions = [127 + 4 * 100, 127 + 4 * 50]
    L, q_idx, _, w, seq, pos = _setup(ck, positions, 4, 64, k)
    out_idx = torch.zeros(2, k, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((2,), 9, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, positions[1], q_idx, w, k, out_idx, out_cnt, status=status)
    assert ck.cskv_get_status(status) == ck.ERR_INVALID_ARG
    assert int(out_cnt[0]) == 0 and (out_idx[0] == -1).all()
    assert int(out_cnt[1]) == k


def test_workspace_too_small_is_rejected(ck):
    k = 16
    positions = [127 + 4 * 100]
    L, q_idx, _, w, seq, pos = _setup(ck, positions, 4, 64, k)
    out_idx = torch.zeros(1, k, dtype=torch.int32, device="cuda")
    out_cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    with pytest.raises(ck.CskvError) as e:
        ck.csa_index_score_topk(L, seq, pos, positions[0], q_idx, w, k, out_idx, out_cnt, workspace=ws)
    assert e.value.code == ck.ERR_WORKSPACE


@pytest.mark.parametrize("hi,di", [(4, 64), (8, 128)])
def test_many_queries_grouped_scan(ck, orc, hi, di):
    # 300 queries (the grouped scan: consecutive queries of one sequence share key tiles) from three
    # sequences in runs of uneven length, at positions that vary inside a run: groups must split where
    # the sequence changes and mask each query to its own visible entries
    k = 128
    g = torch.Generator().manual_seed(77 + hi)
    n_seq, n_e = 3, 3000
    L = make_layer(ck.LAYER_CSA, 4, 128, 128, n_seq, n_e, d_idx=di, seed=hi)
    for s in range(n_seq):
        L.write_entries(s, 0, idx=torch.randn(n_e, di, generator=g).to(torch.bfloat16).cuda())
    runs = [(0, 37), (1, 101), (2, 5), (0, 90), (2, 67)]
    seqs, positions = [], []
    for s, n in runs:
        base = int(torch.randint(200, 4 * n_e - 200, (1,), generator=g))
        for i in range(n):
            seqs.append(s)
            positions.append(min(4 * n_e + 127 - 1, base + 3 * i))
    B = len(seqs)
    assert B >= 256
    q_idx = torch.randn(B, hi, di, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, hi, generator=g).cuda()
    seq = torch.tensor(seqs, dtype=torch.int32, device="cuda")
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    out_idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    out_cnt = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    out_sc = torch.zeros(B, k, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.csa_index_score_topk(L, seq, pos, max(positions), q_idx, w, k, out_idx, out_cnt, out_sc, status=status)
    torch.cuda.synchronize()
    assert ck.cskv_get_status(status) == ck.OK
    idx, cnt, scs = out_idx.cpu().numpy(), out_cnt.cpu().numpy(), out_sc.cpu().numpy()
    ents = [layer_entries(L, s, orc.visible_entries(4 * n_e + 127, 4, 128))["idx"] for s in range(n_seq)]
    for b in range(0, B, 7):
        t, s = positions[b], seqs[b]
        nv = orc.visible_entries(t, 4, 128)
        sc = orc.index_scores(stored_bf16(q_idx[b]), w[b].cpu().double().numpy(), ents[s].rows_subset(0, nv), nv)
        check_topk(idx[b], int(cnt[b]), sc, k)
        chosen = idx[b][:int(cnt[b])]
        assert np.allclose(scs[b][:len(chosen)], sc[chosen], rtol=1e-3, atol=1e-3 * max(1.0, np.abs(sc).max()))
