"""GPU parity: KV compression (bulk fold and the state-cache append) against
the oracle (DeepSeek-V4 report digest, section 3: CSA m = 4, HCA m' = 128;
section 7: state cache of the window and not-yet-compressed tokens)."""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import assert_fold_close, layer_entries, make_layer, stored_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def _stream(B, n, d, gc, seed, dev="cuda"):
    from compressed_sparse_kv_02_b200 import synth
    x, z = synth.raw_stream(B, n, d, seed, 0, "cpu", gate_cols=gc)
    return x.to(dev), z.to(dev)


@pytest.mark.parametrize("kind,m,d,gate", [("csa", 4, 128, "chan"), ("csa", 4, 576, "tok"), ("hca", 128, 128, "chan"),
                                           ("hca", 128, 576, "chan"), ("hca", 128, 576, "tok")])
def test_bulk_compress_matches_oracle(ck, orc, kind, m, d, gate):
    B, n, d_idx = 3, 1024, 64
    is_csa = kind == "csa"
    gc = d if gate == "chan" else 1
    L = make_layer(ck.LAYER_CSA if is_csa else ck.LAYER_HCA, m, d, d, B, n // m, d_idx=d_idx if is_csa else 0,
                   gate_cols=gc, gate_cols_idx=d_idx if gate == "chan" else 1, seed=1)
    x, z = _stream(B, n, d, gc, seed=10)
    xi, zi = _stream(B, n, d_idx, d_idx if gate == "chan" else 1, seed=11)
    seq = torch.tensor([2, 0, 1], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if is_csa:
        ck.csa_compress_kv(L, seq, 0, x, z, xi, zi, status=status)
    else:
        ck.hca_compress_kv(L, seq, 0, x, z, status=status)
    assert ck.cskv_get_status(status) == ck.OK
    for b in range(B):
        s = int(seq[b])
        got = layer_entries(L, s, n // m)
        ref = orc.store(orc.compress(stored_bf16(x[b]), stored_bf16(z[b]), m), orc.BF16)
        assert_fold_close(orc.decode(got["kv"]), orc.decode(ref), orc.decode(stored_bf16(x[b])), m, "kv seq %d" % s)
        if is_csa:
            ref_i = orc.store(orc.compress(stored_bf16(xi[b]), stored_bf16(zi[b]), m), orc.BF16)
            assert_fold_close(orc.decode(got["idx"]), orc.decode(ref_i), orc.decode(stored_bf16(xi[b])), m,
                              "idx seq %d" % s)


def test_position_bias_and_offset_segment(ck, orc):
    # a segment starting at tok0 = 256 lands at entries 64.., with a position bias
    B, n, d, m, tok0 = 2, 512, 128, 4, 256
    L = make_layer(ck.LAYER_CSA, m, d, d, B, (tok0 + n) // m, d_idx=64, seed=2)
    g = torch.Generator().manual_seed(5)
    L.pos_bias = (torch.randn(m, d, generator=g) * 2).cuda()
    L.pos_bias_idx = (torch.randn(m, 64, generator=g)).cuda()
    x, z = _stream(B, n, d, d, seed=12)
    xi, zi = _stream(B, n, 64, 64, seed=13)
    seq = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    ck.csa_compress_kv(L, seq, tok0, x, z, xi, zi)
    torch.cuda.synchronize()
    for b in range(B):
        got = layer_entries(L, b, (tok0 + n) // m)
        ref = orc.store(orc.compress(stored_bf16(x[b]), stored_bf16(z[b]), m, bias=L.pos_bias.cpu().double().numpy()),
                        orc.BF16)
        assert_fold_close(orc.decode(got["kv"])[tok0 // m:], orc.decode(ref), orc.decode(stored_bf16(x[b])), m, "kv")
        ref_i = orc.store(orc.compress(stored_bf16(xi[b]), stored_bf16(zi[b]), m,
                                       bias=L.pos_bias_idx.cpu().double().numpy()), orc.BF16)
        assert_fold_close(orc.decode(got["idx"])[tok0 // m:], orc.decode(ref_i), orc.decode(stored_bf16(xi[b])), m,
                          "idx")


def test_fp8_kv_and_fp4_index_storage(ck, orc):
    B, n, d, d_idx, m = 2, 1024, 576, 128, 4
    L = make_layer(ck.LAYER_CSA, m, d, 512, B, n // m, d_idx=d_idx, kv_dtype=ck.FP8_E4M3, idx_dtype=ck.FP4_E2M1,
                   seed=3)
    x, z = _stream(B, n, d, d, seed=14)
    xi, zi = _stream(B, n, d_idx, d_idx, seed=15)
    seq = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    ck.csa_compress_kv(L, seq, 0, x, z, xi, zi)
    torch.cuda.synchronize()
    for b in range(B):
        got = layer_entries(L, b, n // m)
        c = orc.compress(stored_bf16(x[b]), stored_bf16(z[b]), m)
        ref = orc.store(c, orc.E4M3)
        # per-entry scale: amax / 448 over fp32 values that agree to a few fp32 ulps
        assert np.allclose(got["kv"].scale, ref.scale, rtol=1e-5, atol=0)
        # codes: equal, or one e4m3 step apart where the two sides' values straddle a rounding boundary
        gd, rd = orc.decode(got["kv"]), orc.decode(ref)
        step = np.maximum(np.abs(rd), np.abs(gd)) * 2.0 ** -3 + ref.scale[:, None].astype(np.float64) * 2.0 ** -9
        assert np.all(np.abs(gd - rd) <= step * 1.0001)
        assert np.mean(got["kv"].data == ref.data) > 0.99
        ci = orc.compress(stored_bf16(xi[b]), stored_bf16(zi[b]), m)
        ref_i = orc.store(ci, orc.E2M1)
        assert np.mean(got["idx"].scale == ref_i.scale) > 0.99
        gi, ri = orc.decode(got["idx"]), orc.decode(ref_i)
        sc = orc.e4m3_to_f64(np.repeat(np.maximum(got["idx"].scale, ref_i.scale), 16, axis=1))
        assert np.all(np.abs(gi - ri) <= 2.0 * sc + 1e-12)
        assert np.mean(np.abs(gi - ri) == 0) > 0.99
        # the stored FP4 value is within half a step of the exact fold (the quantiser reading)
        assert np.max(np.abs(ri - ci) / np.maximum(sc, 1e-30)) <= 1.0 + 1e-6


@pytest.mark.parametrize("kind,m", [("csa", 4), ("hca", 128)])
def test_append_equals_bulk_and_fills_ring(ck, orc, kind, m):
    """Token-by-token decode appends produce the entries of one bulk fold (both within the fold
    tolerance of the oracle: the two paths split the token sum differently) and fill the ring."""
    B, d, d_idx = 2, 128, 64
    n = 3 * 128 + 40  # ends mid-block for HCA
    is_csa = kind == "csa"
    mk = lambda: make_layer(ck.LAYER_CSA if is_csa else ck.LAYER_HCA, m, d, d, B, (n + m) // m + 1,
                            d_idx=d_idx if is_csa else 0, seed=4)
    La, Lb = mk(), mk()
    x, z = _stream(B, n, d, d, seed=16)
    xi, zi = _stream(B, n, d_idx, d_idx, seed=17)
    seq = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    nb = (n // m) * m
    if is_csa:
        ck.csa_compress_kv(La, seq, 0, x[:, :nb].contiguous(), z[:, :nb].contiguous(), xi[:, :nb].contiguous(),
                           zi[:, :nb].contiguous())
    else:
        ck.hca_compress_kv(La, seq, 0, x[:, :nb].contiguous(), z[:, :nb].contiguous())
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for t in range(n):
        pos = torch.full((B,), t, dtype=torch.int64, device="cuda")
        sl = slice(t, t + 1)
        ck.cskv_cache_append(Lb, seq, pos, x[:, sl].contiguous(), z[:, sl].contiguous(),
                             xi[:, sl].contiguous() if is_csa else None, zi[:, sl].contiguous() if is_csa else None,
                             status=status)
    assert ck.cskv_get_status(status) == ck.OK
    for b in range(B):
        s = int(seq[b])
        nb_e = n // m
        ref = orc.decode(orc.store(orc.compress(stored_bf16(x[b, :nb_e * m]), stored_bf16(z[b, :nb_e * m]), m),
                                   orc.BF16))
        xd = orc.decode(stored_bf16(x[b]))
        for L, what in ((La, "bulk"), (Lb, "append")):
            e = layer_entries(L, s, nb_e)
            assert_fold_close(orc.decode(e["kv"]), ref, xd, m, "%s kv seq %d" % (what, s))
            if is_csa:
                ref_i = orc.decode(orc.store(orc.compress(stored_bf16(xi[b, :nb_e * m]),
                                                          stored_bf16(zi[b, :nb_e * m]), m), orc.BF16))
                assert_fold_close(orc.decode(e["idx"]), ref_i, orc.decode(stored_bf16(xi[b])), m,
                                  "%s idx seq %d" % (what, s))
        slots = [p % 128 for p in range(n - 128, n)]
        assert torch.equal(Lb.ring_x[s][slots], x[b, n - 128:])
        assert torch.equal(Lb.ring_z[s][slots], z[b, n - 128:])
        if is_csa:
            assert torch.equal(Lb.ring_xi[s][slots], xi[b, n - 128:])


def test_multi_token_append_and_ring_only(ck, orc):
    B, d, d_idx, m = 1, 128, 64, 4
    n = 300
    L1 = make_layer(ck.LAYER_CSA, m, d, d, B, n // m + 1, d_idx=d_idx, seed=5)
    L2 = make_layer(ck.LAYER_CSA, m, d, d, B, n // m + 1, d_idx=d_idx, seed=5)
    x, z = _stream(B, n, d, d, seed=18)
    xi, zi = _stream(B, n, d_idx, d_idx, seed=19)
    seq = torch.zeros(1, dtype=torch.int32, device="cuda")
    # L1: appends of 5 tokens at a time (blocks complete inside and across calls)
    for t0 in range(0, n, 5):
        t1 = min(n, t0 + 5)
        ck.cskv_cache_append(L1, seq, torch.tensor([t0], device="cuda"), x[:, t0:t1].contiguous(),
                             z[:, t0:t1].contiguous(), xi[:, t0:t1].contiguous(), zi[:, t0:t1].contiguous())
    # L2: bulk fold, then ring_only for the last 128 tokens
    ck.csa_compress_kv(L2, seq, 0, x, z, xi, zi)
    ck.cskv_cache_append(L2, seq, torch.tensor([n - 128], device="cuda"), x[:, n - 128:].contiguous(),
                         z[:, n - 128:].contiguous(), xi[:, n - 128:].contiguous(), zi[:, n - 128:].contiguous(),
                         ring_only=True)
    torch.cuda.synchronize()
    ref = orc.decode(orc.store(orc.compress(stored_bf16(x[0]), stored_bf16(z[0]), m), orc.BF16))
    ref_i = orc.decode(orc.store(orc.compress(stored_bf16(xi[0]), stored_bf16(zi[0]), m), orc.BF16))
    for L in (L1, L2):
        e = layer_entries(L, 0, n // m)
        assert_fold_close(orc.decode(e["kv"]), ref, orc.decode(stored_bf16(x[0])), m, "kv")
        assert_fold_close(orc.decode(e["idx"]), ref_i, orc.decode(stored_bf16(xi[0])), m, "idx")
    assert torch.equal(L1.ring_x, L2.ring_x) and torch.equal(L1.ring_zi, L2.ring_zi)


@pytest.mark.parametrize("kind,m", [("csa", 4), ("hca", 128)])
def test_append_ring_then_emit_equals_append(ck, kind, m):
    """The split append of a decode step (ring_only, then emit_only with the same tokens, as the decode
    step issues it to take the compression off its critical path) writes the same ring rows and the same
    entries, bit for bit, as one append; emit_only writes no ring row; both flags at once are refused."""
    B, d, d_idx = 2, 128, 64
    n = 2 * 128 + 8
    is_csa = kind == "csa"
    mk = lambda: make_layer(ck.LAYER_CSA if is_csa else ck.LAYER_HCA, m, d, d, B, n // m + 2,
                            d_idx=d_idx if is_csa else 0, seed=6)
    La, Lb = mk(), mk()
    x, z = _stream(B, n + 1, d, d, seed=20)
    xi, zi = _stream(B, n + 1, d_idx, d_idx, seed=21)
    seq = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")

    def tok(t):
        sl = slice(t, t + 1)
        return (x[:, sl].contiguous(), z[:, sl].contiguous(), xi[:, sl].contiguous() if is_csa else None,
                zi[:, sl].contiguous() if is_csa else None)

    for t in range(n):
        pos = torch.full((B,), t, dtype=torch.int64, device="cuda")
        ck.cskv_cache_append(La, seq, pos, *tok(t), status=status)
        ck.cskv_cache_append(Lb, seq, pos, *tok(t), ring_only=True, status=status)
        ck.cskv_cache_append(Lb, seq, pos, *tok(t), emit_only=True, status=status)
    assert ck.cskv_get_status(status) == ck.OK
    rings = ("ring_x", "ring_z") + (("ring_xi", "ring_zi") if is_csa else ())
    for r in rings:
        assert torch.equal(getattr(La, r), getattr(Lb, r)), r
    for b in range(B):
        ea, eb = layer_entries(La, int(seq[b]), n // m), layer_entries(Lb, int(seq[b]), n // m)
        assert np.array_equal(ea["kv"].data, eb["kv"].data)
        if is_csa:
            assert np.array_equal(ea["idx"].data, eb["idx"].data)
    before = {r: getattr(Lb, r).clone() for r in rings}
    ck.cskv_cache_append(Lb, seq, torch.full((B,), n, dtype=torch.int64, device="cuda"), *tok(n), emit_only=True,
                         status=status)
    assert ck.cskv_get_status(status) == ck.OK
    for r in rings:
        assert torch.equal(getattr(Lb, r), before[r]), r
    with pytest.raises(ck.CskvError) as e:
        ck.cskv_cache_append(Lb, seq, torch.full((B,), n, dtype=torch.int64, device="cuda"), *tok(n),
                             ring_only=True, emit_only=True)
    assert e.value.code == ck.ERR_INVALID_ARG


def test_append_rejects_too_many_tokens(ck):
    L = make_layer(ck.LAYER_CSA, 4, 128, 128, 1, 64, d_idx=64)
    x = torch.zeros(1, 126, 128, dtype=torch.bfloat16, device="cuda")
    xi = torch.zeros(1, 126, 64, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ck.CskvError) as e:
        ck.cskv_cache_append(L, torch.zeros(1, dtype=torch.int32, device="cuda"),
                             torch.zeros(1, dtype=torch.int64, device="cuda"), x, x.clone(), xi, xi.clone())
    assert e.value.code == ck.ERR_INVALID_ARG


def test_bad_page_is_reported_and_skipped(ck, orc):
    # 17 HCA entries on 16-entry pages: entries 0..15 on page slot 0 (made invalid), entry 16 on slot 1
    B, d, m = 1, 128, 128
    n = 17 * m
    L = make_layer(ck.LAYER_HCA, m, d, d, B, 17, page_size=16, seed=6)
    L.page_table[0, 0] = L.n_pages + 5
    L.page_table[0, 1] = 0
    x, z = _stream(B, n, d, d, seed=20)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = L.kv_pool.clone()
    ck.hca_compress_kv(L, torch.zeros(1, dtype=torch.int32, device="cuda"), 0, x, z, status=status)
    assert ck.cskv_get_status(status) == ck.ERR_OUT_OF_RANGE
    assert ck.cskv_get_status(status) == ck.OK  # reading clears the word
    # entry 16 (page 0, slot 0) was still written; nothing else changed
    changed = (L.kv_pool != before).any(dim=1).nonzero().flatten().tolist()
    assert changed == [0]
    ref = orc.store(orc.compress(stored_bf16(x[0]), stored_bf16(z[0]), m), orc.BF16)
    assert_fold_close(orc.decode(stored_bf16(L.kv_pool[0:1])), orc.decode(ref)[16:17],
                      orc.decode(stored_bf16(x[0, 16 * m:17 * m])), m, "entry 16")
