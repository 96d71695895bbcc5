"""GPU parity of whole decode steps.

* tiny (n = 8192, 8 consecutive decode queries, H = 16, d = 128): every
  stage from raw tokens -- bulk compression, state-cache appends that emit
  new entries, indexer + top-512, CSA and HCA attention -- checked stage by
  stage (each stage on the GPU's own inputs to it) and end to end against
  the oracle run from the raw tokens.
* flash (B = 32 x 128K) and pro (B = 8 x 1M, 1% planted keys): the full-size
  workloads in the launch configuration the benchmark times (DecodeModel),
  with the oracle run on sampled queries and heads.
* mixed: the quantised, mixed-length workload (FP8 KV with a scale per entry,
  FP4 indexer keys and queries, per-sequence lengths, layers CSA, HCA, CSA,
  HCA) at a reduced batch and length (every query), and at the benchmark's
  full size (B = 64, lengths up to ~1M; sampled sequences), both layer pairs.
* a step captured in a CUDA graph (compression on the second stream) writes
  what the eager step writes, bit for bit.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from gpu_helpers import (ATOL_BF16, ATOL_LP, REL_BF16, REL_LP, assert_close, assert_fold_close, check_topk, layer_entries,
                         make_layer, ring_window, stored_bf16, stored_fp4)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


@pytest.mark.parametrize("sharp", [False, True])
def test_tiny_decode_end_to_end(ck, orc, sharp):
    from compressed_sparse_kv_02_b200 import synth
    cfg = synth.CONFIGS["tiny"]
    n, H, d, HI, DI, k = cfg.ctx, cfg.heads, cfg.d_qk, cfg.heads_idx, cfg.d_idx, cfg.k
    steps = 8
    t0 = n - steps
    x, z = synth.raw_stream(1, n, d, cfg.seed, 1)
    xi, zi = synth.raw_stream(1, n, DI, cfg.seed, 3)
    x2, z2 = synth.raw_stream(1, n, d, cfg.seed, 5)
    if sharp:  # values of order 1: the absolute tolerance has teeth
        x = (x.float() * math.sqrt(d)).to(torch.bfloat16)
        x2 = (x2.float() * math.sqrt(d)).to(torch.bfloat16)
    q, q_idx, w = synth.decode_queries(steps, H, d, HI, DI, cfg.seed, 7, q_scale=math.sqrt(d) if sharp else 1.0)
    q2, _, _ = synth.decode_queries(steps, H, d, HI, DI, cfg.seed, 11, q_scale=math.sqrt(d) if sharp else 1.0)
    dev = "cuda"
    X, Z, XI, ZI, X2, Z2 = (t.to(dev) for t in (x, z, xi, zi, x2, z2))
    Lc = make_layer(ck.LAYER_CSA, 4, d, d, 1, n // 4, d_idx=DI, seed=21)
    Lh = make_layer(ck.LAYER_HCA, 128, d, d, 1, n // 128, seed=22)
    seq = torch.zeros(1, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    nb_h = (t0 // 128) * 128
    ck.csa_compress_kv(Lc, seq, 0, X[:, :t0].contiguous(), Z[:, :t0].contiguous(), XI[:, :t0].contiguous(),
                       ZI[:, :t0].contiguous(), status=status)
    ck.hca_compress_kv(Lh, seq, 0, X2[:, :nb_h].contiguous(), Z2[:, :nb_h].contiguous(), status=status)
    r0 = torch.tensor([t0 - 128], device=dev)
    sl = slice(t0 - 128, t0)
    ck.cskv_cache_append(Lc, seq, r0, X[:, sl].contiguous(), Z[:, sl].contiguous(), XI[:, sl].contiguous(),
                         ZI[:, sl].contiguous(), ring_only=True, status=status)
    ck.cskv_cache_append(Lh, seq, r0, X2[:, sl].contiguous(), Z2[:, sl].contiguous(), ring_only=True, status=status)
    # HCA tokens nb_h .. t0-1 exist only in the ring until their block completes at t = n-1
    res = []
    for s in range(steps):
        t = t0 + s
        pos = torch.tensor([t], device=dev)
        ts = slice(t, t + 1)
        ck.cskv_cache_append(Lc, seq, pos, X[:, ts].contiguous(), Z[:, ts].contiguous(), XI[:, ts].contiguous(),
                             ZI[:, ts].contiguous(), status=status)
        ck.cskv_cache_append(Lh, seq, pos, X2[:, ts].contiguous(), Z2[:, ts].contiguous(), status=status)
        idx = torch.zeros(1, k, dtype=torch.int32, device=dev)
        cnt = torch.zeros(1, dtype=torch.int32, device=dev)
        ck.csa_index_score_topk(Lc, seq, pos, t, q_idx[s:s + 1].to(dev), w[s:s + 1].to(dev), k, idx, cnt,
                                status=status)
        oc = torch.zeros(1, H, d, dtype=torch.bfloat16, device=dev)
        lc = torch.zeros(1, H, device=dev)
        ck.csa_attend(Lc, seq, pos, t, q[s:s + 1].to(dev), idx, cnt, oc, lc, status=status)
        oh = torch.zeros(1, H, d, dtype=torch.bfloat16, device=dev)
        lh = torch.zeros(1, H, device=dev)
        ck.hca_attend(Lh, seq, pos, t, q2[s:s + 1].to(dev), oh, lh, status=status)
        res.append((t, idx.cpu().numpy()[0], int(cnt[0]), oc.float().cpu().numpy()[0], lc.cpu().numpy()[0],
                    oh.float().cpu().numpy()[0], lh.cpu().numpy()[0]))
    assert ck.cskv_get_status(status) == ck.OK

    # stage 1: every stored entry (bulk-folded and decode-emitted) vs the oracle fold of the raw stream
    ref_c = orc.store(orc.compress(stored_bf16(x[0]), stored_bf16(z[0]), 4), orc.BF16)
    ref_i = orc.store(orc.compress(stored_bf16(xi[0]), stored_bf16(zi[0]), 4), orc.BF16)
    ref_h = orc.store(orc.compress(stored_bf16(x2[0]), stored_bf16(z2[0]), 128), orc.BF16)
    gc, gh = layer_entries(Lc, 0, n // 4), layer_entries(Lh, 0, n // 128)
    assert_fold_close(orc.decode(gc["kv"]), orc.decode(ref_c), orc.decode(stored_bf16(x[0])), 4, "csa kv")
    assert_fold_close(orc.decode(gc["idx"]), orc.decode(ref_i), orc.decode(stored_bf16(xi[0])), 4, "csa idx")
    assert_fold_close(orc.decode(gh["kv"]), orc.decode(ref_h), orc.decode(stored_bf16(x2[0])), 128, "hca kv")

    scale = 1.0 / math.sqrt(d)
    swaps = 0
    for s, (t, idx, cnt, oc, lc, oh, lh) in enumerate(res):
        nv = orc.visible_entries(t, 4, 128)
        win = stored_bf16(x[0, t - 127:t + 1])
        win2 = stored_bf16(x2[0, t - 127:t + 1])
        qs, q2s = stored_bf16(q[s]), stored_bf16(q2[s])
        qis, ws = stored_bf16(q_idx[s]), w[s].double().numpy()
        # stage 2: selection on the GPU's stored indexer keys, with the tie band
        sc = orc.index_scores(qis, ws, gc["idx"], nv)
        swaps += check_topk(idx, cnt, sc, k)
        # stage 3: attention on the GPU's selection and stored entries
        keys = np.vstack([orc.decode(win), orc.decode(gc["kv"])[idx[:cnt]]])
        o, l = orc.attend(qs, orc.f64(keys), d, scale)
        assert_close(oc, o, ATOL_BF16, REL_BF16, "csa stage t=%d" % t)
        assert np.allclose(lc, l, atol=2e-3, rtol=0)
        o, l = orc.hca_query(t, 128, 128, q2s, win2, gh["kv"], d, scale)
        assert_close(oh, o, ATOL_BF16, REL_BF16, "hca stage t=%d" % t)
        assert np.allclose(lh, l, atol=2e-3, rtol=0)
        # end to end from the raw tokens (the oracle's own fold and selection)
        ridx, _, o, _ = orc.csa_query(t, 4, 128, k, qs, qis, ws, win, ref_c, ref_i, d, scale)
        if set(ridx[:cnt].tolist()) == set(idx[:cnt].tolist()):
            assert_close(oc, o, ATOL_BF16, REL_BF16, "csa e2e t=%d" % t)
        o, _ = orc.hca_query(t, 128, 128, q2s, win2, ref_h, d, scale)
        assert_close(oh, o, ATOL_BF16, REL_BF16, "hca e2e t=%d" % t)
    assert swaps <= 2 * steps


def _fullsize(ck, orc, name, sample_b, sample_heads):
    from compressed_sparse_kv_02_b200 import decode
    from compressed_sparse_kv_02_b200 import synth
    cfg = synth.CONFIGS[name]
    model = decode.DecodeModel(cfg)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    csa, hca = model.layers[0], model.layers[1]
    out = model.out[0]
    inp = model.inputs[0]
    t = cfg.ctx - 1
    nv = orc.visible_entries(t, 4, 128)
    nv_h = orc.visible_entries(t, 128, 128)
    scale = 1.0 / math.sqrt(cfg.d_qk)
    for b in sample_b:
        ent = layer_entries(csa, b, nv)
        sc = orc.index_scores(stored_bf16(inp["q_idx"][b]), inp["w"][b].double().cpu().numpy(), ent["idx"], nv)
        idx = out["idx"][b].cpu().numpy()
        cnt = int(out["cnt"][b])
        check_topk(idx, cnt, sc, cfg.k)
        if cfg.planted_frac:
            planted = set(model.planted[0][b].cpu().numpy().tolist())
            assert len(planted) >= cfg.k and set(idx[:cnt].tolist()) <= planted
        heads = np.array(sample_heads)
        win = ring_window(csa, b, t)
        keys = np.vstack([orc.decode(win), orc.decode(ent["kv"].take_rows(idx[:cnt]))])
        q = inp["q_csa"][b][heads]
        o, _ = orc.attend(stored_bf16(q), orc.f64(keys), cfg.d_v, scale)
        assert_close(out["o_csa"][b][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "csa b=%d" % b)
        hent = layer_entries(hca, b, nv_h)["kv"]
        o, _ = orc.hca_query(t, 128, 128, stored_bf16(inp["q_hca"][b][heads]), ring_window(hca, b, t), hent,
                             cfg.d_v, scale)
        assert_close(out["o_hca"][b][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "hca b=%d" % b)
    # the step is repeatable: a second run gives identical outputs
    before = {k_: v.clone() for k_, v in out.items()}
    model.step()
    torch.cuda.synchronize()
    for k_, v in out.items():
        assert torch.equal(v, before[k_]), k_


def test_flash_fullsize_sampled(ck, orc):
    _fullsize(ck, orc, "flash", sample_b=[0, 31], sample_heads=list(range(0, 32, 5)))


def test_pro_fullsize_sampled(ck, orc):
    _fullsize(ck, orc, "pro", sample_b=[0, 7], sample_heads=[0, 1, 63, 64, 127])


def _mixed_checks(orc, model, cfg, lens, sample, heads):
    """Selections (tie band, oracle scores on the stored FP4 keys) and both attentions (FP8 keys,
    5e-2) of the sampled sequences, in both layer pairs."""
    scale = 1.0 / math.sqrt(cfg.d_qk)
    heads = np.array(heads)
    for li in range(2):
        csa, hca = model.layers[2 * li], model.layers[2 * li + 1]
        out, inp = model.out[li], model.inputs[li]
        for b in sample:
            t = int(lens[b]) - 1
            nv = orc.visible_entries(t, 4, 128)
            nv_h = orc.visible_entries(t, 128, 128)
            ent = layer_entries(csa, b, nv)
            qi = stored_fp4(inp["q_idx"][b], inp["q_idx_scale"][b])
            sc = orc.index_scores(qi, inp["w"][b].double().cpu().numpy(), ent["idx"], nv)
            idx = out["idx"][b].cpu().numpy()
            cnt = int(out["cnt"][b])
            check_topk(idx, cnt, sc, cfg.k)
            keys = np.vstack([orc.decode(ring_window(csa, b, t)), orc.decode(ent["kv"].take_rows(idx[:cnt]))])
            o, _ = orc.attend(stored_bf16(inp["q_csa"][b][heads]), orc.f64(keys), cfg.d_v, scale)
            assert_close(out["o_csa"][b][heads].float().cpu().numpy(), o, ATOL_LP, REL_LP,
                         "csa pair %d b=%d" % (li, b))
            hent = layer_entries(hca, b, nv_h)["kv"]
            o, _ = orc.hca_query(t, 128, 128, stored_bf16(inp["q_hca"][b][heads]), ring_window(hca, b, t), hent,
                                 cfg.d_v, scale)
            assert_close(out["o_hca"][b][heads].float().cpu().numpy(), o, ATOL_LP, REL_LP,
                         "hca pair %d b=%d" % (li, b))


def test_mixed_fp8_fp4_two_pairs(ck, orc):
    from compressed_sparse_kv_02_b200 import decode, synth
    cfg = synth.Config("mixed_small", 4, 1 << 16, 128, 576, 512, 8, 128, 1024, seed=4, kv_dtype="fp8",
                       idx_dtype="fp4")
    lens = synth.mixed_lengths(cfg, lo=4096, hi=1 << 16)
    lens[0] = 4096  # a sequence whose last token completes an HCA block (the append emits an entry)
    model = decode.DecodeModel(cfg, ctx_lens=lens, n_pairs=2)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    _mixed_checks(orc, model, cfg, lens, range(len(lens)), [0, 5, 64, 127])


def test_graph_replayed_step_matches_eager(ck):
    """A decode step captured in a CUDA graph (the form the benchmark times: the compression of the
    completed entries on a second stream, forked and joined through events) writes what the eager step
    writes: both layer pairs' outputs, the new ring rows and the entries the appends emit, bit for bit.
    The outputs, the new rows and the emitted entries are cleared before the replay, so each must come
    from it; a sequence whose last token completes both a CSA and an HCA block makes both appends emit."""
    from compressed_sparse_kv_02_b200 import decode, synth
    cfg = synth.Config("mixed_small", 4, 1 << 16, 128, 576, 512, 8, 128, 1024, seed=4, kv_dtype="fp8",
                       idx_dtype="fp4")
    lens = synth.mixed_lengths(cfg, lo=4096, hi=1 << 16)
    lens[0] = 4096
    model = decode.DecodeModel(cfg, ctx_lens=lens, n_pairs=2)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    t = lens[0] - 1
    rings = ("ring_x", "ring_z", "ring_xi", "ring_zi")

    def snapshot():
        snap = {}
        for li, d in model.out.items():
            for k_, v in d.items():
                snap["out%d.%s" % (li, k_)] = v.clone()
        for i, L in enumerate(model.layers):
            for r in rings:
                if getattr(L, r) is not None:
                    snap["L%d.%s" % (i, r)] = getattr(L, r)[0][t % cfg.n_win].clone()
            j = (t + 1) // L.m - 1
            for k_, v in L.read_entries(0, 1, j0=j).items():
                snap["L%d.%s" % (i, k_)] = v.clone()
        return snap

    eager = snapshot()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        model.step(stream)
    for d in model.out.values():
        for v in d.values():
            v.zero_()
    for L in model.layers:
        for r in rings:
            if getattr(L, r) is not None:
                getattr(L, r)[0][t % cfg.n_win].zero_()
        j = (t + 1) // L.m - 1
        e = L.read_entries(0, 1, j0=j)
        L.write_entries(0, j, **{k_: torch.zeros_like(v) for k_, v in e.items()})
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        graph.replay()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    replayed = snapshot()
    for k_, v in eager.items():
        assert torch.equal(v, replayed[k_]), k_


def test_mixed_fullsize_sampled(ck, orc):
    """The mixed workload at the benchmark's own size and launch configuration: B = 64 sequences with
    log-uniform lengths up to ~1M (FP8 KV, FP4 indexer, layers CSA, HCA, CSA, HCA); the shortest and the
    longest sequence and four others drawn at random, in both layer pairs."""
    from compressed_sparse_kv_02_b200 import decode, synth
    cfg = synth.CONFIGS["mixed"]
    lens = synth.mixed_lengths(cfg)
    model = decode.DecodeModel(cfg, ctx_lens=lens, n_pairs=2)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    order = np.argsort(np.asarray(lens))
    rng = np.random.default_rng(5)
    others = rng.choice(order[1:-1], size=4, replace=False).tolist()
    _mixed_checks(orc, model, cfg, lens, [int(order[0]), int(order[-1])] + others, [0, 37, 64, 127])
