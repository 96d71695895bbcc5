"""GPU parity of one prefill pass (PrefillModel), at reduced size and at the
benchmark's full size.

A sequence with 8192 cached tokens receives a chunk of 2048 new tokens
(H = 64, d = 128, indexer 4 x 64, top-512), in two blocks of 1024 query
positions; at full size 65536 new tokens on 65536 cached, in blocks of 4096. Checked against the oracle: the chunk's compressed entries (from
the chunk's raw rows), the top-k and both attentions of sampled positions
(window rows from the chunk or, before the chunk, from the restored ring),
the rings after the pass, and that a second pass gives identical outputs.
"""
import math

import numpy as np
import pytest
import torch

from gpu_helpers import (ATOL_BF16, REL_BF16, assert_close, assert_fold_close, check_topk, layer_entries,
                         stored_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def _check_prefill(ck, orc, model, positions, heads_of):
    """The chunk's compressed entries (from its raw rows), the top-k and both attentions at the given
    positions (heads_of(t) -> head indices; window rows from the chunk or, before it, from the
    restored ring), the rings after the pass, and that a second pass gives identical outputs."""
    cfg, c0, T = model.cfg, model.cached, model.chunk
    csa, hca = model.layers
    inp = model.inputs
    for L, xs, zs, m in ((csa, "x", "z", 4), (hca, "x_h", "z_h", 128)):
        got = L.read_entries(0, T // m, c0 // m)
        x, z = inp[xs][0].cpu(), inp[zs][0].cpu()
        ref = orc.store(orc.compress(stored_bf16(x), stored_bf16(z), m), orc.BF16)
        assert_fold_close(orc.decode(stored_bf16(got["kv"])), orc.decode(ref), orc.decode(stored_bf16(x)), m,
                          "entries m=%d" % m)
        if L is csa:
            ref_i = orc.store(orc.compress(stored_bf16(inp["xi"][0].cpu()), stored_bf16(inp["zi"][0].cpu()), m),
                              orc.BF16)
            assert_fold_close(orc.decode(stored_bf16(got["idx"])), orc.decode(ref_i),
                              orc.decode(stored_bf16(inp["xi"][0].cpu())), m, "indexer entries")
    # raw rows of every position, for the windows: the cached tail, then the chunk
    tail = {"x": inp["tail_x"][0].cpu(), "x_h": inp["tail_x_h"][0].cpu()}

    def window(name, t):
        rows = []
        for p in range(max(0, t - 127), t + 1):
            rows.append(inp[name][0, p - c0].cpu() if p >= c0 else tail[name][p - (c0 - 128)])
        return stored_bf16(torch.stack(rows))

    scale = 1.0 / math.sqrt(cfg.d_qk)
    ent_all = layer_entries(csa, 0, orc.visible_entries(c0 + T - 1, 4, 128))
    hent_all = layer_entries(hca, 0, orc.visible_entries(c0 + T - 1, 128, 128))["kv"]
    for t in positions:
        i = t - c0
        heads = np.asarray(heads_of(t))
        nv = orc.visible_entries(t, 4, 128)
        nv_h = orc.visible_entries(t, 128, 128)
        sc = orc.index_scores(stored_bf16(inp["q_idx"][i]), inp["w"][i].double().cpu().numpy(), ent_all["idx"], nv)
        idx = model.idx[i].cpu().numpy()
        cnt = int(model.cnt[i])
        check_topk(idx, cnt, sc, cfg.k)
        keys = np.vstack([orc.decode(window("x", t)), orc.decode(ent_all["kv"].take_rows(idx[:cnt]))])
        o, _ = orc.attend(stored_bf16(inp["q"][i][heads]), orc.f64(keys), cfg.d_v, scale)
        assert_close(model.o_csa[i][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "csa t=%d" % t)
        o, _ = orc.hca_query(t, 128, 128, stored_bf16(inp["q_h"][i][heads]), window("x_h", t),
                             hent_all.take_rows(np.arange(nv_h)), cfg.d_v, scale)
        assert_close(model.o_hca[i][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "hca t=%d" % t)
    # the rings end with the chunk's last 128 rows (slot p % 128)
    for L, name in ((csa, "x"), (hca, "x_h")):
        for p in (c0 + T - 128, c0 + T - 1):
            assert torch.equal(L.ring_x[0][p % 128], inp[name][0, p - c0])
    # the pass repeats on the same state
    before = [model.idx.clone(), model.o_csa.clone(), model.o_hca.clone()]
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    for a, b in zip(before, [model.idx, model.o_csa, model.o_hca]):
        assert torch.equal(a, b)


def test_prefill_chunk(ck, orc):
    from compressed_sparse_kv_02_b200 import prefill, synth
    cfg = synth.Config("prefill_small", 1, 8192 + 2048, 64, 128, 128, 4, 64, 512, seed=3)
    c0, T = 8192, 2048
    model = prefill.PrefillModel(cfg, cached=c0, chunk=T, q_block=1024)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    _check_prefill(ck, orc, model, (c0, c0 + 1, c0 + 127, c0 + 128, c0 + 1023, c0 + 1024, c0 + T - 1),
                   lambda t: [0, 17, 63])


def test_prefill_fullsize_sampled(ck, orc):
    """The prefill pass at the benchmark's own size and launch configuration: 65536 new tokens on 65536
    cached, query blocks of 4096. Positions at block edges, the chunk's first and last positions and
    twenty drawn at random; every head at five of them, three heads elsewhere."""
    from compressed_sparse_kv_02_b200 import prefill, synth
    cfg = synth.CONFIGS["prefill"]
    c0, T = 65536, 65536
    model = prefill.PrefillModel(cfg, cached=c0, chunk=T, q_block=4096)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    edges = [c0 + 4096 * j + d for j in (1, 8, 15) for d in (-1, 0)]
    rng = np.random.default_rng(11)
    rand = sorted(int(x) for x in rng.integers(c0, c0 + T, size=20))
    positions = [c0, c0 + 1, c0 + 127, c0 + 128] + edges + rand + [c0 + T - 1]
    all_heads = {c0, c0 + 128, c0 + 4096, c0 + 8 * 4096 - 1, c0 + T - 1}
    _check_prefill(ck, orc, model, positions,
                   lambda t: list(range(cfg.heads)) if t in all_heads else [0, 17, 63])


def test_varlen_prefill_several_sequences(ck, orc):
    """Several sequences with their own cached and chunk lengths in one pass: the folds per sequence,
    the indexer and both attentions over query blocks that span sequences (the window rows of each
    from its own packed chunk through the chunk descriptor, or from its ring), and the rings after the
    pass. Blocks of 512 rows cross sequence boundaries; 1024 + 640 + 384 rows in all."""
    from compressed_sparse_kv_02_b200 import prefill, synth
    cfg = synth.Config("prefill_varlen", 3, 6144 + 1024, 64, 128, 128, 4, 64, 256, seed=13)
    cached, chunk = [6144, 1024, 2048], [1024, 640, 384]
    model = prefill.VarlenPrefillModel(cfg, cached, chunk, q_block=512)
    model.fill_synthetic()
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    csa, hca = model.layers
    inp = model.inputs
    scale = 1.0 / math.sqrt(cfg.d_qk)
    heads = np.array([0, 31, 63])
    for b, (c0, T) in enumerate(zip(cached, chunk)):
        r0 = model.row0[b]
        # the chunk's entries, folded from its raw rows
        for L, xs, zs, m in ((csa, "x", "z", 4), (hca, "x_h", "z_h", 128)):
            got = L.read_entries(b, T // m, c0 // m)
            x, z = inp[xs][r0:r0 + T].cpu(), inp[zs][r0:r0 + T].cpu()
            ref = orc.store(orc.compress(stored_bf16(x), stored_bf16(z), m), orc.BF16)
            assert_fold_close(orc.decode(stored_bf16(got["kv"])), orc.decode(ref), orc.decode(stored_bf16(x)), m,
                              "seq %d entries m=%d" % (b, m))

        def window(name, t):
            rows = []
            for p in range(max(0, t - 127), t + 1):
                rows.append(inp[name][r0 + p - c0].cpu() if p >= c0 else
                            inp["tail_" + name][b, p - (c0 - 128)].cpu())
            return stored_bf16(torch.stack(rows))

        for t in (c0, c0 + 1, c0 + 127, c0 + 128, c0 + T // 2 + 3, c0 + T - 1):
            i = r0 + t - c0
            nv = orc.visible_entries(t, 4, 128)
            nv_h = orc.visible_entries(t, 128, 128)
            ent = layer_entries(csa, b, nv)
            sc = orc.index_scores(stored_bf16(inp["q_idx"][i]), inp["w"][i].double().cpu().numpy(), ent["idx"], nv)
            idx = model.idx[i].cpu().numpy()
            cnt = int(model.cnt[i])
            check_topk(idx, cnt, sc, cfg.k)
            keys = np.vstack([orc.decode(window("x", t)), orc.decode(ent["kv"].take_rows(idx[:cnt]))])
            o, _ = orc.attend(stored_bf16(inp["q"][i][heads]), orc.f64(keys), cfg.d_v, scale)
            assert_close(model.o_csa[i][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "seq %d csa t=%d" % (b, t))
            o, _ = orc.hca_query(t, 128, 128, stored_bf16(inp["q_h"][i][heads]), window("x_h", t),
                                 layer_entries(hca, b, nv_h)["kv"], cfg.d_v, scale)
            assert_close(model.o_hca[i][heads].float().cpu().numpy(), o, ATOL_BF16, REL_BF16, "seq %d hca t=%d" % (b, t))
        for L, name in ((csa, "x"), (hca, "x_h")):
            for p in (c0 + T - 128, c0 + T - 1):
                assert torch.equal(L.ring_x[b][p % 128], inp[name][r0 + p - c0])
    # the pass repeats on the same state
    before = [model.idx.clone(), model.o_csa.clone(), model.o_hca.clone()]
    model.step()
    torch.cuda.synchronize()
    assert model.check_status() == ck.OK
    for a, b_ in zip(before, [model.idx, model.o_csa, model.o_hca]):
        assert torch.equal(a, b_)
