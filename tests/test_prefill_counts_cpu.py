"""The prefill bench's algorithmic flop counts (the numerator of its tensor roofline) against an
independent count: per compressed entry, the number of chunk positions that see it (an entry j of
a layer with fold width m is visible to query t iff j m < t + 1 - n_win), instead of the per-query
sum the bench uses. CSA attention is the closed form of the pages' workload: every chunk position
of the 65,536-token chunk on 65,536 cached tokens sees the 128 window rows and a full top-512."""
import types

from compressed_sparse_kv_02_b200 import prefill, synth


def _entry_view_count(m, n_win, t0, t1):
    """sum over t in [t0, t1) of the visible entries, counted per entry: entry j is seen by
    every t >= j m + n_win."""
    total = 0
    j = 0
    while j * m + n_win < t1:
        first = max(t0, j * m + n_win)
        total += t1 - first
        j += 1
    return total


def test_prefill_flops_match_an_independent_count():
    cfg = synth.CONFIGS["prefill"]
    c0 = t = 65536
    fake = types.SimpleNamespace(cfg=cfg, cached=c0, chunk=t)
    fl = prefill.PrefillModel.flops(fake)
    per_key = 2 * (cfg.d_qk + cfg.d_v) * cfg.heads
    assert fl["csa_attend"] == t * (cfg.n_win + cfg.k) * per_key == 65536 * 64 * 640 * 512
    seen_h = _entry_view_count(cfg.m_hca, cfg.n_win, c0, c0 + t)
    assert fl["hca_attend"] == (t * cfg.n_win + seen_h) * per_key
    seen_c = _entry_view_count(cfg.m_csa, cfg.n_win, c0, c0 + t)
    assert fl["index"] == seen_c * cfg.heads_idx * cfg.d_idx * 2
    assert fl["total"] == fl["index"] + fl["csa_attend"] + fl["hca_attend"]
    # the magnitudes the workload description gives: ~0.82, ~1.37 and ~1.92 TFLOP
    assert abs(fl["index"] / 1e12 - 0.82) < 0.01
    assert abs(fl["csa_attend"] / 1e12 - 1.37) < 0.01
    assert abs(fl["hca_attend"] / 1e12 - 1.92) < 0.01


def test_prefill_flops_of_a_short_chunk_by_brute_force():
    cfg = synth.Config("small", 1, 512, 4, 16, 16, 2, 8, 8, seed=0)
    fake = types.SimpleNamespace(cfg=cfg, cached=128, chunk=384)
    fl = prefill.PrefillModel.flops(fake)
    per_key = 2 * (cfg.d_qk + cfg.d_v) * cfg.heads
    fi = fc = fh = 0
    for q in range(128, 512):
        vis_c = [j for j in range(q) if j * cfg.m_csa < q + 1 - cfg.n_win]
        vis_h = [j for j in range(q) if j * cfg.m_hca < q + 1 - cfg.n_win]
        win = len(range(max(0, q - cfg.n_win + 1), q + 1))
        fi += len(vis_c) * cfg.heads_idx * cfg.d_idx * 2
        fc += (win + min(cfg.k, len(vis_c))) * per_key
        fh += (win + len(vis_h)) * per_key
    assert (fl["index"], fl["csa_attend"], fl["hca_attend"]) == (fi, fc, fh)
