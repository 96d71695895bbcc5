"""The decode bench's algorithmic byte counts (the numerator of its HBM roofline) against the
workloads' closed forms: at a 2^20-token context the query sees 262,112 CSA entries and 8,191
HCA entries (an entry j of fold width m is visible iff j m < t + 1 - 128), attends the 128 window
rows plus top-1,024 (CSA) or every visible entry (HCA), and the storage sizes are 256 B per bf16
indexer key, 1,152 B per bf16 latent row, 580 B per FP8 entry (codes + fp32 scale) and 72 B per
FP4 indexer key (codes + one E4M3 scale per 16 elements)."""
import bench
from compressed_sparse_kv_02_b200 import synth


def test_pro_query_bytes():
    cfg = synth.CONFIGS["pro"]
    b = bench.bytes_per_query(cfg)
    assert b["index"] == 262112 * 256
    assert b["csa_attend"] == (128 + 1024) * 1152
    assert b["hca_attend"] == (128 + 8191) * 1152
    # the indexer op's algorithmic bytes per launch of 8 queries, as the roofline line states them
    assert 8 * b["index"] == 536_805_376
    assert abs(b["total"] / 1e6 - 78.9) < 0.2


def test_mixed_query_bytes_use_the_storage_formats():
    cfg = synth.CONFIGS["mixed"]
    lens = [4096, 1 << 20]
    b = bench.bytes_per_query(cfg, ctx_lens=lens, n_pairs=2)
    want_index = want_csa = want_hca = 0
    for n in lens:
        t = n - 1
        nv = -(-(t + 1 - 128) // 4)
        nv_h = -(-(t + 1 - 128) // 128)
        want_index += nv * 72
        want_csa += 128 * 1152 + min(1024, nv) * 580
        want_hca += 128 * 1152 + nv_h * 580
    # averaged over the batch, two layer pairs per query
    scale = 2 / len(lens)
    assert b["index"] == round(want_index * scale)
    assert b["csa_attend"] == round(want_csa * scale)
    assert b["hca_attend"] == round(want_hca * scale)
