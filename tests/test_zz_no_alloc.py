"""csa_index_score_topk_static: the indexer for callers that cannot allocate.

Some callers cannot get device memory where they call the indexer -- a plugin
inside a host engine that owns all device memory and gives plugins no
workspace, or a latency-critical loop that must not call cudaMalloc. The
static entry point uses a fixed scratch array inside the library instead of a
caller-provided workspace. This test calls it through the C ABI and checks
its output against csa_index_score_topk's on two calls in a row (different
shapes, so the shared scratch's leftovers from the first call must not leak
into the second), plus the rejection of a request beyond the scratch size.

The file sorts last so that a stop-at-first-failure run has already run
every other test; it passes alone in a fresh process as well (the first call
on the device sets the scratch up).
"""
import ctypes

import numpy as np
import pytest
import torch

from gpu_helpers import make_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def _case(ck, positions, hi, di, k, seed):
    B = len(positions)
    n_e = max(positions) // 4 + 2
    L = make_layer(ck.LAYER_CSA, 4, 128, 128, B, n_e, d_idx=di, seed=seed)
    g = torch.Generator().manual_seed(seed)
    for b in range(B):
        L.write_entries(b, 0, idx=torch.randn(n_e, di, generator=g).to(torch.bfloat16).cuda())
    q_idx = torch.randn(B, hi, di, generator=g).to(torch.bfloat16).cuda()
    w = torch.rand(B, hi, generator=g).cuda()
    seq = torch.arange(B, dtype=torch.int32, device="cuda")
    pos = torch.tensor(positions, dtype=torch.int64, device="cuda")
    return L, q_idx, w, seq, pos


def _outputs(B, k):
    return (torch.full((B, k), -5, dtype=torch.int32, device="cuda"),
            torch.full((B,), -5, dtype=torch.int32, device="cuda"),
            torch.full((B, k), -5.0, device="cuda"))


def _static_call(ck, L, q_idx, w, seq, pos, max_pos, k, outs, status):
    from compressed_sparse_kv_02_b200 import _binding as b
    a = b._index_args(L, seq, pos, max_pos, q_idx, w, k, outs[0], outs[1], outs[2], None, status)
    return ck.lib().csa_index_score_topk_static(ctypes.byref(a), b._stream(None))


def test_static_scratch_matches_workspace_entry_point(ck):
    cases = [
        # (positions, heads, dims, k): a large call first, then a smaller one with other shapes
        ([127 + 4 * 300000 + 1, 127 + 4 * 90000, 127 + 4 * 30000 + 3], 8, 128, 1024),
        ([127 + 4 * 5000, 60, 127 + 4 * 700 + 2, 127 + 4 * 20000], 4, 64, 512),
    ]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for i, (positions, hi, di, k) in enumerate(cases):
        L, q_idx, w, seq, pos = _case(ck, positions, hi, di, k, seed=40 + i)
        B, max_pos = len(positions), max(positions)
        ref = _outputs(B, k)
        ck.csa_index_score_topk(L, seq, pos, max_pos, q_idx, w, k, *ref, status=status)
        got = _outputs(B, k)
        rc = _static_call(ck, L, q_idx, w, seq, pos, max_pos, k, got, status)
        assert rc == ck.OK, ck.status_string(rc)
        assert ck.cskv_get_status(status) == ck.OK
        assert torch.equal(got[1], ref[1])
        assert torch.equal(got[0], ref[0])
        keff = ref[1].cpu().numpy()
        gs, rs = got[2].cpu().numpy(), ref[2].cpu().numpy()
        for b in range(B):
            n = int(keff[b])
            assert np.allclose(gs[b, :n], rs[b, :n], rtol=1e-4, atol=1e-4 * max(1.0, np.abs(rs[b, :n]).max(initial=0.0)))
            assert np.all(gs[b, n:] == 0)


def test_static_scratch_rejects_requests_beyond_its_size(ck):
    from compressed_sparse_kv_02_b200 import _binding as b
    L, q_idx, w, seq, pos = _case(ck, [127 + 4 * 100], 4, 64, 16, seed=50)
    outs = _outputs(1, 16)
    before = [t.clone() for t in outs]
    # max_pos sizes the scratch: 1 query x 2^24 visible entries is 64 MiB of scores
    rc = _static_call(ck, L, q_idx, w, seq, pos, (1 << 26), 16, outs, None)
    assert rc == ck.ERR_WORKSPACE
    torch.cuda.synchronize()
    for t, t0 in zip(outs, before):
        assert torch.equal(t, t0)  # nothing was launched
