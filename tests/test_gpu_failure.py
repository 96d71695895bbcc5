"""Failure detection on the GPU without a fault: the bounded device wait.

Every mbarrier hand-off in the library's kernels goes through one bounded wait
that gives up after a fixed number of polls, records CSKV_ERR_TIMEOUT in the
caller's status word and lets the kernel return. Here that wait is made to run
out: one warp waits on an mbarrier that nothing arrives at (no asynchronous
copy outstanding), with a short poll limit. The status word must read the
timeout, and the context must stay usable: a following wait that is satisfied
leaves the status clean, and the decode path still runs.
"""
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ck(cskv_built):
    import compressed_sparse_kv_02_b200 as ck
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return ck


def test_wait_that_is_satisfied_reports_nothing(ck):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.cskv_selftest_wait(True, 1000, st)
    assert ck.cskv_get_status(st) == ck.OK


@pytest.mark.parametrize("limit", [1, 1000, 100000])
def test_wait_that_runs_out_reports_timeout(ck, limit):
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.cskv_selftest_wait(False, limit, st)
    assert ck.cskv_get_status(st) == ck.ERR_TIMEOUT
    # read-and-clear: the word is clean again, and the context still works
    assert ck.cskv_get_status(st) == ck.OK
    ck.cskv_selftest_wait(True, limit, st)
    assert ck.cskv_get_status(st) == ck.OK


def test_first_error_wins(ck):
    st = torch.full((1,), ck.ERR_OUT_OF_RANGE, dtype=torch.int32, device="cuda")
    ck.cskv_selftest_wait(False, 100, st)
    assert ck.cskv_get_status(st) == ck.ERR_OUT_OF_RANGE


def test_decode_path_runs_after_a_timeout(ck):
    from compressed_sparse_kv_02_b200 import decode, synth
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ck.cskv_selftest_wait(False, 100, st)
    assert ck.cskv_get_status(st) == ck.ERR_TIMEOUT
    cfg = synth.Config("after_timeout", 2, 4096, 16, 128, 128, 4, 64, 128, seed=5)
    m = decode.DecodeModel(cfg)
    m.fill_synthetic()
    m.step()
    torch.cuda.synchronize()
    assert m.check_status() == ck.OK
