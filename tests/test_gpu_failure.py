"""Failure detection on the GPU without a fault: the library's bounded waits, made to run
out on purpose by a wait that nothing satisfies (clsa_selftest_timeout), end with
CLSA_ERR_TIMEOUT in the workspace and leave the context usable."""
import time

import pytest
import torch

from long_context_sparse_clsa_b200 import clsa
from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_clsa_b200.build import build
    build()
    clsa.load_library()


@pytest.mark.parametrize("which", [0, 1], ids=["count_barrier", "mbarrier"])
def test_bounded_wait_runs_out_and_reports(which):
    ws = clsa.Workspace(512)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    clsa.selftest_timeout(which, ws)
    status, detail = ws.status()  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert (status, detail) == ("CLSA_ERR_TIMEOUT", 900 + which)
    assert 0.15 < elapsed < 10.0  # the 200 ms limit, not a hang
    assert ws.status()[0] == "CLSA_OK"  # reading the status cleared it
    # the context still works: a decode step after the timeout is clean
    w = WORKLOADS["tiny"]
    dv = clsa.to_device(make_inputs(w))
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k)
    torch.cuda.synchronize()
    assert r["ws"].status()[0] == "CLSA_OK"
    assert int(r["count"][0]) == w.k
