"""The N > 1 path of the benchmark on CPU: two gloo ranks run the replica plumbing that
bench.py uses on GPUs (process group from the torchrun environment, each rank's own
seeded sequences, the max-over-ranks step time, the whole-job rate), and the reference
arm's rule that only rank 0 times the oracle."""
import io
import os
import socket
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch.multiprocessing as mp

from long_context_sparse_clsa_b200 import replicas
from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    try:
        r, wsz, local = replicas.init("gloo", timeout_s=60)
        w = replicas.rank_workload(WORKLOADS["tiny"], r, wsz)
        inp = make_inputs(w)
        replicas.barrier(wsz)
        step_ms = 2.0 + 3.0 * r  # this rank's (made-up) device time
        slowest = replicas.max_over_ranks(step_ms, wsz)
        q.put((r, wsz, local, w.seed, inp.q_idx.astype(np.float64).sum(), slowest,
               replicas.job_rate(wsz, w.B, slowest)))
        replicas.finish(wsz)
    except Exception as ex:  # report instead of hanging the parent
        q.put(("error", rank, repr(ex)))


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert not [g for g in got if g[0] == "error"], got
    got.sort()
    (r0, w0, l0, s0, q0, m0, v0), (r1, w1, l1, s1, q1, m1, v1) = got
    assert (r0, r1, w0, w1, l0, l1) == (0, 1, 2, 2, 0, 1)
    base = WORKLOADS["tiny"]
    assert (s0, s1) == (base.seed, base.seed + 1)  # each rank its own sequences
    assert q0 != q1
    assert q0 == make_inputs(base).q_idx.astype(np.float64).sum()  # rank 0 = the seeded workload
    assert m0 == m1 == 5.0  # the slowest rank's time, on every rank
    assert v0 == v1 == pytest.approx(2 * base.B / 5e-3)  # every rank's units over the slowest time


def test_single_process_needs_no_group():
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        assert k not in os.environ or os.environ[k] in ("0", "1")
    w = WORKLOADS["tiny"]
    assert replicas.rank_workload(w, 0, 1) is w
    assert replicas.max_over_ranks(3.5, 1) == 3.5
    assert replicas.job_rate(1, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = bench.parse(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--gpus", "2"])
    out = io.StringIO()
    with redirect_stdout(out):
        assert bench.run_reference(args) is None
    assert out.getvalue() == ""

