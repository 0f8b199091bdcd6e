"""Host-side checks of the benchmark: the reference arm's line, the rotation of input sets,
the algorithmic bytes behind the roofline and the currency of the committed profiles."""
import io
from contextlib import redirect_stdout

import pytest

from long_context_sparse_clsa_b200.inputs import WORKLOADS


def test_reference_arm_line_matches_the_decode_line():
    """The reference arm times exactly K steps after W warm-up steps and reports the decode
    line's metric, unit, direction and config."""
    import json
    import bench
    args = bench.parse(["--impl", "reference", "--workload", "tiny", "--steps", "4", "--warmup", "3"])
    out = io.StringIO()
    with redirect_stdout(out):
        bench.run_reference(args)
    line = json.loads(out.getvalue())
    w = WORKLOADS["tiny"]
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["higher_is_better"] is True and line["data"] == bench.DATA
    assert line["steps"] == 4 and line["warmup"] == 3
    assert line["config"] == bench.decode_config(w, args, 1, graphs_ok=True)
    assert line["value"] > 0 and line["value"] == pytest.approx(w.B / (line["ms_per_step"] * 1e-3))
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"


def test_rotation_sets_divide_the_timed_steps():
    import bench
    kb = WORKLOADS["decode128k"].B * WORKLOADS["decode128k"].n_max * 128 * 2   # 32 MiB: at least 8 sets
    for steps, want in [(1000, 8), (20, 10), (50, 10), (200, 8), (7, 8), (31, 31), (37, 8)]:
        assert bench.rotation_sets(bench.parse(["--steps", str(steps)]), kb) == want, steps
    assert bench.rotation_sets(bench.parse(["--steps", "20", "--l2", "flush"]), kb) == 1
    big = 64 << 20                                                              # the --sets minimum, 6
    for steps, want in [(20, 10), (1000, 8), (12, 6), (5, 6)]:
        assert bench.rotation_sets(bench.parse(["--steps", str(steps)]), big) == want, steps


def test_algorithmic_bytes_per_step():
    """K_idx scan + the selected K/V rows once + Q and O of every layer + q_idx, per step:
    tiny 1,048,576 + 262,144 + 16,384 + 256; decode32k 8 MiB + 8 MiB + 256 KiB + 256;
    decode128k 32 MiB + 8 MiB + 384 KiB + 256."""
    import bench
    for name, want in [("tiny", 1327360), ("decode32k", 17039616), ("decode128k", 42336512)]:
        w = WORKLOADS[name]
        assert bench.step_bytes(w, [w.n_max] * w.B)["total"] == want, name


def test_committed_profiles_match_the_kernel_sources():
    """The bench reads each dominant kernel's DRAM traffic from its profile summary only while
    the summary's source hash matches the sources; the committed summaries are current."""
    import bench
    fused = ["long_context_sparse_clsa_b200/csrc/decode_fused.cu", "long_context_sparse_clsa_b200/csrc/common.cuh",
             "long_context_sparse_clsa_b200/csrc/tcgen05.cuh"]
    for wl in ("decode128k", "ragged16"):
        t = bench.profile_traffic("decode_fused_kernel", wl, fused)
        assert t is not None and t > 0, wl
    scan = ["long_context_sparse_clsa_b200/csrc/index_scores.cu", "long_context_sparse_clsa_b200/csrc/common.cuh"]
    assert bench.profile_traffic("index_scores_kernel", "decode128k", scan) is not None


def test_profile_summaries_are_short_text_with_their_commands():
    """Every summary under profiles/ is a few KB of text that gives the ncu command behind it,
    and every ncu command there leaves the clocks alone."""
    import os
    import re
    root = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "profiles")
    names = sorted(os.listdir(root))
    assert names and all(n.endswith((".txt", ".md")) for n in names)
    for n in names:
        text = open(os.path.join(root, n)).read()
        assert len(text.encode()) < 16384, n
        cmds = [m.group(0) for m in re.finditer(r"ncu (?:\\\n#?|[^\n])*", text) if "--" in m.group(0)]
        assert cmds, n
        for c in cmds:
            assert "--clock-control none" in c, (n, c)
