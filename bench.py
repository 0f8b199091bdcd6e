#!/usr/bin/env python
"""Benchmark of the CLSA decode step (indexer scan + exact top-k + gather +
L-layer sparse GQA attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload decode128k]
                    [--impl {clsa,reference}] [--no-graph] [--no-cpu-baseline]
                    [--l2 {rotate,flush}] [--sets R]
                    [--variant {clsa,per_layer_routing,yoco_dense,standard,distill_target}]

One JSON line on rank 0.  A step is one decode token per sequence through the
whole path; the default workload is the 128K-context decode (batch 1, n=131072,
d_idx=128, k=2048, L=24, 32 query / 8 KV heads, d=128, bf16, 1% planted tokens).
Device time is measured with CUDA events on the stream the library launches on: one
pair around the K back-to-back steps (``--l2 rotate``), or one pair per step.  Between steps the inputs rotate through R sets whose K_idx
copies together exceed twice the 126 MB L2 (``--l2 rotate``, the default: each step
reads its K_idx and K/V rows from HBM, the kernel code stays cached), or L2 is
flushed by a 512 MiB write and read-back outside the timed events (``--l2 flush``).  With N > 1 every rank runs its own sequences (weak
scaling, no collective on the data path); the step time is the max over ranks.

``--impl reference`` times the CPU oracle (float64 numpy) on the host cores on a
bounded sample of the same workload and prints the same line with
``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CLSA decode step µs & tokens/s at 128K ctx; achieved HBM GB/s vs roofline"
UNIT = "tokens/s"
DATA = "synthetic (seeded N(0,1), 1% planted index keys)"


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="decode128k")
    ap.add_argument("--impl", default="clsa", choices=["clsa", "reference"])
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush"],
                    help="between steps: rotate through input sets larger than L2 (default), or flush L2")
    ap.add_argument("--sets", type=int, default=6, help="input sets rotated through (--l2 rotate)")
    ap.add_argument("--variant", default="clsa",
                    choices=["clsa", "per_layer_routing", "yoco_dense", "standard", "distill_target", "attention_mass"],
                    help="a comparison system built from the library's calls (one GPU; not the default line)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-steps", type=int, default=2)
    return ap.parse_args(argv)


# ------------------------------------------------------------------ algorithmic bytes

def step_bytes(w, lens):
    """K_idx scan + gathered K/V rows once + Q/O + q_idx (per step, all sequences)."""
    e = w.elem_bytes
    kidx = sum(int(n) for n in lens) * w.d_idx * e
    kv = sum(min(w.k, int(n)) for n in lens) * w.Hkv * w.d * e * 2
    qo = 2 * w.L * w.B * w.Hq * w.d * e
    qi = w.B * w.d_idx * e
    return {"kidx": kidx, "kv": kv, "qo": qo, "qidx": qi, "total": kidx + kv + qo + qi}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def profile_traffic(kernel: str, workload: str, src_files):
    """dram bytes per launch recorded in profiles/<kernel>__<workload>.txt, or None
    when the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    h = hashlib.sha256()
    for f in src_files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    if vals.get("source_sha256") != h.hexdigest():
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi streaming its clocks every 25 ms while the timed region runs (started half a
    second ahead, so that the stream is flowing when the region starts)."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self._p = None
        self._t = None

    def _read(self):
        for line in self._p.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9:
                self.samples.append(parts)

    def __enter__(self):
        try:
            self._p = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                        "--format=csv,noheader,nounits", "-lms", "25"],
                                       stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._t = threading.Thread(target=self._read, daemon=True)
            self._t.start()
            time.sleep(0.5)
        except Exception:
            self._p = None
        return self

    def __exit__(self, *a):
        if self._p is not None:
            time.sleep(0.15)
            self._p.terminate()
            try:
                self._p.wait(timeout=5)
            except Exception:
                self._p.kill()
            self._t.join(timeout=5)

    def summary(self):
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [v for v in (num(s[1]) for s in self.samples) if v is not None]
        mx = [v for v in (num(s[2]) for s in self.samples) if v is not None]
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4) if s[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle timing

def time_oracle(inp, w, steps: int):
    """Run the oracle's decode step on the host cores, once with its BLAS pool limited to one
    thread and once with one thread per core this process may use (os.sched_getaffinity).
    Returns (s per step all-cores, cores, s per step single-thread, note)."""
    from oracle import clsa_oracle as O
    # the cache is upcast once (state a real decoder keeps resident); each sample step
    # re-scores, re-selects and attends
    qf = inp.f32("q_idx").astype(np.float64)
    kf = inp.f32("k_idx").astype(np.float64)
    Kf = inp.f32("K").astype(np.float64)
    Vf = inp.f32("V").astype(np.float64)
    Qf = inp.f32("Q").astype(np.float64)
    cores = len(os.sched_getaffinity(0))

    def run(n):
        t0 = time.perf_counter()
        for _ in range(n):
            O.decode_step(qf, kf, Kf, Vf, Qf, inp.seq_lens, w.k)
        return (time.perf_counter() - t0) / n

    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            dt1 = run(1)
        with threadpool_limits(limits=cores):
            dt = run(steps)
    except Exception:  # no control over the BLAS pool: one measurement as it stands
        dt = run(steps)
        dt1 = None
    return dt, cores, dt1, f"{steps} full decode step(s) of {w.name} (B={w.B}, n={w.n_max}); single-thread: 1 step"


# ------------------------------------------------------------------ the decode line's config

def kidx_nbytes(w) -> int:
    return w.B * w.n_max * w.d_idx * w.elem_bytes


def rotation_sets(args, kidx_bytes: int) -> int:
    """Input sets rotated through between steps: with --l2 rotate at least two, and at least
    twice L2 in K_idx alone; one set with --l2 flush.  Above that minimum, the smallest count
    (up to 32) that divides K: the timed steps are then whole replays of the R-step graph,
    with no single-step graphs at the end (each graph launch restarts the launch pipeline)."""
    if args.l2 != "rotate":
        return 1
    r_min = max(2, min(max(1, args.sets), 16), int(np.ceil(2 * 126e6 / kidx_bytes)))
    for r in range(r_min, max(r_min, 32) + 1):
        if args.steps % r == 0:
            return r
    return r_min


def decode_config(w, args, world: int, graphs_ok: bool, kb: int = 0) -> dict:
    """The ``config`` of the decode line (kb: bytes of one K_idx set, by default from the
    workload's shape); the reference arm prints the same one."""
    kb = kb or kidx_nbytes(w)
    R = rotation_sets(args, kb)
    return {"workload": w.name, "B": w.B, "n": w.n_max, "d_idx": w.d_idx, "k": w.k, "L": w.L,
            "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "parallelism": f"replicas x{world}",
            "l2": (f"inputs larger than L2: {R} rotating K_idx sets ({R * kb / 2**20:.0f} MiB, row "
                   f"permutations of the seeded cache), step i uses set i % {R}; no flush"
                   if args.l2 == "rotate" else
                   "flushed before every step (512 MiB write + read-back, outside the timed events)"),
            "launch": (f"cuda graph ({R} steps per graph, one per input set)" if graphs_ok and
                       args.l2 == "rotate" else "cuda graph" if graphs_ok else "eager")}


# ------------------------------------------------------------------ main paths

def run_reference(args):
    """The oracle on the host cores, on the decode line's metric, unit and config: W warm-up
    and exactly K timed steps, each a bounded sample of one decode step.  Step i runs the
    routing in full (scores over the whole cache, then the TopK) and the attention of KV head
    g = i mod Hkv (its G query heads in every layer, the oracle given that head's slice of
    the cache); the attention time is scaled by Hkv, the heads being alike in shape and work."""
    from long_context_sparse_clsa_b200 import replicas
    rank, world, _ = replicas.env_ranks()
    if rank != 0:  # rank 0 alone times the oracle; the other ranks exit without work
        return
    from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs
    from oracle import clsa_oracle as O
    if args.workload.startswith("prefill"):
        raise SystemExit("--impl reference times the decode workloads")
    w = replicas.rank_workload(WORKLOADS[args.workload], 0, world)
    inp = make_inputs(w)
    # the cache is upcast once (state a real decoder keeps resident)
    qf = inp.f32("q_idx").astype(np.float64)
    kf = inp.f32("k_idx").astype(np.float64)
    Kf = inp.f32("K").astype(np.float64)
    Vf = inp.f32("V").astype(np.float64)
    Qf = inp.f32("Q").astype(np.float64)
    cores = len(os.sched_getaffinity(0))
    warmup = max(args.warmup, 3)
    G = w.Hq // w.Hkv

    def sample(i: int):
        g = i % w.Hkv
        t0 = time.perf_counter()
        I = O.index_scores(qf, kf, inp.seq_lens)
        idx, count = O.topk_select(I, inp.seq_lens, w.k)
        t1 = time.perf_counter()
        O.sparse_attention(Qf[:, :, g * G:(g + 1) * G], Kf[:, :, g:g + 1], Vf[:, :, g:g + 1], idx, count)
        return t1 - t0, time.perf_counter() - t1

    import contextlib
    with contextlib.ExitStack() as stack:
        try:
            from threadpoolctl import threadpool_limits
            stack.enter_context(threadpool_limits(limits=cores))
        except Exception:  # no control over the BLAS pool: it runs as it stands
            pass
        for i in range(warmup):
            sample(i)
        route = attn = 0.0
        for i in range(args.steps):
            a, b = sample(warmup + i)
            route += a
            attn += b
    dt = (route + attn * w.Hkv) / args.steps
    v = w.B / dt
    note = (f"each step: the routing of {w.name} (B={w.B}, n={w.n_max}) in full and the attention of one "
            f"of its {w.Hkv} KV heads in turn (all {w.L} layers), scaled by {w.Hkv}")
    line = {"metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": warmup, "ms_per_step": dt * 1e3, "us_per_step": dt * 1e6, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": DATA, "impl": "reference",
            "config": decode_config(w, args, world, graphs_ok=not args.no_graph),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": note},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_clsa(args):
    import torch
    from long_context_sparse_clsa_b200 import replicas
    rank, world, local = replicas.init("nccl")
    torch.cuda.set_device(local)
    from long_context_sparse_clsa_b200 import clsa
    from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs
    clsa.load_library()
    w = replicas.rank_workload(WORKLOADS[args.workload], rank, world)  # each rank its own sequences
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    L, B, Hq, d, k = w.L, w.B, w.Hq, w.d, w.k

    def packed(shapes_dtypes):
        """one device buffer holding several tensors (256-byte aligned views): a step's
        inputs (or outputs) then cross PCIe in one copy"""
        offs, off = [], 0
        for shp, dt in shapes_dtypes:
            off = (off + 255) // 256 * 256
            offs.append(off)
            off += int(np.prod(shp)) * torch.empty((), dtype=dt).element_size()
        buf = torch.empty(off, dtype=torch.uint8, device=dev)
        views = [buf[o:o + int(np.prod(shp)) * torch.empty((), dtype=dt).element_size()].view(dt).view(shp)
                 for (shp, dt), o in zip(shapes_dtypes, offs)]
        return buf, views

    # the per-step inputs q_idx and Q in one buffer, the outputs O, idx, count in another
    in_buf, (qv, Qv) = packed([(tuple(dv["q_idx"].shape), dv["q_idx"].dtype), (tuple(dv["Q"].shape), dv["Q"].dtype)])
    qv.copy_(dv["q_idx"])
    Qv.copy_(dv["Q"])
    dv["q_idx"], dv["Q"] = qv, Qv
    out_buf, (Ov, iv, cv) = packed([(tuple(dv["Q"].shape), dv["Q"].dtype), ((B, k), torch.int32), ((B,), torch.int32)])
    out = {"O": Ov, "idx": iv, "count": cv}
    # Input sets: set 0 is the seeded workload; set r > 0 permutes the rows of every
    # sequence's K_idx (the same scores, planted tokens included, at other positions, so
    # each set selects and gathers other K/V rows).  With --l2 rotate, step i uses set
    # i % R and the R K_idx copies together exceed L2, so every step streams its K_idx
    # and K/V rows from HBM while the kernel code stays cached; with --l2 flush, one set
    # and a 512 MiB write + read-back before every step.
    kidx_bytes = dv["k_idx"].numel() * dv["k_idx"].element_size()
    R = rotation_sets(args, kidx_bytes)
    gen = torch.Generator(device="cpu").manual_seed(1234 + rank)
    kidx_sets = [dv["k_idx"]]
    for r in range(1, R):
        kr = dv["k_idx"].clone()
        for b in range(B):
            nb = int(inp.seq_lens[b])
            perm = torch.randperm(nb, generator=gen).to(dev)
            kr[b, :nb] = dv["k_idx"][b, perm]
        kidx_sets.append(kr)
    args_sets = [clsa.decode_args(dv["q_idx"], kx, dv["K"], dv["V"], dv["Q"], dv["seq_lens"], k, out["O"],
                                  out["idx"], out["count"]) for kx in kidx_sets]
    a = args_sets[0]
    ws = clsa.Workspace(clsa.decode_workspace_size(a))
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    flush_view = flush.view(torch.int32)

    def flush_l2():
        # write 512 MiB, then read 512 MiB back: every line the step may touch is evicted
        # and the dirty lines of the write are written back before the timed events
        flush.fill_(1)
        flush_view.max()

    def between_steps():
        if args.l2 == "flush":
            flush_l2()

    def step(r=0):
        clsa.decode_step_args(args_sets[r], ws)

    step()
    torch.cuda.synchronize()
    launches_per_step = clsa.last_launch_count()
    graphs = round_graph = None
    if not args.no_graph:
        try:
            s2 = torch.cuda.Stream()
            s2.wait_stream(stream)
            with torch.cuda.stream(s2):
                step()
            stream.wait_stream(s2)
            torch.cuda.synchronize()
            graphs = []
            for r in range(R):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    step(r)
                graphs.append(g)
            # the R steps of one rotation in one graph: consecutive steps keep the launch's
            # programmatic serialization (the next step's launch overlaps this one's run)
            round_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(round_graph):
                for r in range(R):
                    step(r)
            torch.cuda.synchronize()
        except Exception as ex:  # graph capture unsupported: time eager launches
            graphs = round_graph = None
            print(f"# graph capture failed, timing eager launches: {ex}", file=sys.stderr)

    def run_step(i):
        if graphs is not None:
            graphs[i % R].replay()
        else:
            step(i % R)

    def run_steps(n):
        """n steps, set i % R for step i: whole rotations from the R-step graph"""
        i = 0
        if graphs is not None:
            while n - i >= R:
                round_graph.replay()
                i += R
        while i < n:
            run_step(i)
            i += 1

    for i in range(max(args.warmup, 3, R)):
        between_steps()
        run_step(i)
    if round_graph is not None and args.l2 == "rotate":
        round_graph.replay()  # the first replay uploads the graph
    torch.cuda.synchronize()

    def barrier():
        replicas.barrier(world)
        torch.cuda.synchronize()

    # The timed region: K steps back to back on the stream, one event pair around them (with
    # --l2 flush, one pair per step so that the flushes stay outside the timed events).
    barrier()
    with ClockSampler(local) as clk:
        if args.l2 == "rotate":
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            run_steps(args.steps)
            e1.record(stream)
            torch.cuda.synchronize()
            total_ms = e0.elapsed_time(e1)
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for i, (a0, a1) in enumerate(evs):
                between_steps()
                a0.record(stream)
                run_step(i)
                a1.record(stream)
            torch.cuda.synchronize()
            total_ms = sum(a0.elapsed_time(a1) for a0, a1 in evs)
    barrier()
    st = ws.status()
    if st[0] != "CLSA_OK":
        raise RuntimeError(f"device error during timing: {st}")
    total_ms = replicas.max_over_ranks(total_ms, world, dev)
    ms_per_step = total_ms / args.steps
    value = replicas.job_rate(world, B, ms_per_step)

    # ---- per-kernel timing: each C-ABI stage alone, back to back over the R input sets -------
    # Each stage is captured once per input set into one CUDA graph (R calls, set r's inputs
    # in call r) and the graph is replayed between one event pair, so the per-call time is the
    # device time of a stream of such calls, with no host marshalling in it.  index_scores
    # and gather_kv then read their K_idx / K/V rows from HBM (the R sets exceed L2 with
    # --l2 rotate); the attention calls read the compact K_S/V_S that gather_kv wrote, which
    # a step has just produced and which stay in L2 (8 MiB per set at 128K).
    lib = clsa.load_library()
    sc_sets = [torch.empty(B, w.n_max, dtype=torch.float32, device=dev) for _ in range(R)]
    idx_sets = [torch.empty(B, k, dtype=torch.int32, device=dev) for _ in range(R)]
    cnt_sets = [torch.empty(B, dtype=torch.int32, device=dev) for _ in range(R)]
    KS_sets = [torch.empty(B, k, w.Hkv, d, dtype=dv["K"].dtype, device=dev) for _ in range(R)]
    VS_sets = [torch.empty_like(x) for x in KS_sets]
    tws = clsa.Workspace(max(256, lib.clsa_topk_workspace_size(B, w.n_max, k)))
    attn_ws = clsa.Workspace(lib.clsa_sparse_attn_workspace_size(B, k, L, Hq, w.Hkv, d))
    Q1 = dv["Q"][:1].contiguous()
    O1 = torch.empty_like(Q1)
    stages = {
        "index_scores": lambda r: clsa.index_scores(dv["q_idx"], kidx_sets[r], dv["seq_lens"], sc_sets[r]),
        "topk": lambda r: clsa.topk(sc_sets[r], dv["seq_lens"], k, tws, idx_sets[r], cnt_sets[r]),
        "gather_kv": lambda r: clsa.gather_kv(dv["K"], dv["V"], idx_sets[r], cnt_sets[r], tws, KS_sets[r],
                                              VS_sets[r]),
        "sparse_attn_all_layers": lambda r: clsa.sparse_attn(dv["Q"], KS_sets[r], VS_sets[r], cnt_sets[r],
                                                             ws=attn_ws, O=out["O"], want_lse=False),
        # the model-faithful per-layer call (a model's layer l needs layer l - 1's output first)
        "sparse_attn_one_layer_l2_resident": lambda r: clsa.sparse_attn(Q1, KS_sets[r], VS_sets[r], cnt_sets[r],
                                                                        ws=attn_ws, O=O1, want_lse=False),
    }

    def timed(fn, reps=max(2, 64 // R)):
        for r in range(R):  # eager once: the sets' inputs exist before the next stage runs
            fn(r)
        torch.cuda.synchronize()
        try:
            g = torch.cuda.CUDAGraph()
            s2 = torch.cuda.Stream()
            s2.wait_stream(stream)
            with torch.cuda.stream(s2):
                fn(0)
            stream.wait_stream(s2)
            with torch.cuda.graph(g):
                for r in range(R):
                    fn(r)
            g.replay()
            torch.cuda.synchronize()
            run = g.replay
        except Exception:  # graph capture unsupported: eager calls
            def run():
                for r in range(R):
                    fn(r)
        torch.cuda._sleep(200_000)  # keep the stream busy while the host issues the first call
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / (reps * R) * 1e3  # us per call

    by = step_bytes(w, inp.seq_lens)
    kern = {name: timed(fn) for name, fn in stages.items()}
    kern_method = (f"per call, back to back: a CUDA graph of {R} calls (one per input set) replayed; "
                   "the attention calls read the gathered K_S/V_S from L2")

    hbm, bf16, peak_kind = peaks()
    if launches_per_step == 1:
        # the step is one fused launch: it is the dominant (only) kernel of the timed region
        dom, dom_us, dom_bytes = "decode_fused_kernel", ms_per_step * 1e3, by["total"]
        traffic = profile_traffic("decode_fused_kernel", w.name,
                                  ["long_context_sparse_clsa_b200/csrc/decode_fused.cu",
                                   "long_context_sparse_clsa_b200/csrc/common.cuh",
                                   "long_context_sparse_clsa_b200/csrc/tcgen05.cuh"])
    else:
        dom, dom_us = "index_scores", kern["index_scores"]
        dom_bytes = by["kidx"] + by["qidx"] + 4 * sum(int(n) for n in inp.seq_lens)
        traffic = profile_traffic("index_scores_kernel", w.name, ["long_context_sparse_clsa_b200/csrc/index_scores.cu",
                                                           "long_context_sparse_clsa_b200/csrc/common.cuh"])
    achieved = dom_bytes / (dom_us * 1e-6) / 1e9
    step_gbs = by["total"] / (ms_per_step * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers --------------------------
    # Every step copies its inputs (q_idx, Q: one packed pinned host buffer) to the device,
    # runs clsa_decode_step and copies its outputs (O, idx, count: one packed buffer) back
    # to pinned host memory.  As in a serving loop the copies are pipelined with the compute:
    # two device buffer pairs alternate, the H2D of step i + 1 and the D2H of step i run on
    # copy streams ordered by events (step i waits for its H2D; step i + 2 waits for the D2H
    # of step i before it overwrites that output buffer).  M steps are captured in one CUDA
    # graph (copies included) and the timed region replays it; the pipeline drains at each
    # replay's end.
    in_h = [in_buf.cpu().pin_memory() for _ in range(2)]
    out_h = [torch.empty(out_buf.shape, dtype=torch.uint8).pin_memory() for _ in range(2)]
    h2d = in_h[0].numel()
    d2h = out_h[0].numel()
    in_b = [in_buf, torch.empty_like(in_buf)]
    out_b = [out_buf, torch.empty_like(out_buf)]

    def rebase(t, old_buf, new_buf):
        off = t.data_ptr() - old_buf.data_ptr()
        return new_buf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)

    e2e_args = [[clsa.decode_args(rebase(dv["q_idx"], in_buf, in_b[p_]), kidx_sets[r], dv["K"], dv["V"],
                                  rebase(dv["Q"], in_buf, in_b[p_]), dv["seq_lens"], k,
                                  rebase(out["O"], out_buf, out_b[p_]), rebase(out["idx"], out_buf, out_b[p_]),
                                  rebase(out["count"], out_buf, out_b[p_]))
                 for p_ in range(2)] for r in range(R)]
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    M = 2 * R

    def e2e_steps_on(cs, n):
        """n pipelined steps issued from stream cs (capturable); returns nothing"""
        ev = lambda: torch.cuda.Event()
        c_done, d_done = [None] * n, [None] * n
        s_h2d.wait_stream(cs)
        s_d2h.wait_stream(cs)
        for i in range(n):
            p_ = i % 2
            if i >= 2:
                s_h2d.wait_event(c_done[i - 2])          # step i - 2 has read in_b[p_]
            with torch.cuda.stream(s_h2d):
                in_b[p_].copy_(in_h[p_], non_blocking=True)
                h_ev = ev()
                h_ev.record(s_h2d)
            cs.wait_event(h_ev)
            if i >= 2:
                cs.wait_event(d_done[i - 2])              # the D2H of out_b[p_] is done
            clsa.decode_step_args(e2e_args[i % R][p_], ws, stream=cs)
            c_done[i] = ev()
            c_done[i].record(cs)
            s_d2h.wait_event(c_done[i])
            with torch.cuda.stream(s_d2h):
                out_h[p_].copy_(out_b[p_], non_blocking=True)
                d_done[i] = ev()
                d_done[i].record(s_d2h)
        cs.wait_stream(s_h2d)
        cs.wait_stream(s_d2h)

    e2e_graph = None
    if not args.no_graph:
        try:
            cap = torch.cuda.Stream()
            cap.wait_stream(stream)
            with torch.cuda.stream(cap):
                e2e_steps_on(cap, 4)  # warm the streams and events outside capture
            stream.wait_stream(cap)
            torch.cuda.synchronize()
            e2e_graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(e2e_graph):
                e2e_steps_on(torch.cuda.current_stream(), M)
            torch.cuda.synchronize()
        except Exception as ex:
            e2e_graph = None
            print(f"# e2e graph capture failed, eager pipeline: {ex}", file=sys.stderr)
    reps = max(1, min(args.steps, 400) // M)
    for _ in range(2):  # warm-up (the first replay uploads the graph)
        e2e_graph.replay() if e2e_graph is not None else e2e_steps_on(stream, M)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        e2e_graph.replay() if e2e_graph is not None else e2e_steps_on(stream, M)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / (reps * M)
    e2e_ms = replicas.max_over_ranks(e2e_ms, world, dev)
    e2e_launch = (f"{M} pipelined steps per CUDA graph (H2D, step, D2H on three streams)"
                  if e2e_graph is not None else f"{M} pipelined steps, eager")
    st = ws.status()
    if st[0] != "CLSA_OK":
        raise RuntimeError(f"device error during the end-to-end timing: {st}")

    # selection path of one extra step, read from the library's phase trace: CTAs whose group
    # resolved the TopK from the candidate windows, and CTAs whose group took the whole-row path
    sel_path = None
    if launches_per_step == 1:
        os.environ["CLSA_TRACE"] = "1"
        clsa.decode_step_args(args_sets[0], ws)
        torch.cuda.synchronize()
        del os.environ["CLSA_TRACE"]
        tr = clsa.fused_decode_trace(ws)
        used = (tr[:, 0] > 0) & ((tr[:, 31] & 0xFFFFFFFF) > 0)
        fast = int(((tr[:, 31] >> 32) > 0)[used].sum())
        sel_path = {"ctas_window_path": fast, "ctas_whole_row_path": int(used.sum()) - fast}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, threads, dt1, note = time_oracle(inp, w, args.cpu_sample_steps)
        cpu = {"value": w.B / dt, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": note,
               "single_thread_value": (w.B / dt1) if dt1 else None}

    replicas.finish(world)
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": DATA,
        "config": decode_config(w, args, world, graphs_ok=graphs is not None, kb=kidx_bytes),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_launch": dom_bytes, "us_per_launch": dom_us},
        "step_roofline": {"algorithmic_bytes": by["total"], "achieved_gbs": step_gbs, "peak": hbm,
                          "frac": step_gbs / hbm, "peak_kind": peak_kind},
        "kernels_us": kern,
        "kernels_method": kern_method,
        "e2e": {"value": replicas.job_rate(world, B, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "launch": e2e_launch},
        "gpu_launches": launches_per_step * args.steps,
        "selection": sel_path,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


class _DistillStep:
    """The distillation target as one timed step (preallocated outputs and workspace)."""

    def __init__(self, Q, K, scores, seq_lens):
        from long_context_sparse_clsa_b200 import clsa
        import torch
        self.args = (Q, K, scores, seq_lens)
        L, B, Hq, d = Q.shape
        self.ws = clsa.Workspace(clsa.load_library().clsa_distill_workspace_size(B, K.shape[1], L, Hq, K.shape[2], d))
        self.abar = torch.empty(B, K.shape[1], dtype=torch.float32, device=Q.device)
        self.kl = torch.empty(B, dtype=torch.float32, device=Q.device)

    def step(self) -> int:
        from long_context_sparse_clsa_b200 import clsa
        clsa.distill_target(*self.args, ws=self.ws, abar=self.abar, kl=self.kl)
        return clsa.last_launch_count()


class _MassStep:
    """The attention-mass coverage as one timed step (preallocated outputs and workspace)."""

    def __init__(self, Q, K, lse_sparse, seq_lens):
        from long_context_sparse_clsa_b200 import clsa
        import torch
        self.args = (Q, K, lse_sparse, seq_lens)
        L, B, Hq, d = Q.shape
        self.ws = clsa.Workspace(clsa.load_library().clsa_attention_mass_workspace_size(B, K.shape[1], L, Hq,
                                                                                        K.shape[2], d))
        self.mass = torch.empty(L, B, Hq, dtype=torch.float32, device=Q.device)

    def step(self) -> int:
        from long_context_sparse_clsa_b200 import clsa
        clsa.attention_mass(*self.args, ws=self.ws, mass=self.mass, want_lse_all=False)
        return clsa.last_launch_count()


def run_variant(args):
    """Time a comparison system of the pages' ablation (per-layer routing, YOCO only,
    standard attention) on the same workload, built from the library's own calls."""
    import torch
    from long_context_sparse_clsa_b200 import clsa
    from long_context_sparse_clsa_b200 import baselines
    from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs
    if args.gpus != 1:
        raise SystemExit("--variant runs on one GPU")
    torch.cuda.set_device(0)
    clsa.load_library()
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    dev = dv["K"].device
    stream = torch.cuda.current_stream()
    L, B, Hq, Hkv, d, k, n = w.L, w.B, w.Hq, w.Hkv, w.d, w.k, w.n_max
    eb = 2 if w.dtype == "bf16" else 4
    Ob = torch.empty_like(dv["Q"])
    lens = [int(x) for x in inp.seq_lens]
    gen = torch.Generator(device="cpu").manual_seed(4321)

    def permuted(x):
        """x [B][n_max][...] with every sequence's valid rows in a seeded random order"""
        y = x.clone()
        for b in range(B):
            perm = torch.randperm(lens[b], generator=gen).to(dev)
            y[b, :lens[b]] = x[b, perm]
        return y

    # every layer's extra inputs are row permutations of the seeded ones (layer 0: the seeded
    # tensors): the same value distribution, other rows selected / read
    qo_bytes = 2 * L * B * Hq * d * eb
    if args.variant == "per_layer_routing":
        kx = [dv["k_idx"]] + [permuted(dv["k_idx"]) for _ in range(L - 1)]
        qx = [dv["q_idx"]] * L
        idx = torch.empty(L, B, k, dtype=torch.int32, device=dev)
        cnt = torch.empty(L, B, dtype=torch.int32, device=dev)
        sysm = baselines.PerLayerRouting(qx, kx, dv["K"], dv["V"], dv["Q"], dv["seq_lens"], k, Ob, idx, cnt)
        sel = sum(min(k, x) for x in lens)
        step_bytes_ = L * (sum(lens) * w.d_idx * eb + B * w.d_idx * eb + 2 * sel * Hkv * d * eb) + qo_bytes
        note = "every layer: its own indexer scan over the shared cache, its own TopK, attention (L fused steps)"
    elif args.variant == "yoco_dense":
        sysm = baselines.YocoDense(dv["K"], dv["V"], dv["Q"], dv["seq_lens"], Ob)
        step_bytes_ = 2 * sum(lens) * Hkv * d * eb + qo_bytes
        note = "every layer dense over the one shared cache (one call, the L*G rows of a head read each row once)"
    elif args.variant == "attention_mass":
        r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], k)
        sysm = _MassStep(dv["Q"], dv["K"], r["lse"], dv["seq_lens"])
        # the cache's K once, Q once, the selection's lse in and the mass out
        step_bytes_ = sum(lens) * Hkv * d * eb + qo_bytes // 2 + 2 * L * B * Hq * 4
        note = "share of the dense softmax mass on the selection: one lse pass over K, merged with the step's lse"
    elif args.variant == "distill_target":
        sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
        sysm = _DistillStep(dv["Q"], dv["K"], sc, dv["seq_lens"])
        # the two passes each stream the cache (K) once; I read and Abar written once
        step_bytes_ = 2 * sum(lens) * Hkv * d * eb + 2 * sum(lens) * 4 + qo_bytes // 2
        note = "Abar and KL(Abar || softmax(I)) over the whole cache: row lse pass + Abar pass (K read twice)"
    else:
        Ks = [dv["K"]] + [permuted(dv["K"]) for _ in range(L - 1)]
        Vs = [dv["V"]] + [permuted(dv["V"]) for _ in range(L - 1)]
        sysm = baselines.StandardAttention(Ks, Vs, dv["Q"], dv["seq_lens"], Ob)
        step_bytes_ = L * 2 * sum(lens) * Hkv * d * eb + qo_bytes
        note = "every layer dense over its own cache (L calls)"
    launches = sysm.step()
    torch.cuda.synchronize()
    graph = None
    if not args.no_graph:
        s2 = torch.cuda.Stream()
        s2.wait_stream(stream)
        with torch.cuda.stream(s2):
            sysm.step()
        stream.wait_stream(s2)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            sysm.step()
        torch.cuda.synchronize()
    run = graph.replay if graph is not None else sysm.step
    for _ in range(max(args.warmup, 3)):
        run()
    torch.cuda.synchronize()
    with ClockSampler(0) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            run()
        e1.record(stream)
        torch.cuda.synchronize()
    st = sysm.ws.status()
    if st[0] != "CLSA_OK":
        raise RuntimeError(f"device error during timing: {st}")
    ms = e0.elapsed_time(e1) / args.steps
    hbm, _, peak_kind = peaks()
    gbs = step_bytes_ / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "variant": args.variant, "value": B / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "us_per_step": ms * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1); extra layers' inputs are seeded row permutations)",
        "config": {"workload": w.name, "B": B, "n": n, "d_idx": w.d_idx, "k": k, "L": L, "Hq": Hq, "Hkv": Hkv,
                   "d": d, "system": note, "l2": "every step reads more than L2 (no flush)",
                   "launch": "cuda graph" if graph is not None else "eager"},
        "roofline": {"bound": "hbm", "kernel": "whole step", "achieved": gbs, "peak": hbm, "unit": "GB/s",
                     "frac": gbs / hbm, "traffic": None, "peak_kind": peak_kind,
                     "algorithmic_bytes_per_step": step_bytes_},
        "gpu_launches": launches * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def run_prefill(args):
    """One prefill chunk per step (clsa_prefill_chunk: causal indexer GEMM with the candidate
    filter, exact per-row TopK, per-row sparse attention over L layers).  Reports chunk
    rows/s and the indexer kernel's useful-FLOP rate against the bf16 tensor peak."""
    import torch
    from long_context_sparse_clsa_b200 import clsa
    from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs
    if args.gpus != 1:
        raise SystemExit("the prefill line runs on one GPU")
    torch.cuda.set_device(0)
    clsa.load_library()
    w = WORKLOADS[args.workload]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    stream = torch.cuda.current_stream()
    T, n, k, L, Hq, d = w.T, w.n_max, w.k, w.L, w.Hq, w.d
    out = {"O": torch.empty_like(dv["Q"]), "idx": torch.empty(T, k, dtype=torch.int32, device="cuda"),
           "count": torch.empty(T, dtype=torch.int32, device="cuda")}
    a = clsa.prefill_args(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], k, out["O"], out["idx"],
                          out["count"])
    ws = clsa.Workspace(clsa.prefill_workspace_size(a))
    lib = clsa.load_library()

    def chunk():
        clsa._check(lib.clsa_prefill_chunk(ctypes.byref(a), ws.ptr, ws.nbytes, clsa._stream()), "clsa_prefill_chunk")

    for _ in range(max(args.warmup, 3)):
        chunk()
    torch.cuda.synchronize()
    launches = clsa.last_launch_count()
    steps = max(1, min(args.steps, 50))
    timer = clsa.LaunchTimer(16)
    per_launch = []
    with ClockSampler(0) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            chunk()
        e1.record(stream)
        torch.cuda.synchronize()
        for _ in range(min(steps, 10)):  # per-launch times of whole chunks (the attention of each
            timer.arm()                  # chunk streams > 500 MB, so every route launch starts cold)
            chunk()
            torch.cuda.synchronize()
            per_launch.append(timer.times_ms())
        # the attention stage alone on the chunk's selection: per row (mode 0, the chunk's own)
        # and key-centric row pairs over the union of their selections (mode 1)
        attn_modes = {}
        for mode in (0, 1):
            ts = []
            for _ in range(4):
                timer.arm()
                clsa._check(lib.clsa_prefill_attention(ctypes.byref(a), mode, ws.ptr, ws.nbytes, clsa._stream()),
                            "clsa_prefill_attention")
                torch.cuda.synchronize()
                ts.append(timer.times_ms()[0])
            attn_modes["per_row" if mode == 0 else "key_centric_pairs"] = statistics.median(ts[1:])
    st = ws.status()
    if st[0] != "CLSA_OK":
        raise RuntimeError(f"device error during timing: {st}")
    ms = e0.elapsed_time(e1) / steps
    route_ms = statistics.median(pl_[0] for pl_ in per_launch)
    attn_ms = statistics.median(pl_[-1] for pl_ in per_launch)
    hbm, bf16, peak_kind = peaks()
    sustained = None
    pk = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk):
        sustained = json.load(open(pk)).get("bf16_tflops_sustained")
    t0 = n - T
    useful = 2 * w.d_idx * sum(t0 + i + 1 for i in range(T))   # causal rectangle of the indexer
    tfs = useful / (route_ms * 1e-3) / 1e12
    attn_flops = T * L * Hq * k * d * 4
    line = {
        "metric": METRIC, "variant": "prefill_chunk", "value": T / (ms * 1e-3), "unit": "rows/s", "n_gpus": 1,
        "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype, "data": "synthetic (seeded N(0,1))",
        "config": {"workload": w.name, "T": T, "n": n, "d_idx": w.d_idx, "k": k, "L": L, "Hq": Hq, "Hkv": w.Hkv,
                   "d": d, "l2": "each chunk's attention streams > 500 MB: every route launch starts cold",
                   "launch": "eager (one clsa_prefill_chunk per step)"},
        "roofline": {"bound": "tensor", "kernel": "prefill_route_kernel", "achieved": tfs, "peak": bf16,
                     "unit": "TFLOP/s", "frac": tfs / bf16, "traffic": None, "peak_kind": f"{peak_kind} burst",
                     "frac_of_sustained": (tfs / sustained) if sustained else None,
                     "useful_flops_per_launch": useful, "us_per_launch": route_ms * 1e3},
        "launch_ms_median": [statistics.median(x) for x in zip(*per_launch)],
        "attention": {"kernel": "last launch of the chunk", "ms": attn_ms,
                      "useful_tflops": attn_flops / (attn_ms * 1e-3) / 1e12,
                      "stage_alone_ms": attn_modes},
        "gpu_launches": launches * steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload.startswith("prefill"):
        run_prefill(args)
    elif args.variant != "clsa":
        run_variant(args)
    else:
        run_clsa(args)


if __name__ == "__main__":
    main()
