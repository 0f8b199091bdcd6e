"""Run one stage of the CLSA path on a named workload, for profilers.

    python -m long_context_sparse_clsa_b200.profile_cases --stage decode_step \
        [--workload decode128k] [--reps 3] [--batch B] [--rows T] [--layers L]

Stages: index_scores, topk, gather_kv, sparse_attn, decode_step, prefill_chunk, distill_target.
Inputs are the seeded synthetic workloads of ``inputs.py``; ``--batch`` replaces
the workload's batch (decode only).  Each stage runs once untimed and then
``--reps`` times, with a synchronize at the end and nothing else on the GPU.
"""
from __future__ import annotations

import argparse

import torch

from long_context_sparse_clsa_b200 import clsa
from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs, replace


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--stage", required=True, choices=["index_scores", "topk", "gather_kv", "sparse_attn",
                                                       "decode_step", "prefill_chunk", "distill_target"])
    ap.add_argument("--workload", default="decode128k")
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--rows", type=int, default=0, help="prefill rows T (default: the workload's)")
    ap.add_argument("--layers", type=int, default=0,
                    help="sparse_attn: attend with the first LAYERS layers' queries (default: all)")
    a = ap.parse_args()
    w = WORKLOADS[a.workload]
    if a.batch:
        w = replace(w, B=a.batch)
    if a.rows:
        w = replace(w, T=a.rows)
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    if w.mode == "prefill":
        fn = lambda: clsa.prefill_chunk(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], w.k)  # noqa: E731
    else:
        sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
        idx, cnt = clsa.topk(sc, dv["seq_lens"], w.k)
        KS, VS = clsa.gather_kv(dv["K"], dv["V"], idx, cnt)
        Qa = dv["Q"][:a.layers].contiguous() if a.layers else dv["Q"]
        dws = clsa.Workspace(clsa.load_library().clsa_distill_workspace_size(w.B, w.n_max, w.L, w.Hq, w.Hkv, w.d))
        fns = {
            "index_scores": lambda: clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"], sc),
            "topk": lambda: clsa.topk(sc, dv["seq_lens"], w.k, idx=idx, count=cnt),
            "gather_kv": lambda: clsa.gather_kv(dv["K"], dv["V"], idx, cnt, K_S=KS, V_S=VS),
            "sparse_attn": lambda: clsa.sparse_attn(Qa, KS, VS, cnt),
            "decode_step": lambda: clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"],
                                                    dv["seq_lens"], w.k),
            "distill_target": lambda: clsa.distill_target(dv["Q"], dv["K"], sc, dv["seq_lens"], ws=dws),
        }
        fn = fns[a.stage]
    fn()
    torch.cuda.synchronize()
    for _ in range(a.reps):
        fn()
    torch.cuda.synchronize()
    print(f"{a.stage} on {w.name} (B={w.B}): ok")


if __name__ == "__main__":
    main()
