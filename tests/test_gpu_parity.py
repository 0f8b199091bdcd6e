"""GPU parity: every C-ABI call against the CPU oracle on the same seeded inputs.

Acceptance (stated for this path): TopK index sets bit-exact on identical fp32
scores; end-to-end sets may differ only at near-ties (|I_j - I_(k)| <= 1e-4 max|I|);
attention max-abs <= 2e-2 for bf16 inputs (fp32 accumulation) and <= 1e-4 in fp32
mode, against the oracle evaluated on the GPU's own selection.  Scores are held
to the fp32 forward-error bound of a d-term dot product.
"""
import numpy as np
import pytest
import torch

from oracle import clsa_oracle as O
from long_context_sparse_clsa_b200 import clsa
from long_context_sparse_clsa_b200.inputs import WORKLOADS, make_inputs, scaled
from parity_util import check_near_tie_sets, max_abs, score_tol, tensor_f64

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}
LSE_TOL = {"f32": 1e-4, "bf16": 2e-3}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_clsa_b200.build import build
    build()
    clsa.load_library()


CASES = {
    "tiny": WORKLOADS["tiny"],
    "d32k_small": scaled("decode32k", n_max=8192 + 77, k=512, L=3),
    "ragged_small": scaled("ragged16", B=5, n_max=6000, lens=(0, 6000), k=700, L=2, seed=3),
    # more sequences than the grid has groups of Hkv CTAs for: the fused step's proportional
    # split, where a CTA attends several head units one after the other
    "ragged_b24": scaled("ragged16", B=24, n_max=3000, lens=(1, 3000), k=300, L=2, seed=4),
    "bf16_d64": scaled("decode32k", n_max=3000, d_idx=64, d=64, k=300, L=2, Hq=8, Hkv=2, plant=0.0),
    "f32_d128": scaled("tiny", n_max=2500, d_idx=128, d=128, k=333, L=2, Hq=6, Hkv=3, seed=5),
}


def _inputs(name):
    inp = make_inputs(CASES[name])
    return inp, clsa.to_device(inp)


# ----------------------------------------------------------------------- A1 scores

@pytest.mark.parametrize("name", list(CASES))
def test_index_scores(name):
    inp, dv = _inputs(name)
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    torch.cuda.synchronize()
    got = tensor_f64(sc)
    want = O.index_scores(inp.q_idx, inp.k_idx, inp.seq_lens)
    tol = score_tol(inp.f32("q_idx"), inp.f32("k_idx"), inp.seq_lens)
    for b, n in enumerate(inp.seq_lens):
        assert np.all(np.abs(got[b, :n] - want[b, :n]) <= tol[b, :n])
        assert np.isneginf(got[b, n:]).all()


# ----------------------------------------------------------------------- A2 top-k

def _topk_case(scores, lens, k):
    s = torch.tensor(scores, dtype=torch.float32, device="cuda")
    L = torch.tensor(lens, dtype=torch.int32, device="cuda")
    idx, cnt = clsa.topk(s, L, k)
    torch.cuda.synchronize()
    want_idx, want_cnt = O.topk_select(scores.astype(np.float64), lens, k)
    np.testing.assert_array_equal(cnt.cpu().numpy(), want_cnt)
    np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)


@pytest.mark.parametrize("B,n,k,kind", [
    (1, 131072, 2048, "normal"), (1, 131072, 2048, "ties"), (1, 32768, 2048, "normal"),
    (3, 5000, 4096, "normal"), (16, 40000, 2048, "ragged"), (2, 777, 1, "ties"),
    (1, 4096, 256, "allequal"), (1, 1000, 999, "signedzero"), (200, 3000, 100, "normal"),
    (4, 100, 200, "normal"),
])
def test_topk_bit_exact(B, n, k, kind):
    rng = np.random.default_rng(B * 7 + n + k)
    if kind == "ties":
        scores = rng.integers(-20, 20, size=(B, n)).astype(np.float32)
    elif kind == "allequal":
        scores = np.full((B, n), 1.5, dtype=np.float32)
    elif kind == "signedzero":
        scores = rng.choice(np.array([-0.0, 0.0, 1.0, -1.0], dtype=np.float32), size=(B, n))
    else:
        scores = (rng.standard_normal((B, n)) * 11).astype(np.float32)
    lens = np.full(B, n, dtype=np.int32)
    if kind == "ragged":
        lens = rng.integers(0, n + 1, size=B).astype(np.int32)
        lens[0] = 0
        lens[1] = 1
    _topk_case(scores, lens, k)


def test_topk_on_gpu_scores_bit_exact():
    inp, dv = _inputs("d32k_small")
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    torch.cuda.synchronize()
    _topk_case(sc.cpu().numpy(), inp.seq_lens, CASES["d32k_small"].k)


# ----------------------------------------------------------------------- A3 gather

def test_gather_bit_exact_and_bad_index():
    inp, dv = _inputs("ragged_small")
    w = CASES["ragged_small"]
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    idx, cnt = clsa.topk(sc, dv["seq_lens"], w.k)
    KS, VS = clsa.gather_kv(dv["K"], dv["V"], idx, cnt)
    torch.cuda.synchronize()
    i_np, c_np = idx.cpu().numpy(), cnt.cpu().numpy()
    want_K, want_V = O.gather_kv(inp.K, inp.V, i_np, c_np)
    got_K, got_V = tensor_f64(KS), tensor_f64(VS)
    for b in range(w.B):
        c = int(c_np[b])
        assert np.array_equal(got_K[b, :c], want_K[b, :c])   # a copy: bit-exact
        assert np.array_equal(got_V[b, :c], want_V[b, :c])
    bad = idx.clone()
    bad[0, 0] = w.n_max + 5
    cnt1 = cnt.clone()
    cnt1[0] = max(int(c_np[0]), 1)
    ws = clsa.Workspace(256)
    clsa.gather_kv(dv["K"], dv["V"], bad, cnt1, ws=ws)
    status, detail = ws.status()
    assert status == "CLSA_ERR_BAD_INDEX" and detail == 0
    assert ws.status()[0] == "CLSA_OK"   # reading clears it


# ----------------------------------------------------------------------- A4 attention

@pytest.mark.parametrize("name,L", [("tiny", None), ("tiny", 1), ("d32k_small", None), ("d32k_small", 1),
                                    ("ragged_small", None), ("bf16_d64", None), ("f32_d128", None)])
def test_sparse_attn(name, L):
    w = CASES[name]
    inp, dv = _inputs(name)
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    idx, cnt = clsa.topk(sc, dv["seq_lens"], w.k)
    KS, VS = clsa.gather_kv(dv["K"], dv["V"], idx, cnt)
    Q = dv["Q"] if L is None else dv["Q"][:1].contiguous()
    out, lse = clsa.sparse_attn(Q, KS, VS, cnt)
    torch.cuda.synchronize()
    i_np, c_np = idx.cpu().numpy(), cnt.cpu().numpy()
    Qh = inp.Q if L is None else inp.Q[:1]
    want, want_lse = O.sparse_attention(Qh, inp.K, inp.V, i_np, c_np)
    assert max_abs(tensor_f64(out), want) <= TOL[w.dtype]
    got_lse = tensor_f64(lse)
    fin = np.isfinite(want_lse)
    assert (np.isneginf(got_lse) == ~fin).all()
    assert max_abs(got_lse[fin], want_lse[fin]) <= LSE_TOL[w.dtype] * (1 + np.abs(want_lse[fin]).max())


@pytest.mark.parametrize("layers", ["all", "one"])
def test_sparse_attn_full_size(layers):
    """decode128k through the stage calls, as the per-kernel timings run them: gathered
    compact K_S/V_S, then clsa_sparse_attn over all 24 layers or over one layer (the
    model-faithful per-layer call); every head of the first and last layers against the
    oracle, with the LSE."""
    w = WORKLOADS["decode128k"]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    idx, cnt = clsa.topk(sc, dv["seq_lens"], w.k)
    KS, VS = clsa.gather_kv(dv["K"], dv["V"], idx, cnt)
    Q = dv["Q"] if layers == "all" else dv["Q"][-1:].contiguous()
    out, lse = clsa.sparse_attn(Q, KS, VS, cnt)
    torch.cuda.synchronize()
    i_np, c_np = idx.cpu().numpy(), cnt.cpu().numpy()
    got, got_lse = tensor_f64(out), tensor_f64(lse)
    # the oracle over the selected rows only (its gather, then its attention)
    c = int(c_np[0])
    sel = i_np[0, :c]
    Kc, Vc = inp.K[:, sel], inp.V[:, sel]
    ic = np.arange(c, dtype=np.int64)[None]
    ls = (0, w.L - 1) if layers == "all" else (w.L - 1,)
    for l in ls:
        want, want_lse = O.sparse_attention(inp.Q[l:l + 1], Kc, Vc, ic, c_np)
        lq = l if layers == "all" else 0
        assert max_abs(got[lq], want[0]) <= TOL[w.dtype], l
        assert max_abs(got_lse[lq], want_lse[0]) <= LSE_TOL[w.dtype] * (1 + np.abs(want_lse).max()), l


def test_sparse_attn_workspace_reuse_is_clean():
    """One workspace through per-layer calls (the in-kernel split merge and its arrival
    counters), an all-layer call (split partials and the combine) and per-layer calls again:
    every repeat is bit-identical to the first, so each call left the workspace clean."""
    w = CASES["d32k_small"]
    inp, dv = _inputs("d32k_small")
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    idx, cnt = clsa.topk(sc, dv["seq_lens"], w.k)
    KS, VS = clsa.gather_kv(dv["K"], dv["V"], idx, cnt)
    Qall = torch.cat([dv["Q"]] * 8)  # 24 layers: 96 rows per KV head, the tensor-core kernel
    lib = clsa.load_library()
    ws = clsa.Workspace(max(lib.clsa_sparse_attn_workspace_size(w.B, w.k, L, w.Hq, w.Hkv, w.d) for L in (1, 24)))
    outs = []
    for Q in (dv["Q"][:1], Qall, dv["Q"][:1], Qall, dv["Q"][1:2]):
        o, l = clsa.sparse_attn(Q.contiguous(), KS, VS, cnt, ws=ws)
        outs.append((o.clone(), l.clone()))
    torch.cuda.synchronize()
    assert ws.status()[0] == "CLSA_OK"
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])
    assert torch.equal(outs[1][0], outs[3][0]) and torch.equal(outs[1][1], outs[3][1])
    # layer 1 alone equals layer 1 of the all-layer call, against the oracle too
    i_np, c_np = idx.cpu().numpy(), cnt.cpu().numpy()
    want, _ = O.sparse_attention(inp.Q[1:2], inp.K, inp.V, i_np, c_np)
    assert max_abs(tensor_f64(outs[4][0][0]), want[0]) <= TOL[w.dtype]
    assert max_abs(tensor_f64(outs[1][0][1]), want[0]) <= TOL[w.dtype]


@pytest.mark.parametrize("dtype,L", [("bf16", 3), ("bf16", 6), ("f32", 3)])
def test_sparse_attn_growing_scores(dtype, L):
    """Scores that grow along the selection by far more than 2^8 per 64-token chunk: the
    tensor-core kernel's reference max must move and its running output be rescaled (L = 6:
    24 rows per KV head), the few-rows kernel's splits merge across very different maxima
    (L = 3: 12 rows), the f32 kernel is the control.  Ragged counts, one empty sequence,
    several splits."""
    rng = np.random.default_rng(11)
    B, k, Hq, Hkv, d = 3, 700, 32, 8, 128
    K = rng.standard_normal((B, k, Hkv, d))
    K *= (1.0 + np.arange(k) / 40.0)[None, :, None, None]  # |scores| ~ 1 .. 18 sigma
    V = rng.standard_normal((B, k, Hkv, d))
    Q = rng.standard_normal((L, B, Hq, d))
    cnt = np.array([700, 0, 333], dtype=np.int32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    # the oracle sees the values the device holds
    Kd, Vd, Qd = (torch.tensor(a, dtype=tdt, device="cuda") for a in (K, V, Q))
    out, lse = clsa.sparse_attn(Qd, Kd, Vd, torch.tensor(cnt, device="cuda"))
    torch.cuda.synchronize()
    Kh, Vh, Qh = (tensor_f64(t) for t in (Kd, Vd, Qd))
    idx = np.tile(np.arange(k, dtype=np.int64), (B, 1))
    want, want_lse = O.sparse_attention(Qh, Kh, Vh, idx, cnt)
    assert max_abs(tensor_f64(out), want) <= TOL[dtype]
    got_lse = tensor_f64(lse)
    fin = np.isfinite(want_lse)
    assert (np.isneginf(got_lse) == ~fin).all()
    assert max_abs(got_lse[fin], want_lse[fin]) <= LSE_TOL[dtype] * (1 + np.abs(want_lse[fin]).max())


# ----------------------------------------------------------------------- A5 decode step

@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("compact", [False, True])
def test_decode_step(name, compact):
    w = CASES[name]
    inp, dv = _inputs(name)
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k,
                         compact=compact, want_scores=True)
    torch.cuda.synchronize()
    assert r["ws"].status()[0] == "CLSA_OK"
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    ora_scores = O.index_scores(inp.q_idx, inp.k_idx, inp.seq_lens)
    check_near_tie_sets(i_np, c_np, ora_scores, inp.seq_lens, w.k)
    # the selection the GPU made is exactly TopK of the scores it computed
    gi, gc = O.topk_select(tensor_f64(r["scores"]), inp.seq_lens, w.k)
    np.testing.assert_array_equal(gi, i_np)
    want, want_lse = O.sparse_attention(inp.Q, inp.K, inp.V, i_np, c_np)
    assert max_abs(tensor_f64(r["O"]), want) <= TOL[w.dtype]
    fin = np.isfinite(want_lse)
    assert max_abs(tensor_f64(r["lse"])[fin], want_lse[fin]) <= LSE_TOL[w.dtype] * (1 + np.abs(want_lse[fin]).max())


def test_decode_step_deterministic():
    w = CASES["d32k_small"]
    _, dv = _inputs("d32k_small")
    a = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k)
    b = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k, ws=a["ws"])
    torch.cuda.synchronize()
    assert torch.equal(a["O"], b["O"]) and torch.equal(a["idx"], b["idx"]) and torch.equal(a["lse"], b["lse"])


@pytest.mark.parametrize("name", ["decode128k", "decode32k"])
def test_decode_step_full_size(name):
    """Full-size workloads in the launch configuration the benchmark times:
    selection bit-exact against TopK of the GPU scores, near-tie rule against the
    oracle's float64 scores, and attention against the oracle on sampled heads."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k,
                         want_scores=True)
    torch.cuda.synchronize()
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    gi, _ = O.topk_select(tensor_f64(r["scores"]), inp.seq_lens, w.k)
    np.testing.assert_array_equal(gi, i_np)
    ora_scores = O.index_scores(inp.q_idx, inp.k_idx, inp.seq_lens)
    check_near_tie_sets(i_np, c_np, ora_scores, inp.seq_lens, w.k)
    # the planted salient tokens the exact TopK keeps are the ones the GPU keeps
    exact = set(O.topk_select(ora_scores, inp.seq_lens, w.k)[0][0].tolist())
    planted = set(inp.planted[0].tolist())
    assert len(planted & set(i_np[0, : c_np[0]].tolist())) == len(planted & exact) > len(planted) // 2
    # every head of the first and last layers, sampled heads of a middle layer
    rng = np.random.default_rng(0)
    mid = int(rng.integers(1, w.L - 1))
    pairs = [(l, h) for l in (0, w.L - 1) for h in range(w.Hq)]
    pairs += [(mid, int(h)) for h in sorted(set(rng.choice(w.Hq, 6, replace=False).tolist()))]
    got = tensor_f64(r["O"])
    for l, h in pairs:
        want, _ = O.sparse_attention(inp.Q[l:l + 1, :, h:h + 1], inp.K[:, :, h // w.G: h // w.G + 1],
                                     inp.V[:, :, h // w.G: h // w.G + 1], i_np, c_np)
        assert max_abs(got[l, :, h], want[0, :, 0]) <= TOL[w.dtype], (l, h)


def test_ragged16_full_size_sampled():
    w = WORKLOADS["ragged16"]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k,
                         want_scores=True)
    torch.cuda.synchronize()
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    gi, _ = O.topk_select(tensor_f64(r["scores"]), inp.seq_lens, w.k)
    np.testing.assert_array_equal(gi, i_np)
    got = tensor_f64(r["O"])
    for b in (0, 7, 15):
        ora_scores = O.index_scores(inp.q_idx[b:b + 1], inp.k_idx[b:b + 1], inp.seq_lens[b:b + 1])
        check_near_tie_sets(i_np[b:b + 1], c_np[b:b + 1], ora_scores, inp.seq_lens[b:b + 1], w.k)
        for l, h in ((0, 0), (w.L - 1, w.Hq - 1), (11, 13)):
            g = h // w.G
            want, _ = O.sparse_attention(inp.Q[l:l + 1, b:b + 1, h:h + 1], inp.K[b:b + 1, :, g:g + 1],
                                         inp.V[b:b + 1, :, g:g + 1], i_np[b:b + 1], c_np[b:b + 1])
            assert max_abs(got[l, b, h], want[0, 0, 0]) <= TOL[w.dtype]


# ----------------------------------------------------------------------- A6-A8 prefill

def _prefill_check(w, rows):
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    r = clsa.prefill_chunk(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], w.k)
    torch.cuda.synchronize()
    assert r["ws"].status()[0] == "CLSA_OK"
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    n, T = w.n_max, w.T
    assert c_np.tolist() == [min(w.k, n - T + i + 1) for i in range(T)]
    ora_scores = O.prefill_scores(inp.q_idx, inp.k_idx, n, rows)
    lens = [n - T + i + 1 for i in rows]
    check_near_tie_sets(i_np[rows], c_np[rows], ora_scores, lens, w.k)
    want, want_lse = O.prefill_attention(inp.Q, inp.K, inp.V, i_np[rows], c_np[rows], rows)
    got = tensor_f64(r["O"])[:, rows]
    assert max_abs(got, want) <= TOL[w.dtype]
    got_lse = tensor_f64(r["lse"])[:, rows]
    assert max_abs(got_lse, want_lse) <= LSE_TOL[w.dtype] * (1 + np.abs(want_lse).max())


def test_prefill_small():
    w = scaled("prefill4k", n_max=3000, T=300, k=256, L=2)
    _prefill_check(w, list(range(300)))


def test_prefill_all_rows_new():
    """n = T: row i selects among i + 1 tokens (k_eff = 1, 2, ..., k): partial and single-token
    chunks of the per-row attention; 20 (layer, head) rows per KV head (not a multiple of 32)."""
    w = scaled("prefill4k", n_max=700, T=700, k=300, L=5)
    _prefill_check(w, [0, 1, 2, 62, 63, 64, 65, 127, 128, 299, 300, 511, 699])


def test_prefill_layer_groups():
    """L*G = 180 > 128 rows per KV head: the attention runs in two layer groups of 23 layers
    (92 rows; the second group's last layer slot is past L)."""
    w = scaled("prefill4k", n_max=1500, T=200, k=160, L=45, Hq=16, Hkv=4)
    _prefill_check(w, list(range(0, 200, 7)) + [199])


@pytest.mark.parametrize("kw", [dict(L=2, Hq=8, Hkv=2),     # 8 rows per KV head: the few-rows kernel
                                dict(L=6, Hq=16, Hkv=4)])   # 24 rows per KV head: the mma.sync kernel
def test_prefill_head_dim_64(kw):
    """d = 64 (the tensor-core attention takes d = 128 only): prefill rows through the
    other attention kernels, gathering from the one shared cache."""
    w = scaled("prefill4k", n_max=2000, T=150, k=200, d=64, **kw)
    _prefill_check(w, list(range(0, 150, 3)) + [149])


def test_prefill_full_size_sampled():
    w = WORKLOADS["prefill4k"]
    _prefill_check(w, [0, 1, 2047, 2048, 4095])


@pytest.mark.parametrize("name,kw,rows", [
    ("prefill4k_corr", dict(n_max=3000, T=301, k=256, L=2), None),    # correlated rows: a small union; odd T
    ("prefill4k", dict(n_max=3000, T=300, k=256, L=2), None),         # independent rows: a large union
    # k_eff = 1 .. k: pairs of unequal sizes
    ("prefill4k", dict(n_max=700, T=700, k=300, L=5), [0, 1, 2, 62, 63, 64, 65, 127, 128, 299, 300, 511, 698, 699]),
    # two layer groups
    ("prefill4k_corr", dict(n_max=1500, T=200, k=160, L=45, Hq=16, Hkv=4), list(range(0, 200, 7)) + [199]),
])
def test_prefill_attention_key_centric(name, kw, rows):
    """clsa_prefill_attention mode 1 (row pairs over the union of their selections) on the
    selection clsa_prefill_chunk made: every row against the oracle's per-row attention, and
    against mode 0 on the same selection."""
    w = scaled(name, **kw)
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    r = clsa.prefill_chunk(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], w.k)
    o1, l1 = clsa.prefill_attention(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], w.k, r["idx"], r["count"],
                                    mode=1)
    o0, l0 = clsa.prefill_attention(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], w.k, r["idx"], r["count"],
                                    mode=0)
    torch.cuda.synchronize()
    assert r["ws"].status()[0] == "CLSA_OK"
    assert torch.equal(o0, r["O"]) and torch.equal(l0, r["lse"])  # mode 0 is the chunk's own attention
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    rows = rows or list(range(w.T))
    want, want_lse = O.prefill_attention(inp.Q, inp.K, inp.V, i_np[rows], c_np[rows], rows)
    assert max_abs(tensor_f64(o1)[:, rows], want) <= TOL[w.dtype]
    got_lse = tensor_f64(l1)[:, rows]
    assert max_abs(got_lse, want_lse) <= LSE_TOL[w.dtype] * (1 + np.abs(want_lse).max())
    assert max_abs(tensor_f64(o1), tensor_f64(o0)) <= TOL[w.dtype]  # every row


# ----------------------------------------------------------------------- fused vs four-kernel plan

def _decode(dv, w, plan, monkeypatch, **kw):
    monkeypatch.setenv("CLSA_DECODE_PLAN", plan)
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k,
                         want_scores=True, **kw)
    torch.cuda.synchronize()
    assert r["ws"].status()[0] == "CLSA_OK"
    return r


@pytest.mark.parametrize("name", ["d32k_small", "ragged_small"])
def test_fused_matches_unfused(name, monkeypatch):
    w = CASES[name]
    _, dv = _inputs(name)
    a = _decode(dv, w, "fused", monkeypatch)
    b = _decode(dv, w, "unfused", monkeypatch)
    assert torch.equal(a["scores"], b["scores"])      # same fp32 arithmetic order
    assert torch.equal(a["idx"], b["idx"]) and torch.equal(a["count"], b["count"])
    assert max_abs(tensor_f64(a["O"]), tensor_f64(b["O"])) <= TOL[w.dtype]


@pytest.mark.parametrize("n,k,mode", [(10000, 2048, "equal"), (40000, 2048, "equal"), (20000, 3000, "blocks"),
                                      (5000, 4096, "equal"), (3000, 4000, "normal")])
def test_decode_step_adversarial_selection(n, k, mode, monkeypatch):
    """Ties everywhere (every index key equal, or a few distinct values): the
    candidate list of the fused plan overflows shared memory (n > 16384) or holds
    every token; selection must still be the exact TopK with lower-index ties."""
    w = scaled("decode32k", n_max=n, k=k, L=2, plant=0.0)
    inp = make_inputs(w)
    if mode == "equal":
        inp.k_idx[:] = inp.k_idx[:, :1, :]
    elif mode == "blocks":
        inp.k_idx[0] = inp.k_idx[0][np.arange(n) % 7]
    dv = clsa.to_device(inp)
    r = _decode(dv, w, "fused", monkeypatch)
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    gi, gc = O.topk_select(tensor_f64(r["scores"]), inp.seq_lens, w.k)
    np.testing.assert_array_equal(gi, i_np)
    np.testing.assert_array_equal(gc, c_np)
    want, _ = O.sparse_attention(inp.Q, inp.K, inp.V, i_np, c_np)
    assert max_abs(tensor_f64(r["O"]), want) <= TOL[w.dtype]
