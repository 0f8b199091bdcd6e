"""GPU parity of the comparison systems built from the library's calls (per-layer
routing, dense attention over one shared cache, standard attention with per-layer
caches) against the CPU oracle, at sizes that span several attention splits and a
cache longer than the selection limit.  Tolerances as in test_gpu_parity.py."""
import numpy as np
import pytest
import torch

from oracle import clsa_oracle as O
from long_context_sparse_clsa_b200 import clsa
from long_context_sparse_clsa_b200.baselines import PerLayerRouting, StandardAttention, YocoDense, attention_mass
from long_context_sparse_clsa_b200.inputs import make_inputs, scaled
from parity_util import check_near_tie_sets, max_abs, tensor_f64

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_clsa_b200.build import build
    build()
    clsa.load_library()


def _dense_oracle(inp_Q, inp_K, inp_V, lens):
    """Dense attention = sparse attention over every valid row (idx = 0..len-1)."""
    B = len(lens)
    n_max = inp_K.shape[1]
    idx = np.tile(np.arange(n_max, dtype=np.int64), (B, 1))
    return O.sparse_attention(inp_Q, inp_K, inp_V, idx, np.asarray(lens))[0]


def test_per_layer_routing():
    base = scaled("decode32k", n_max=5000 + 13, k=400, L=3)
    layers = [make_inputs(base, seed=21 + l) for l in range(base.L)]
    kv = layers[0]  # the shared cache and the queries
    dvs = [clsa.to_device(x) for x in layers]
    Q, K, V, lens = dvs[0]["Q"], dvs[0]["K"], dvs[0]["V"], dvs[0]["seq_lens"]
    Ob = torch.empty_like(Q)
    idx = torch.empty(base.L, base.B, base.k, dtype=torch.int32, device=Q.device)
    cnt = torch.empty(base.L, base.B, dtype=torch.int32, device=Q.device)
    sysm = PerLayerRouting([d["q_idx"] for d in dvs], [d["k_idx"] for d in dvs], K, V, Q, lens, base.k, Ob, idx, cnt)
    sysm.step()
    torch.cuda.synchronize()
    assert sysm.ws.status()[0] == "CLSA_OK"
    got = tensor_f64(Ob)
    for l, x in enumerate(layers):
        i_np, c_np = idx[l].cpu().numpy(), cnt[l].cpu().numpy()
        check_near_tie_sets(i_np, c_np, O.index_scores(x.q_idx, x.k_idx, x.seq_lens), x.seq_lens, base.k)
        want, _ = O.sparse_attention(kv.Q[l:l + 1], kv.K, kv.V, i_np, c_np)
        assert max_abs(got[l:l + 1], want) <= TOL[base.dtype]
    # the layers' selections differ: the routing really ran per layer
    assert not torch.equal(idx[0], idx[1])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_yoco_dense_longer_than_selection_limit(dtype):
    """Dense attention over a shared cache of 6000+ rows (above the 4096 selection
    limit), ragged lengths, several splits."""
    w = scaled("ragged16", B=3, n_max=6000 + 37, lens=(4097, 6037), k=16, L=2, Hq=8, Hkv=2, d=64, d_idx=64,
               dtype=dtype, plant=0.0, seed=9)
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    Ob = torch.empty_like(dv["Q"])
    sysm = YocoDense(dv["K"], dv["V"], dv["Q"], dv["seq_lens"], Ob)
    sysm.step()
    torch.cuda.synchronize()
    assert sysm.ws.status()[0] == "CLSA_OK"
    want = _dense_oracle(inp.Q, inp.K, inp.V, inp.seq_lens)
    assert max_abs(tensor_f64(Ob), want) <= TOL[dtype]


def test_standard_attention_per_layer_caches():
    w = scaled("decode32k", n_max=4500, k=16, L=2, plant=0.0)
    caches = [make_inputs(w, seed=40 + l) for l in range(w.L)]
    dvs = [clsa.to_device(x) for x in caches]
    Q = dvs[0]["Q"]
    Ob = torch.empty_like(Q)
    sysm = StandardAttention([d["K"] for d in dvs], [d["V"] for d in dvs], Q, dvs[0]["seq_lens"], Ob)
    sysm.step()
    torch.cuda.synchronize()
    assert sysm.ws.status()[0] == "CLSA_OK"
    got = tensor_f64(Ob)
    for l, x in enumerate(caches):
        want = _dense_oracle(caches[0].Q[l:l + 1], x.K, x.V, x.seq_lens)
        assert max_abs(got[l:l + 1], want) <= TOL[w.dtype]


@pytest.mark.parametrize("name", ["bf16_small", "f32_d64", "decode128k"])
def test_attention_mass(name):
    """clsa_attention_mass (the share of dense softmax mass on the selection) against the
    oracle's full softmax summed over the GPU's selected rows (picx.dev summary, Attention
    Sparsity Analysis).  bf16 d = 128 takes the tensor-core lse pass; fp32 d = 64 the
    split-k kernel; decode128k at full size is checked on the first and last layers."""
    from long_context_sparse_clsa_b200.inputs import WORKLOADS
    w = {"bf16_small": scaled("decode32k", n_max=6000, k=500, L=2, plant=0.0),
         "f32_d64": scaled("tiny", n_max=3000, k=300, L=3, Hq=8, Hkv=2, seed=4),
         "decode128k": WORKLOADS["decode128k"]}[name]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    r = clsa.decode_step(dv["q_idx"], dv["k_idx"], dv["K"], dv["V"], dv["Q"], dv["seq_lens"], w.k)
    mass, lse_all = attention_mass(dv["Q"], dv["K"], dv["V"], dv["seq_lens"], r["lse"])
    torch.cuda.synchronize()
    got = mass.cpu().double().numpy()
    i_np, c_np = r["idx"].cpu().numpy(), r["count"].cpu().numpy()
    layers = list(range(w.L)) if w.L <= 4 else [0, w.L - 1]
    want = O.attention_mass(inp.Q[layers], inp.K, i_np, c_np, inp.seq_lens)
    assert np.abs(got[layers] - want).max() <= 1e-3 * max(1.0, want.max()) + 1e-4
    assert np.all((got > 0) & (got <= 1 + 1e-3))
    # the relation it reports: mass = exp(lse_S - lse_all)
    np.testing.assert_allclose(got, np.exp(r["lse"].cpu().double().numpy() - lse_all.cpu().double().numpy()),
                               rtol=1e-5)


DISTILL_CASES = {
    # (workload, explicit seq_lens or None)
    "bf16_d128": (scaled("decode32k", n_max=3000 + 17, k=16, L=2, plant=0.0), None),
    # rows = L G = 12 per KV head: the MMA's N rounds up to 16 (the 16-column tail)
    "bf16_rows12": (scaled("ragged16", B=2, n_max=2000, lens=(1999, 2000), k=16, L=3, Hq=8, Hkv=2, d=128,
                           d_idx=128, plant=0.0, seed=6), (1999, 2000)),
    # G = 32, L = 5: two layer groups (128 and 32 rows); an empty sequence; ragged tails
    "bf16_groups_ragged": (scaled("ragged16", B=3, n_max=9000, lens=(4097, 9000), k=16, L=5, Hq=32, Hkv=1,
                                  d=128, d_idx=128, plant=0.0, seed=8), (9000, 0, 4097)),
    "f32_d64_ragged": (scaled("ragged16", B=3, n_max=1500, lens=(0, 1500), k=16, L=3, Hq=8, Hkv=2, d=64, d_idx=64,
                              dtype="f32", plant=0.0, seed=4), (None, 0, None)),
    # the full decode workload (131072 cached rows, 24 layers x 32 heads)
    "bf16_decode128k": (scaled("decode128k"), None),
}


@pytest.mark.parametrize("case", list(DISTILL_CASES))
def test_distill_target(case):
    """Abar (the layer/head-averaged attention over the cache) and KL(Abar || softmax(I))
    against the oracle, on the GPU's own indexer scores.  bf16 with d = 128 runs the
    tensor-core passes, fp32 the CUDA-core path."""
    w, lens = DISTILL_CASES[case]
    inp = make_inputs(w)
    dv = clsa.to_device(inp)
    if lens is not None:
        for b, n in enumerate(lens):
            if n is not None:
                inp.seq_lens[b] = n
                dv["seq_lens"][b] = n
    sc = clsa.index_scores(dv["q_idx"], dv["k_idx"], dv["seq_lens"])
    abar, kl, ws = clsa.distill_target(dv["Q"], dv["K"], sc, dv["seq_lens"])
    torch.cuda.synchronize()
    assert ws.status()[0] == "CLSA_OK"
    I = tensor_f64(sc)
    want_a, want_kl = O.distill_target(inp.Q, inp.K, I, inp.seq_lens)
    got_a, got_kl = tensor_f64(abar), tensor_f64(kl)
    for b, n in enumerate(inp.seq_lens):
        n = int(n)
        assert np.all(got_a[b, n:] == 0.0)
        if n == 0:
            assert got_kl[b] == 0.0
            continue
        assert np.max(np.abs(got_a[b, :n] - want_a[b, :n])) <= 1e-4 * np.max(want_a[b, :n])
        assert abs(got_a[b, :n].sum() - 1.0) < 1e-4
        assert abs(got_kl[b] - want_kl[b]) <= 1e-4 * max(1.0, abs(want_kl[b]))
