"""Pins for the CPU oracle: each check ties it to something other than itself.

* TopK against a brute-force rank count (a different formulation from the
  oracle's stable sort), with forced ties, -0.0/+0.0 and ragged lengths.
* Attention against torch's scaled_dot_product_attention in float64 on the CPU
  (dense when k >= n, boolean-masked for an arbitrary S, causal for prefill).
* Closed forms, invariances, the GQA head map against explicit head expansion,
  and a hand-worked example under tests/golden/.

The arithmetic these check is the routing equation and the per-layer attention
equation of the picx.dev summary (Methodology > Architecture Overview) with the
1/sqrt(d_k) scale of the zhichai.net post (Background: Attention and Its Limits).
"""
import math
import os

import numpy as np
import pytest
import torch
from hypothesis import given, settings, strategies as st

from oracle import clsa_oracle as O
from long_context_sparse_clsa_b200.inputs import (WORKLOADS, make_inputs, scaled,
                                                  bf16_bits_to_f32, f32_to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------- helpers (independent)

def brute_topk(scores, n, k):
    """Token j is selected iff fewer than k tokens beat it: a larger score, or the
    same score and a lower index.  Counting formulation, no sort."""
    s = [float(x) for x in scores[:n]]
    sel = []
    for j in range(n):
        beats = sum(1 for i in range(n) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if beats < k:
            sel.append(j)
    return sel


def sdpa(q, k, v, mask=None, scale=None):
    """torch SDPA in float64: q [H][Mq][d], k/v [H][N][d], mask bool [Mq][N] (True=keep)."""
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    m = None if mask is None else torch.as_tensor(np.asarray(mask, dtype=bool))
    return torch.nn.functional.scaled_dot_product_attention(
        q[None], k[None], v[None], attn_mask=m, scale=scale)[0].numpy()


def rand(rng, *shape):
    return rng.standard_normal(shape)


# ----------------------------------------------------------------- worked example

def _golden():
    vals = {}
    for line in open(os.path.join(GOLDEN, "worked_example_n4.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val = (x.strip() for x in line.split("=", 1))
        vals[key] = val
    consts = {"sqrt2ln3": math.sqrt(2) * math.log(3), "ln4": math.log(4), "ln2": math.log(2)}

    def num(tok):
        return consts[tok] if tok in consts else float(tok)

    def arr(key):
        rows = [[num(t) for t in r.split()] for r in vals[key].split(";")]
        return np.array(rows if len(rows) > 1 else rows[0])
    return arr


def test_worked_example():
    g = _golden()
    q_idx = g("q_idx")[None]
    k_idx = g("k_idx")[None]
    lens = [4]
    I = O.index_scores(q_idx, k_idx, lens)
    np.testing.assert_array_equal(I[0], g("scores"))
    for kk in (1, 2, 3, 9):
        idx, cnt = O.topk_select(I, lens, kk)
        want = g(f"topk_{kk}").astype(int).reshape(-1)
        assert cnt[0] == want.size
        np.testing.assert_array_equal(idx[0, : cnt[0]], want)
        assert (idx[0, cnt[0]:] == -1).all()
    idx, cnt = O.topk_select(I, lens, 2)
    K = g("K").reshape(1, 4, 1, 2)
    V = g("V").reshape(1, 4, 1, 2)
    Q = np.stack([g("Q0"), g("Q1")]).reshape(2, 1, 1, 2)
    out, lse = O.sparse_attention(Q, K, V, idx, cnt)
    np.testing.assert_allclose(out[0, 0, 0], g("O_k2_layer0"), rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[1, 0, 0], g("O_k2_layer1"), rtol=0, atol=1e-12)
    assert abs(lse[0, 0, 0] - g("lse_k2_layer0").item()) < 1e-12
    assert abs(lse[1, 0, 0] - g("lse_k2_layer1").item()) < 1e-12


# ----------------------------------------------------------------- indexer

def test_index_scores_unit_vectors_and_mask():
    rng = np.random.default_rng(1)
    B, n, dI = 3, 37, 8
    kx = rand(rng, B, n, dI)
    lens = [37, 20, 1]
    for c in range(dI):
        q = np.zeros((B, dI))
        q[:, c] = 1.0
        I = O.index_scores(q, kx, lens)
        for b in range(B):
            np.testing.assert_array_equal(I[b, : lens[b]], kx[b, : lens[b], c])
            assert np.isneginf(I[b, lens[b]:]).all()


def test_index_scores_bilinear():
    rng = np.random.default_rng(2)
    B, n, dI = 2, 50, 16
    kx = rand(rng, B, n, dI)
    q1, q2 = rand(rng, B, dI), rand(rng, B, dI)
    lens = [n, n]
    I1, I2 = O.index_scores(q1, kx, lens), O.index_scores(q2, kx, lens)
    I12 = O.index_scores(2.0 * q1 - 3.0 * q2, kx, lens)
    np.testing.assert_allclose(I12, 2.0 * I1 - 3.0 * I2, rtol=1e-12, atol=1e-12)


def test_index_scores_bf16_bits_are_upcast_exactly():
    rng = np.random.default_rng(3)
    q = rng.standard_normal((1, 8)).astype(np.float32)
    kx = rng.standard_normal((1, 5, 8)).astype(np.float32)
    qb, kb = f32_to_bf16_bits(q), f32_to_bf16_bits(kx)
    I_bits = O.index_scores(qb, kb, [5])
    I_vals = O.index_scores(bf16_bits_to_f32(qb), bf16_bits_to_f32(kb), [5])
    np.testing.assert_array_equal(I_bits, I_vals)


# ----------------------------------------------------------------- TopK

@settings(max_examples=200, deadline=None)
@given(st.integers(1, 48).flatmap(lambda n: st.tuples(
    st.just(n),
    st.lists(st.integers(-3, 3), min_size=n, max_size=n),
    st.integers(1, 56),
    st.integers(1, n))))
def test_topk_matches_brute_force_with_ties(case):
    n, vals, k, length = case
    scores = np.array([vals], dtype=np.float64)
    idx, cnt = O.topk_select(scores, [length], k)
    want = brute_topk(scores[0], length, k)
    assert cnt[0] == len(want) == min(k, length)
    assert list(idx[0, : cnt[0]]) == want
    assert (idx[0, cnt[0]:] == -1).all()


@settings(max_examples=100, deadline=None)
@given(st.lists(st.floats(-1e3, 1e3, allow_nan=False, width=32), min_size=1, max_size=64),
       st.integers(1, 70))
def test_topk_matches_brute_force_continuous(vals, k):
    scores = np.array([vals], dtype=np.float64)
    idx, cnt = O.topk_select(scores, [len(vals)], k)
    assert list(idx[0, : cnt[0]]) == brute_topk(scores[0], len(vals), k)


def test_topk_negative_zero_ties_to_lower_index():
    scores = np.array([[-1.0, 0.0, -0.0, 0.0, -0.0, -2.0]])
    idx, cnt = O.topk_select(scores, [6], 3)
    assert list(idx[0]) == [1, 2, 3]       # the four zeros tie; the lower indices win
    idx, cnt = O.topk_select(scores, [6], 2)
    assert list(idx[0]) == [1, 2]
    scores = np.array([[-0.0, 0.0]])
    assert list(O.topk_select(scores, [2], 1)[0][0]) == [0]


def test_topk_rejects_nan():
    with pytest.raises(ValueError):
        O.topk_select(np.array([[1.0, np.nan]]), [2], 1)


def test_topk_empty_row():
    idx, cnt = O.topk_select(np.zeros((2, 4)), [0, 4], 3)
    assert cnt.tolist() == [0, 3]
    assert (idx[0] == -1).all()


# ----------------------------------------------------------------- attention

@pytest.mark.parametrize("L,B,Hq,Hkv,d,n", [(2, 1, 4, 1, 8, 9), (3, 2, 8, 2, 16, 13), (1, 1, 2, 2, 4, 1)])
def test_full_selection_equals_dense_sdpa(L, B, Hq, Hkv, d, n):
    rng = np.random.default_rng(10 + L)
    Q, K, V = rand(rng, L, B, Hq, d), rand(rng, B, n, Hkv, d), rand(rng, B, n, Hkv, d)
    idx = np.tile(np.arange(n, dtype=np.int32), (B, 1))
    out, lse = O.sparse_attention(Q, K, V, idx, np.full(B, n))
    G = Hq // Hkv
    for l in range(L):
        for b in range(B):
            Kx = np.repeat(K[b].transpose(1, 0, 2), G, axis=0)   # [Hq][n][d], head h -> kv h//G
            Vx = np.repeat(V[b].transpose(1, 0, 2), G, axis=0)
            ref = sdpa(Q[l, b][:, None, :], Kx, Vx)[:, 0]
            np.testing.assert_allclose(out[l, b], ref, rtol=1e-12, atol=1e-12)
            s = np.einsum("hd,hnd->hn", Q[l, b], Kx) / math.sqrt(d)
            np.testing.assert_allclose(lse[l, b], np.log(np.exp(s).sum(1)), rtol=1e-12)


def test_restricted_equals_masked_sdpa():
    rng = np.random.default_rng(20)
    L, B, Hq, Hkv, d, n, k = 2, 2, 4, 2, 8, 31, 7
    Q, K, V = rand(rng, L, B, Hq, d), rand(rng, B, n, Hkv, d), rand(rng, B, n, Hkv, d)
    idx = np.full((B, k), -1, dtype=np.int32)
    cnt = np.array([7, 4])
    for b in range(B):
        idx[b, : cnt[b]] = np.sort(rng.choice(n, cnt[b], replace=False))
    out, _ = O.sparse_attention(Q, K, V, idx, cnt)
    for b in range(B):
        mask = np.zeros((1, n), dtype=bool)
        mask[0, idx[b, : cnt[b]]] = True
        for l in range(L):
            for h in range(Hq):
                g = h // (Hq // Hkv)
                ref = sdpa(Q[l, b, h][None, None], K[b, :, g][None], V[b, :, g][None], mask)
                np.testing.assert_allclose(out[l, b, h], ref[0, 0], rtol=1e-12, atol=1e-12)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(21)
    for _ in range(20):
        Ks = rand(rng, 50, 16) * 10
        w, _ = O.attention_weights(rand(rng, 16), Ks)
        assert abs(w.sum() - 1.0) < 1e-12 and (w >= 0).all()


def test_closed_forms():
    rng = np.random.default_rng(22)
    d, n = 8, 12
    q = rand(rng, 1, 1, 1, d)
    idx = np.arange(n, dtype=np.int32)[None]
    # all keys equal -> output is the mean of the selected values
    K = np.tile(rand(rng, 1, 1, 1, d), (1, n, 1, 1))
    V = rand(rng, 1, n, 1, d)
    out, lse = O.sparse_attention(q, K, V, idx, [n])
    np.testing.assert_allclose(out[0, 0, 0], V[0, :, 0].mean(0), atol=1e-12)
    s0 = float(q[0, 0, 0] @ K[0, 0, 0]) / math.sqrt(d)
    assert abs(lse[0, 0, 0] - (s0 + math.log(n))) < 1e-12
    # all value rows equal c -> output is c
    V2 = np.tile(np.arange(d, dtype=np.float64)[None, None, None], (1, n, 1, 1))
    out, _ = O.sparse_attention(q, rand(rng, 1, n, 1, d), V2, idx, [n])
    np.testing.assert_allclose(out[0, 0, 0], np.arange(d), atol=1e-12)
    # one key aligned with q and scaled up -> output is its value row
    K3 = rand(rng, 1, n, 1, d)
    K3[0, 5, 0] = q[0, 0, 0] * 200.0
    out, _ = O.sparse_attention(q, K3, V, idx, [n])
    np.testing.assert_allclose(out[0, 0, 0], V[0, 5, 0], atol=1e-9)


def test_gqa_equals_mha_with_repeated_heads():
    rng = np.random.default_rng(23)
    L, B, Hq, Hkv, d, n, k = 2, 1, 8, 2, 8, 20, 6
    Q, K, V = rand(rng, L, B, Hq, d), rand(rng, B, n, Hkv, d), rand(rng, B, n, Hkv, d)
    idx = np.sort(rng.choice(n, k, replace=False)).astype(np.int32)[None]
    a, _ = O.sparse_attention(Q, K, V, idx, [k])
    G = Hq // Hkv
    b_, _ = O.sparse_attention(Q, np.repeat(K, G, axis=2), np.repeat(V, G, axis=2), idx, [k])
    np.testing.assert_allclose(a, b_, atol=1e-12)


def test_layer_and_token_permutations():
    rng = np.random.default_rng(24)
    L, B, Hq, Hkv, d, n, k = 5, 1, 4, 2, 8, 40, 9
    inp_q = rand(rng, B, d)
    kx = rand(rng, B, n, d)
    Q, K, V = rand(rng, L, B, Hq, d), rand(rng, B, n, Hkv, d), rand(rng, B, n, Hkv, d)
    r = O.decode_step(inp_q, kx, K, V, Q, [n], k)
    perm = rng.permutation(L)
    r2 = O.decode_step(inp_q, kx, K, V, Q[perm], [n], k)
    np.testing.assert_allclose(r2["O"], r["O"][perm], atol=1e-12)
    np.testing.assert_array_equal(r2["idx"], r["idx"])
    tp = rng.permutation(n)                      # cache row i of the new cache = old row tp[i]
    r3 = O.decode_step(inp_q, kx[:, tp], K[:, tp], V[:, tp], Q, [n], k)
    np.testing.assert_array_equal(np.sort(tp[r3["idx"][0]]), r["idx"][0])
    np.testing.assert_allclose(r3["O"], r["O"], atol=1e-12)


def test_gather_matches_index_select():
    rng = np.random.default_rng(25)
    K, V = rand(rng, 2, 30, 2, 4), rand(rng, 2, 30, 2, 4)
    idx = np.array([[3, 7, 29, -1], [0, 1, 2, 3]], dtype=np.int32)
    KS, VS = O.gather_kv(K, V, idx, [3, 4])
    for b, c in ((0, 3), (1, 4)):
        t = torch.as_tensor(K[b]).index_select(0, torch.as_tensor(idx[b, :c], dtype=torch.long))
        np.testing.assert_array_equal(KS[b, :c], t.numpy())
    assert (KS[0, 3] == 0).all() and (VS[0, 3] == 0).all()


def test_decode_ragged_full_selection_equals_masked_dense():
    rng = np.random.default_rng(26)
    L, B, Hq, Hkv, d, n, dI = 2, 2, 4, 2, 8, 24, 8
    lens = [24, 11]
    q, kx = rand(rng, B, dI), rand(rng, B, n, dI)
    Q, K, V = rand(rng, L, B, Hq, d), rand(rng, B, n, Hkv, d), rand(rng, B, n, Hkv, d)
    r = O.decode_step(q, kx, K, V, Q, lens, 64)
    G = Hq // Hkv
    for b in range(B):
        assert r["count"][b] == lens[b]
        mask = np.zeros((1, n), dtype=bool)
        mask[0, : lens[b]] = True
        Kx = np.repeat(K[b].transpose(1, 0, 2), G, axis=0)
        Vx = np.repeat(V[b].transpose(1, 0, 2), G, axis=0)
        for l in range(L):
            ref = sdpa(Q[l, b][:, None, :], Kx, Vx, mask)[:, 0]
            np.testing.assert_allclose(r["O"][l, b], ref, atol=1e-12)


# ----------------------------------------------------------------- prefill

def test_prefill_full_budget_equals_causal_sdpa():
    rng = np.random.default_rng(30)
    L, T, n, Hq, Hkv, d, dI = 2, 6, 14, 4, 2, 8, 8
    q, kx = rand(rng, T, dI), rand(rng, n, dI)
    Q, K, V = rand(rng, L, T, Hq, d), rand(rng, n, Hkv, d), rand(rng, n, Hkv, d)
    r = O.prefill_chunk(q, kx, K, V, Q, n, k=n)
    mask = np.zeros((T, n), dtype=bool)
    for i in range(T):
        mask[i, : n - T + i + 1] = True
    assert r["count"].tolist() == [n - T + i + 1 for i in range(T)]
    G = Hq // Hkv
    Kx = np.repeat(K.transpose(1, 0, 2), G, axis=0)
    Vx = np.repeat(V.transpose(1, 0, 2), G, axis=0)
    for l in range(L):
        ref = sdpa(Q[l].transpose(1, 0, 2), Kx, Vx, mask)            # [Hq][T][d]
        np.testing.assert_allclose(r["O"][l], ref.transpose(1, 0, 2), atol=1e-12)


def test_prefill_topk_budget_and_causality():
    rng = np.random.default_rng(31)
    T, n, dI, k = 9, 12, 4, 5
    q, kx = rand(rng, T, dI), rand(rng, n, dI)
    idx, cnt = O.prefill_topk(q, kx, n, k)
    for i in range(T):
        t = n - T + i
        assert cnt[i] == min(k, t + 1)
        sel = idx[i, : cnt[i]]
        assert sel.max() <= t
        s = kx[: t + 1] @ q[i]
        assert list(sel) == brute_topk(s, t + 1, k)


def test_prefill_rows_subset_matches_full():
    rng = np.random.default_rng(32)
    L, T, n, Hq, Hkv, d, dI, k = 1, 5, 10, 2, 1, 4, 4, 3
    args = (rand(rng, T, dI), rand(rng, n, dI), rand(rng, n, Hkv, d), rand(rng, n, Hkv, d),
            rand(rng, L, T, Hq, d))
    full = O.prefill_chunk(*args, n=n, k=k)
    sub = O.prefill_chunk(*args, n=n, k=k, rows=[4, 0])
    np.testing.assert_array_equal(sub["idx"], full["idx"][[4, 0]])
    np.testing.assert_allclose(sub["O"], full["O"][:, [4, 0]], atol=1e-12)


# ----------------------------------------------------------------- generator sanity

def test_inputs_are_deterministic_and_shaped():
    w = scaled("decode32k", n_max=2048, k=64, L=2)
    a, b = make_inputs(w), make_inputs(w)
    for name in ("q_idx", "k_idx", "K", "V", "Q"):
        np.testing.assert_array_equal(getattr(a, name), getattr(b, name))
    assert a.K.shape == (1, 2048, 8, 128) and a.Q.shape == (2, 1, 32, 128)
    assert len(a.planted[0]) == 20
    r = make_inputs(scaled("ragged16", B=3, n_max=512, lens=(100, 512), L=1, k=32))
    for bb in range(3):
        assert (r.K[bb, r.seq_lens[bb]:] == 0).all()
    v = a.f32("K").ravel()
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01


# ----------------------------------------------------------------------- distillation target

def _softmax_t(x):
    return torch.softmax(torch.as_tensor(x, dtype=torch.float64), dim=-1).numpy()


def test_distill_single_head_is_that_heads_softmax():
    """L = 1, one head: Abar is that head's attention distribution (torch's softmax of the
    scaled scores over the valid rows), zero past len."""
    rng = np.random.default_rng(11)
    d, n_max, n = 16, 30, 23
    Q = rng.normal(size=(1, 1, 1, d))
    K = rng.normal(size=(1, n_max, 1, d))
    I = rng.normal(size=(1, n_max))
    A, _ = O.distill_target(Q, K, I, [n])
    want = _softmax_t((K[0, :n, 0] @ Q[0, 0, 0]) / np.sqrt(d))
    assert np.allclose(A[0, :n], want, rtol=1e-12, atol=1e-15)
    assert np.all(A[0, n:] == 0.0)


def test_distill_head_mapping_with_a_zero_kv_head():
    """Hq = 4, Hkv = 2: query heads 2, 3 read KV head 1.  With KV head 1 all zeros their
    distributions are uniform, so Abar = (softmax_h0 + softmax_h1 + 2 / n) / 4 with h0, h1
    on KV head 0 (a mapping h % Hkv would put heads 1 and 3 on the zero head instead)."""
    rng = np.random.default_rng(12)
    d, n = 8, 17
    Q = rng.normal(size=(1, 1, 4, d))
    K = rng.normal(size=(1, n, 2, d))
    K[:, :, 1] = 0.0
    A, _ = O.distill_target(Q, K, rng.normal(size=(1, n)), [n])
    s0 = _softmax_t((K[0, :, 0] @ Q[0, 0, 0]) / np.sqrt(d))
    s1 = _softmax_t((K[0, :, 0] @ Q[0, 0, 1]) / np.sqrt(d))
    assert np.allclose(A[0], (s0 + s1 + 2.0 / n) / 4.0, rtol=1e-12, atol=1e-15)


def test_distill_kl_against_scipy_and_closed_forms():
    """kl = KL(Abar || softmax(I)) equals scipy's entropy(Abar, softmax(I)); it is >= 0, and
    0 when I = log Abar + c; Abar sums to 1 over each sequence's rows."""
    from scipy.stats import entropy
    rng = np.random.default_rng(13)
    L, B, Hq, Hkv, d, n_max = 3, 3, 4, 2, 8, 40
    Q = rng.normal(size=(L, B, Hq, d))
    K = rng.normal(size=(B, n_max, Hkv, d))
    I = 3.0 * rng.normal(size=(B, n_max))
    lens = [40, 7, 0]
    A, kl = O.distill_target(Q, K, I, lens)
    for b, n in enumerate(lens):
        if n == 0:
            assert kl[b] == 0.0 and np.all(A[b] == 0.0)
            continue
        assert abs(A[b, :n].sum() - 1.0) < 1e-12 and np.all(A[b, n:] == 0.0)
        assert kl[b] >= 0.0
        assert abs(kl[b] - entropy(A[b, :n], _softmax_t(I[b, :n]))) < 1e-12
    I2 = I.copy()
    I2[0, :40] = np.log(A[0, :40]) + 5.0
    _, kl2 = O.distill_target(Q, K, I2, lens)
    assert abs(kl2[0]) < 1e-12


def test_distill_invariances():
    """Properties the definition fixes: softmax(I) is shift invariant, so kl ignores a constant
    added to I (a missing lse of I would not); permuting the cached tokens (K rows with their
    I) permutes Abar the same way and keeps kl; permuting the layers, or the query heads inside
    one KV group, leaves the average Abar unchanged."""
    rng = np.random.default_rng(14)
    L, B, Hq, Hkv, d, n = 3, 2, 4, 2, 8, 33
    Q = rng.normal(size=(L, B, Hq, d))
    K = rng.normal(size=(B, n, Hkv, d))
    I = 2.0 * rng.normal(size=(B, n))
    lens = [n, 20]
    A, kl = O.distill_target(Q, K, I, lens)
    _, kl_shift = O.distill_target(Q, K, I + 7.5, lens)
    np.testing.assert_allclose(kl_shift, kl, rtol=1e-10, atol=1e-12)
    perm = rng.permutation(n)
    K2, I2 = K[:, perm].copy(), I[:, perm].copy()
    lens2 = [n, n]  # every row valid, so the permutation stays inside the valid range
    A_full, kl_full = O.distill_target(Q, K, I, lens2)
    A2, kl2 = O.distill_target(Q, K2, I2, lens2)
    np.testing.assert_allclose(A2, A_full[:, perm], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(kl2, kl_full, rtol=1e-10)
    Q3 = Q[rng.permutation(L)][:, :, [1, 0, 3, 2]]  # layers shuffled; heads swapped within each KV group
    A3, kl3 = O.distill_target(Q3, K, I, lens)
    np.testing.assert_allclose(A3, A, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(kl3, kl, rtol=1e-10)


# --------------------------------------------------------------------- attention-mass coverage
# picx.dev CLSA summary, Attention Sparsity Analysis: the share of the dense softmax mass on S

def test_attention_mass_against_torch_softmax_and_closed_forms():
    rng = np.random.default_rng(17)
    L, B, Hq, Hkv, d, n = 2, 2, 4, 2, 16, 40
    Q = rng.standard_normal((L, B, Hq, d))
    K = rng.standard_normal((B, n, Hkv, d))
    lens = np.array([n, 23])
    idx = np.full((B, 10), -1)
    count = np.array([10, 7])
    for b in range(B):
        idx[b, :count[b]] = np.sort(rng.choice(lens[b], count[b], replace=False))
    got = O.attention_mass(Q, K, idx, count, lens)
    # an independent route: torch's float64 softmax over the whole row, summed over S
    for l in range(L):
        for b in range(B):
            for h in range(Hq):
                s = torch.tensor(K[b, :lens[b], h // 2] @ Q[l, b, h] / math.sqrt(d))
                p = torch.softmax(s, dim=0).numpy()
                assert abs(got[l, b, h] - p[idx[b, :count[b]]].sum()) < 1e-12
    assert np.all((got > 0) & (got < 1))
    # every row selected: the whole mass
    full = np.tile(np.arange(n), (B, 1))
    np.testing.assert_allclose(O.attention_mass(Q, K, full, lens, lens), 1.0, atol=1e-12)
    # equal keys: the mass is the selected fraction |S| / n
    Ke = np.repeat(K[:, :1], n, axis=1)
    np.testing.assert_allclose(O.attention_mass(Q, Ke, idx, count, lens)[:, 0], count[0] / n, atol=1e-12)
    np.testing.assert_allclose(O.attention_mass(Q, Ke, idx, count, lens)[:, 1], count[1] / lens[1], atol=1e-12)
    # one dominant key: ~1 when it is selected, ~0 when not
    Kd = K.copy()
    j = int(idx[0, 0])
    Kd[0, j, :] = 60 * Q[0, 0, 0] / np.linalg.norm(Q[0, 0, 0])
    assert O.attention_mass(Q, Kd, idx, count, lens)[0, 0, 0] > 1 - 1e-9
    other = np.array([[k for k in range(n) if k != j][:10], idx[1]])
    assert O.attention_mass(Q, Kd, other, count, lens)[0, 0, 0] < 1e-9
    # an empty sequence: 0
    assert np.all(O.attention_mass(Q, K, idx, np.array([0, 7]), np.array([0, 23]))[:, 0] == 0)
