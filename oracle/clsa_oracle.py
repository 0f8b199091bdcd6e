"""CPU oracle for the CLSA shared-routing sparse-attention path.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import or call this
module: only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` use it.  It shares no code, constant or
helper with the CUDA library; the only thing both sides share is the seeded input
generator (``long_context_sparse_clsa_b200.inputs``), which holds none of the
method's arithmetic.

What it computes is the plain definition from the pages about "You Only Index
Once: Cross-Layer Sparse Attention with Shared Routing" (CLSA):

* picx.dev summary, "Methodology > Architecture Overview", routing equation:
  ``I = Q_idx K_idx^T`` and ``S_t = TopK(I_t, k)``, computed once.
* same section, per-layer equation: ``O_t^(l) = Attn(Q_t^(l), K_{S_t}, V_{S_t})``
  for every cross-decoder layer l, reusing the one S_t.
* zhichai.net forum post "CLSA Explained", "Background: Attention and Its
  Limits": ``Attn(Q, K, V) = softmax(Q K^T / sqrt(d_k)) V`` (fixes the scale).
* zhichai.net post, "CLSA: Sharing the Index Across Layers": the "Selector"
  gathers K/V rows by the shared index.
* picx.dev summary, "Methodology > Architecture Overview", multi-layer
  distillation: ``Abar = 1/(L H) sum_{l,h} softmax(Q^(l,h) K^(h)^T)`` and the
  per-query term ``KL(sg[Abar_t] || softmax(I_t))`` (forward only).

All floating arithmetic is float64 on inputs upcast from their storage values.
Readings where the pages are silent:

* the indexer has no scale, bias or activation (the routing equation is a bare
  product, single head);
* attention scale is 1/sqrt(d) with d the head dimension;
* TopK ties go to the lower token index; -0.0 and +0.0 are equal;
* S_t is returned in ascending token order, padded with -1 when fewer than k
  tokens exist (k_eff = min(k, available tokens));
* the decode query attends over all len_b cached tokens; a prefill row at cache
  position t sees tokens j <= t (causal);
* one S_t per query token, shared by every layer and every head;
* GQA maps query head h to KV head h // (Hq / Hkv).
* the distillation target averages the distributions the layers attend with, so
  its softmax takes the attention scale 1/sqrt(d) (the printed formula omits any
  scale); softmax(I_t) takes none (the routing equation has none); a decode query
  sees all len_b cached tokens; 0 log 0 = 0.

Pins (tests/test_oracle_pins.py) tie every function here to something other than
itself: brute-force rank counting for TopK, torch's scaled_dot_product_attention
for dense and masked attention, closed forms, invariances and a hand-worked
example stored under tests/golden/.
"""
from __future__ import annotations

import math
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "index_scores", "topk_select", "gather_kv", "sparse_attention", "attention_weights",
    "decode_step", "prefill_scores", "prefill_topk", "prefill_attention", "prefill_chunk",
    "distill_target",
]


def _f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:          # bf16 bit patterns -> exact float values
        a = (a.astype(np.uint32) << np.uint32(16)).view(np.float32)
    return a.astype(np.float64)


# --------------------------------------------------------------------------
# indexer: picx.dev summary, Methodology > Architecture Overview, routing eq.
# --------------------------------------------------------------------------

def index_scores(q_idx, k_idx, seq_lens) -> np.ndarray:
    """I[b, j] = q_idx[b] . k_idx[b, j] for j < seq_lens[b]; -inf beyond.

    q_idx [B][d_idx], k_idx [B][n_max][d_idx]; returns float64 [B][n_max].
    """
    q = _f64(q_idx)
    kx = _f64(k_idx)
    B, n_max, _ = kx.shape
    out = np.full((B, n_max), -np.inf)
    for b in range(B):
        n = int(seq_lens[b])
        out[b, :n] = kx[b, :n] @ q[b]
    return out


# --------------------------------------------------------------------------
# routing: S_t = TopK(I_t, k)  (same equation)
# --------------------------------------------------------------------------

def _topk_row(scores_row: np.ndarray, n: int, k: int) -> np.ndarray:
    """Indices of the k_eff = min(k, n) largest of scores_row[:n], ascending.

    Order used to pick them: score descending, then token index ascending (a
    stable sort on the negated score).  NaN is rejected.
    """
    s = np.asarray(scores_row[:n], dtype=np.float64)
    if np.isnan(s).any():
        raise ValueError("NaN score")
    keff = min(k, n)
    order = np.lexsort((np.arange(n), -s))          # primary: -score; secondary: index
    return np.sort(order[:keff])


def topk_select(scores, seq_lens, k: int):
    """Per-row exact TopK.  Returns (idx int32 [B][k] ascending, -1 padded; count int32 [B])."""
    scores = np.asarray(scores)
    B = scores.shape[0]
    idx = np.full((B, k), -1, dtype=np.int32)
    count = np.zeros(B, dtype=np.int32)
    for b in range(B):
        sel = _topk_row(scores[b], int(seq_lens[b]), k)
        idx[b, : sel.size] = sel
        count[b] = sel.size
    return idx, count


# --------------------------------------------------------------------------
# Selector: gather the shared K/V rows once (zhichai.net post, CLSA section)
# --------------------------------------------------------------------------

def gather_kv(K, V, idx, count):
    """K_S[b, i] = K[b, idx[b, i]], V_S likewise, for i < count[b]; zeros beyond.

    K, V [B][n_max][Hkv][d]; returns float64 K_S, V_S [B][k][Hkv][d].
    """
    Kf, Vf = _f64(K), _f64(V)
    B, _, Hkv, d = Kf.shape
    k = idx.shape[1]
    KS = np.zeros((B, k, Hkv, d))
    VS = np.zeros((B, k, Hkv, d))
    for b in range(B):
        c = int(count[b])
        KS[b, :c] = Kf[b, idx[b, :c]]
        VS[b, :c] = Vf[b, idx[b, :c]]
    return KS, VS


# --------------------------------------------------------------------------
# per-layer attention: O^(l) = Attn(Q^(l), K_S, V_S), softmax(QK^T/sqrt(d))V
# --------------------------------------------------------------------------

def attention_weights(q, Ks, scale: Optional[float] = None):
    """softmax(Ks q * scale) over the rows of Ks; returns (weights, lse)."""
    q = np.asarray(q, dtype=np.float64)
    d = q.shape[-1]
    scale = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else scale
    s = (Ks @ q) * scale
    m = s.max()
    p = np.exp(s - m)
    den = p.sum()
    return p / den, m + math.log(den)


def _attend(q, Ks, Vs, scale):
    w, lse = attention_weights(q, Ks, scale)
    return w @ Vs, lse


def sparse_attention(Q, K, V, idx, count, scale: Optional[float] = None):
    """Token-sparse GQA attention of every layer over the shared selected rows.

    Q [L][B][Hq][d]; K, V [B][n_max][Hkv][d]; idx [B][>=count] token indices.
    Head h of any layer reads KV head h // (Hq // Hkv).  Returns float64
    (O [L][B][Hq][d], lse [L][B][Hq]).  A row with count 0 gives O = 0, lse = -inf.
    """
    Qf, Kf, Vf = _f64(Q), _f64(K), _f64(V)
    L, B, Hq, d = Qf.shape
    Hkv = Kf.shape[2]
    G = Hq // Hkv
    O = np.zeros((L, B, Hq, d))
    lse = np.full((L, B, Hq), -np.inf)
    for b in range(B):
        c = int(count[b])
        if c == 0:
            continue
        sel = np.asarray(idx[b, :c], dtype=np.int64)
        for h in range(Hq):
            g = h // G
            Ks = Kf[b, sel, g]          # [c][d]  (the Selector's gather)
            Vs = Vf[b, sel, g]
            for l in range(L):
                O[l, b, h], lse[l, b, h] = _attend(Qf[l, b, h], Ks, Vs, scale)
    return O, lse


def decode_step(q_idx, k_idx, K, V, Q, seq_lens, k: int, scale: Optional[float] = None):
    """One CLSA decode step: score once, select once, attend in every layer."""
    I = index_scores(q_idx, k_idx, seq_lens)
    idx, count = topk_select(I, seq_lens, k)
    O, lse = sparse_attention(Q, K, V, idx, count, scale)
    return {"scores": I, "idx": idx, "count": count, "O": O, "lse": lse}


# --------------------------------------------------------------------------
# prefill chunk: the same equations for T new rows, causal
# --------------------------------------------------------------------------

def prefill_scores(q_idx, k_idx, n: int, rows: Optional[Sequence[int]] = None) -> np.ndarray:
    """I[i, j] = q_idx[i] . k_idx[j] for j <= t_i = n - T + i; -inf for j > t_i.

    q_idx [T][d_idx], k_idx [n][d_idx]; ``rows`` limits the output to those i.
    """
    q = _f64(q_idx)
    kx = _f64(k_idx)[:n]
    T = q.shape[0]
    rows = range(T) if rows is None else rows
    out = np.full((len(rows), n), -np.inf)
    for r, i in enumerate(rows):
        t = n - T + i
        out[r, : t + 1] = kx[: t + 1] @ q[i]
    return out


def prefill_topk(q_idx, k_idx, n: int, k: int, rows: Optional[Sequence[int]] = None):
    """Per-row TopK with k_eff = min(k, t + 1).  Returns (idx [R][k], count [R])."""
    T = np.asarray(q_idx).shape[0]
    rows = list(range(T)) if rows is None else list(rows)
    idx = np.full((len(rows), k), -1, dtype=np.int32)
    count = np.zeros(len(rows), dtype=np.int32)
    for r, i in enumerate(rows):
        t = n - T + i
        s = prefill_scores(q_idx, k_idx, n, [i])[0]
        sel = _topk_row(s, t + 1, k)
        idx[r, : sel.size] = sel
        count[r] = sel.size
    return idx, count


def prefill_attention(Q, K, V, idx, count, rows: Optional[Sequence[int]] = None,
                      scale: Optional[float] = None):
    """Per-row sparse attention, each prefill row over its own S_t.

    Q [L][T][Hq][d]; K, V [n][Hkv][d]; idx/count indexed like ``rows`` (all rows
    when None).  Returns (O [L][R][Hq][d], lse [L][R][Hq]).
    """
    Qf = _f64(Q)
    L, T, Hq, d = Qf.shape
    rows = list(range(T)) if rows is None else list(rows)
    Kb = np.asarray(K)[None]
    Vb = np.asarray(V)[None]
    O = np.zeros((L, len(rows), Hq, d))
    lse = np.full((L, len(rows), Hq), -np.inf)
    for r, i in enumerate(rows):
        o, s = sparse_attention(Qf[:, i: i + 1], Kb, Vb, np.asarray(idx)[r: r + 1],
                                np.asarray(count)[r: r + 1], scale)
        O[:, r] = o[:, 0]
        lse[:, r] = s[:, 0]
    return O, lse


def prefill_chunk(q_idx, k_idx, K, V, Q, n: int, k: int,
                  rows: Optional[Sequence[int]] = None, scale: Optional[float] = None):
    """Prefill path for the chosen rows: causal scores, per-row TopK, attention."""
    idx, count = prefill_topk(q_idx, k_idx, n, k, rows)
    O, lse = prefill_attention(Q, K, V, idx, count, rows, scale)
    return {"idx": idx, "count": count, "O": O, "lse": lse}


# --------------------------------------------------------------------------
# distillation target of the shared indexer (forward only)
# --------------------------------------------------------------------------

def attention_mass(Q, K, idx, count, seq_lens, scale: Optional[float] = None):
    """Attention-mass coverage (picx.dev CLSA summary, Attention Sparsity Analysis): for each
    layer l, sequence b and query head h, the share of the dense softmax over the len_b cached
    rows that falls on the selected rows idx[b, :count[b]].  Query head h reads KV head
    h // (Hq / Hkv).  Q [L][B][Hq][d], K [B][n_max][Hkv][d]; float64 [L][B][Hq], 0 for a
    sequence with no tokens.
    """
    Qf, Kf = _f64(Q), _f64(K)
    L, B, Hq, _ = Qf.shape
    G = Hq // Kf.shape[2]
    out = np.zeros((L, B, Hq))
    for b in range(B):
        n, c = int(seq_lens[b]), int(count[b])
        if n == 0 or c == 0:
            continue
        sel = np.asarray(idx[b, :c], dtype=np.int64)
        for l in range(L):
            for h in range(Hq):
                w, _ = attention_weights(Qf[l, b, h], Kf[b, :n, h // G], scale)
                out[l, b, h] = w[sel].sum()
    return out


def distill_target(Q, K, I, seq_lens, scale: Optional[float] = None):
    """Per decode query b: Abar_b = mean over every (layer, query head) of that head's
    softmax over the len_b cached tokens (query head h reads KV head h // (Hq / Hkv)),
    and kl[b] = KL(Abar_b || softmax(I_b[:len_b])).

    Q [L][B][Hq][d]; K [B][n_max][Hkv][d]; I [B][n_max] indexer scores.  Returns float64
    (Abar [B][n_max] with zeros past len_b, kl [B]; a sequence with no tokens gets kl 0).
    """
    Qf, Kf = _f64(Q), _f64(K)
    If = np.asarray(I, dtype=np.float64)
    L, B, Hq, d = Qf.shape
    Hkv = Kf.shape[2]
    G = Hq // Hkv
    n_max = Kf.shape[1]
    Abar = np.zeros((B, n_max))
    kl = np.zeros(B)
    for b in range(B):
        n = int(seq_lens[b])
        if n == 0:
            continue
        acc = np.zeros(n)
        for l in range(L):
            for h in range(Hq):
                w, _ = attention_weights(Qf[l, b, h], Kf[b, :n, h // G], scale)
                acc += w
        a = acc / (L * Hq)
        Abar[b, :n] = a
        z = If[b, :n]
        log_p = z - (z.max() + math.log(np.exp(z - z.max()).sum()))  # log softmax(I_b)
        nz = a > 0
        kl[b] = float(np.sum(a[nz] * (np.log(a[nz]) - log_p[nz])))
    return Abar, kl

