"""Comparison systems for the CLSA decode step, built only from this library's calls.

The pages compare CLSA with the same model family with parts of its sharing taken
away (zhichai.net post, Ablations: per-layer index recompute, YOCO only, standard
attention; picx.dev CLSA summary, Complexity Comparison: the indexer cost is paid
once instead of once per layer as in DSA, and Inference Efficiency).  On B200 they
are:

* ``per_layer_routing`` (DSA-style; "without cross-layer shared index"): every
  cross-decoder layer scores the shared cache with its own indexer (its own q_idx and
  K_idx), selects its own TopK and attends over it.  One fused decode step per layer
  (L = 1 each) over the one shared K/V cache: the scan and the selection run L times.
* ``yoco_dense`` (YOCO only, no sparsity): every layer attends densely over the one
  shared cache.  One ``clsa_sparse_attn`` call with the whole cache as K_S/V_S and
  count = seq_lens: the L*G query rows of a KV head read each cached row once.
* ``standard`` (standard attention): every layer has its own K/V cache and attends
  densely over it.  One ``clsa_sparse_attn`` call per layer over that layer's cache.

Each is argument marshalling around the C ABI: every step runs in the library's
kernels, and the calls of one step go out back to back on one stream.

``attention_mass`` is the pages' sparsity diagnostic (picx.dev CLSA summary, Attention
Sparsity Analysis): the share of each (layer, query head)'s dense softmax mass that the
shared selection S captures, sum_{j in S} softmax_j = exp(lse_S - lse_all), from the lse
of the sparse attention over S and of the dense attention over the whole cache.
"""
from __future__ import annotations

from typing import Sequence

from . import clsa


class PerLayerRouting:
    """One fused decode step per layer, each with that layer's indexer inputs.

    q_idx_layers[l] [B][d_idx], k_idx_layers[l] [B][n_max][d_idx]; K, V [B][n_max][Hkv][d]
    shared by every layer; Q [L][B][Hq][d].  Outputs O [L][B][Hq][d], idx [L][B][k],
    count [L][B] (layer l's selection).
    """

    def __init__(self, q_idx_layers: Sequence, k_idx_layers: Sequence, K, V, Q, seq_lens, k: int,
                 O, idx, count, scale: float = 0.0):
        L = Q.shape[0]
        if len(q_idx_layers) != L or len(k_idx_layers) != L:
            raise ValueError("one indexer input per layer")
        self.args = [clsa.decode_args(q_idx_layers[l], k_idx_layers[l], K, V, Q[l:l + 1], seq_lens, k,
                                      O[l:l + 1], idx[l], count[l], scale=scale) for l in range(L)]
        self._keep = (q_idx_layers, k_idx_layers, K, V, Q, seq_lens, O, idx, count)
        self.ws = clsa.Workspace(clsa.decode_workspace_size(self.args[0]))

    def step(self) -> int:
        """Run one step; returns the kernel launches it made."""
        n = 0
        for a in self.args:  # one workspace: the calls run one after another on the stream
            clsa.decode_step_args(a, self.ws)
            n += clsa.last_launch_count()
        return n


class YocoDense:
    """Dense attention of every layer over the one shared cache (one call)."""

    def __init__(self, K, V, Q, seq_lens, O, scale: float = 0.0):
        self.K, self.V, self.Q, self.seq_lens, self.O, self.scale = K, V, Q, seq_lens, O, scale
        L, B, Hq, d = Q.shape
        n_max, Hkv = K.shape[1], K.shape[2]
        self.ws = clsa.Workspace(clsa.load_library().clsa_sparse_attn_workspace_size(B, n_max, L, Hq, Hkv, d))

    def step(self) -> int:
        clsa.sparse_attn(self.Q, self.K, self.V, self.seq_lens, self.scale, ws=self.ws, O=self.O, want_lse=False)
        return clsa.last_launch_count()


class StandardAttention:
    """Dense attention of layer l over its own cache K_layers[l], V_layers[l] (L calls)."""

    def __init__(self, K_layers: Sequence, V_layers: Sequence, Q, seq_lens, O, scale: float = 0.0):
        L, B, Hq, d = Q.shape
        if len(K_layers) != L or len(V_layers) != L:
            raise ValueError("one K/V cache per layer")
        self.K, self.V, self.Q, self.seq_lens, self.O, self.scale = K_layers, V_layers, Q, seq_lens, O, scale
        n_max, Hkv = K_layers[0].shape[1], K_layers[0].shape[2]
        self.ws = clsa.Workspace(clsa.load_library().clsa_sparse_attn_workspace_size(B, n_max, 1, Hq, Hkv, d))

    def step(self) -> int:
        n = 0
        for l in range(self.Q.shape[0]):
            clsa.sparse_attn(self.Q[l:l + 1], self.K[l], self.V[l], self.seq_lens, self.scale, ws=self.ws,
                             O=self.O[l:l + 1], want_lse=False)
            n += clsa.last_launch_count()
        return n


def attention_mass(Q, K, V, seq_lens, lse_sparse, scale: float = 0.0, ws=None):
    """Share of the dense softmax mass on the selected rows, per (layer, sequence, head):
    clsa_attention_mass (one streaming pass over K for the dense lse; V is not needed).
    Returns (mass [L][B][Hq] fp32, lse_all).  The pages' figure (~80 % at 2048 of 32K
    tokens) needs trained weights; on synthetic N(0, 1) inputs the indexer keys are
    independent of K, so the share is close to |S| / n.
    """
    del V  # the lse over the cache does not depend on V
    return clsa.attention_mass(Q, K, lse_sparse, seq_lens, scale, ws=ws)
