"""Shared helpers for the GPU parity tests (no method arithmetic of their own,
except the fp32 rounding bound used as the score tolerance)."""
import numpy as np
import torch

U32 = 2.0 ** -24  # unit roundoff of fp32


def score_tol(q_idx, k_idx, lens):
    """Forward-error bound of an fp32 dot product of exact products (bf16 x bf16,
    or fp32 x fp32 rounded once): |fl(sum) - sum| <= gamma_{d+1} * sum |q_c k_c|,
    gamma_m = m u / (1 - m u).  Per element, [B][n_max], float64."""
    q = np.abs(np.asarray(q_idx, dtype=np.float64))
    kx = np.abs(np.asarray(k_idx, dtype=np.float64))
    d = q.shape[-1]
    m = d + 1
    gamma = m * U32 / (1 - m * U32)
    out = np.zeros(kx.shape[:2])
    for b in range(kx.shape[0]):
        out[b, : lens[b]] = kx[b, : lens[b]] @ q[b] * gamma
    return out + 1e-30


def tensor_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check_near_tie_sets(gpu_idx, gpu_cnt, ora_scores, lens, k, rel=1e-4):
    """End-to-end rule: the GPU's set may differ from the exact TopK of the oracle
    scores only at tokens whose oracle score lies within rel * max|I| of the
    k-th largest oracle score."""
    for b in range(len(lens)):
        n = int(lens[b])
        keff = min(k, n)
        assert int(gpu_cnt[b]) == keff
        g = np.asarray(gpu_idx[b, :keff], dtype=np.int64)
        assert (np.diff(g) > 0).all(), "indices must be strictly ascending"
        assert (gpu_idx[b, keff:] == -1).all()
        if keff == 0:
            continue
        s = ora_scores[b, :n]
        kth = np.sort(s)[::-1][keff - 1]
        tol = rel * np.abs(s).max()
        exact = set(np.lexsort((np.arange(n), -s))[:keff].tolist())
        for j in set(g.tolist()) ^ exact:
            assert abs(s[j] - kth) <= tol, (b, j, s[j], kth, tol)


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))
