"""The seeded input generator, pinned to definitions outside this repository.

Both the oracle and the CUDA path consume these inputs, so parity cannot see a mistake
here; these tests pin each step instead:

* the hash is SplitMix64's output function (Steele, Lea and Flood, OOPSLA 2014): its
  published first outputs for seed 0;
* bf16 storage is round-to-nearest-even: torch's float32 -> bfloat16 conversion, bit for
  bit, ties included;
* the normals are standard normal (Kolmogorov-Smirnov against scipy's N(0, 1)), and the
  stream is counter-based (any slice equals the same positions of a longer draw);
* the planted-token recipe: floor(1 % of len) rows of K_idx, moved by 3 q_idx / |q_idx|
  before rounding, so that their scores rise by exactly 3 |q_idx| (+3 sigma of the score
  distribution, whose sigma is |q_idx| for N(0, 1) keys).
"""
import math

import numpy as np
import torch
from scipy import stats

from long_context_sparse_clsa_b200 import inputs as I
from long_context_sparse_clsa_b200.inputs import (bf16_bits_to_f32, counter_normal, f32_to_bf16_bits,
                                                  make_inputs, scaled)


def test_splitmix64_reference_outputs():
    # SplitMix64 seeded with 0: state += 0x9E3779B97F4A7C15, output = mix(state)
    i = np.arange(1, 4, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = I._mix64(i * I._GAMMA)
    assert [int(x) for x in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def _torch_bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).view(torch.int16) \
        .numpy().view(np.uint16)


def test_bf16_round_to_nearest_even_matches_torch():
    rng = np.random.default_rng(3)
    x = (rng.normal(size=20000) * np.exp2(rng.integers(-30, 30, size=20000))).astype(np.float32)
    # exact halfway cases below and above an even and an odd bf16 mantissa, and their neighbours
    sign = rng.integers(0, 2, size=2000, dtype=np.uint32) << np.uint32(31)
    expo = rng.integers(1, 254, size=2000, dtype=np.uint32) << np.uint32(23)  # finite, normal
    mant = rng.integers(0, 1 << 7, size=2000, dtype=np.uint32) << np.uint32(16)  # the bf16 mantissa
    hi = sign | expo | mant
    ties = np.concatenate([hi | np.uint32(0x8000), hi | np.uint32(0x7FFF), hi | np.uint32(0x8001)]).view(np.float32)
    assert np.isfinite(ties).all()
    for v in (x, ties, np.array([0.0, -0.0, 1.0, -2.5, 3.0e38, -3.0e38, 1e-40], dtype=np.float32)):
        np.testing.assert_array_equal(f32_to_bf16_bits(v), _torch_bf16_bits(v))
    b = f32_to_bf16_bits(x)
    np.testing.assert_array_equal(bf16_bits_to_f32(b), torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_counter_normal_is_a_standard_normal_counter_stream():
    full = counter_normal(5, 3, 0, 20000)
    np.testing.assert_array_equal(counter_normal(5, 3, 1000, 5000), full[1000:6000])
    np.testing.assert_array_equal(counter_normal(5, 3, 1000, 5000, bf16=True), f32_to_bf16_bits(full[1000:6000]))
    assert not np.array_equal(counter_normal(5, 4, 0, 100), full[:100])  # another stream
    assert not np.array_equal(counter_normal(6, 3, 0, 100), full[:100])  # another seed
    big = counter_normal(1, 2, 0, 1 << 20).astype(np.float64)
    assert stats.kstest(big, "norm").pvalue > 1e-3
    assert np.isfinite(big).all()


def test_planted_rows_move_scores_by_three_norms():
    w = scaled("decode32k", n_max=3000, k=64, L=1)
    inp = make_inputs(w)
    n, d = int(inp.seq_lens[0]), w.d_idx
    js = inp.planted[0]
    assert len(js) == math.floor(w.plant * n) == 30 and len(set(js.tolist())) == 30
    q = inp.f32("q_idx")[0]
    u = q / np.float32(np.linalg.norm(q.astype(np.float64)))
    raw = counter_normal(w.seed, I._S_KIDX, 0, n * d).reshape(n, d)  # the rows before planting
    want = raw.copy()
    want[js] += np.float32(3.0) * u.astype(np.float32)
    np.testing.assert_array_equal(inp.k_idx[0, :n], f32_to_bf16_bits(want))
    # in exact arithmetic on the unrounded rows the planted scores rise by 3 |q|
    qn = np.linalg.norm(q.astype(np.float64))
    shift = want[js].astype(np.float64) @ q.astype(np.float64) - raw[js].astype(np.float64) @ q.astype(np.float64)
    np.testing.assert_allclose(shift, 3.0 * qn, rtol=1e-5)
    # and after bf16 rounding they still stand ~3 sigma above the rest (sigma = |q|)
    s = bf16_bits_to_f32(inp.k_idx[0, :n]).astype(np.float64) @ q.astype(np.float64)
    rest = np.setdiff1d(np.arange(n), js)
    assert abs(s[rest].std() / qn - 1.0) < 0.05
    assert abs((s[js].mean() - s[rest].mean()) / qn - 3.0) < 0.6


def test_correlated_prefill_queries():
    """q_corr: an AR(1) sequence of index queries over the prefill rows.  rho = 0 gives the
    independent draws bit for bit; rho = 0.95 keeps each row N(0, 1), correlates neighbours
    at ~rho, and makes neighbouring rows' TopK sets (the oracle's) overlap heavily, where
    independent rows share few tokens."""
    from oracle import clsa_oracle as O
    base = scaled("prefill4k", n_max=2048, T=256, L=1, k=64)
    np.testing.assert_array_equal(make_inputs(base).q_idx, make_inputs(scaled("prefill4k", n_max=2048, T=256, L=1,
                                                                               k=64, q_corr=0.0)).q_idx)
    overlap = {}
    for rho in (0.0, 0.95):
        inp = make_inputs(scaled("prefill4k", n_max=2048, T=256, L=1, k=64, q_corr=rho))
        q = bf16_bits_to_f32(inp.q_idx).astype(np.float64)
        if rho:
            assert abs(q.std() - 1.0) < 0.05
            assert abs(np.corrcoef(q[1:].ravel(), q[:-1].ravel())[0, 1] - rho) < 0.02
        idx, cnt = O.prefill_topk(inp.q_idx, inp.k_idx, 2048, 64)
        shared = [len(set(idx[t, :cnt[t]]) & set(idx[t + 1, :cnt[t + 1]])) / cnt[t] for t in range(255)]
        overlap[rho] = float(np.mean(shared))
    assert overlap[0.0] < 0.1 and overlap[0.95] > 0.5, overlap
