"""Seeded synthetic inputs for the CLSA decode and prefill paths.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path.  It holds
no arithmetic of the method itself: it only draws numbers, rounds them to the
storage precision, and lays them out.

Workloads follow the shapes of the 128K-context efficiency runs of
"You Only Index Once: Cross-Layer Sparse Attention with Shared Routing"
(picx.dev summary, "Inference Efficiency"; the pages give no model shape, so the
head layout, k and the value distribution are the stated synthetic stand-ins).

Random numbers
--------------
Every tensor is filled from a counter-based stream, so element ``i`` of stream
``s`` depends only on ``(seed, s, i)``.  That keeps generation chunkable (a thread
pool fills 8M-element chunks) and independent of the tensor's padding:

* 64-bit hash: SplitMix64's output function (Steele, Lea and Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014) applied to
  ``base + i * 0x9E3779B97F4A7C15``, with ``base`` derived from (seed, stream).
* N(0,1) pairs: the Box-Muller transform (Box and Muller, 1958) on two 24-bit
  uniforms taken from the hash, computed in float32.

Small integer draws (ragged lengths, planted-token positions) use numpy's PCG64
with a SeedSequence spawned from the same seed.

bf16 values are rounded from float32 with round-to-nearest-even and stored as
raw ``uint16`` bits; ``Inputs.f32(name)`` returns the exact float32 values those
bits encode, which is what the oracle upcasts to float64.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "Inputs", "make_inputs", "counter_normal",
    "f32_to_bf16_bits", "bf16_bits_to_f32",
]

# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------


@dataclass(frozen=True)
class Workload:
    """One synthetic CLSA workload.

    mode      "decode" (one query token per sequence) or "prefill" (T new rows)
    B         sequences (decode); 1 for prefill
    n_max     cache capacity per sequence (prefill: total cache length n)
    lens      None -> every sequence holds n_max tokens; (lo, hi) -> uniform
              integer lengths in [lo, hi] per sequence
    d_idx     index-key width (single indexer head)
    k         top-k budget (prefill uses min(k, t+1) for row t)
    L         cross-decoder layers sharing the routing index
    Hq, Hkv   query heads / KV heads (GQA, contiguous grouping)
    d         head dimension
    dtype     "f32" or "bf16" storage of every floating input
    plant     fraction of cache tokens whose index key is boosted toward the
              query (salient tokens), 0 for none
    T         prefill rows (the last T positions of the n-token cache)
    q_corr    prefill only: correlation rho of consecutive rows' index queries, an AR(1)
              sequence q_t = rho q_{t-1} + sqrt(1 - rho^2) z_t over the N(0, 1) draws
              z_t (each row stays N(0, 1)); 0 leaves the draws independent
    """

    name: str
    mode: str = "decode"
    B: int = 1
    n_max: int = 4096
    lens: Optional[Tuple[int, int]] = None
    d_idx: int = 64
    k: int = 256
    L: int = 4
    Hq: int = 8
    Hkv: int = 2
    d: int = 64
    dtype: str = "f32"
    plant: float = 0.0
    T: int = 0
    seed: int = 0
    q_corr: float = 0.0

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


WORKLOADS: Dict[str, Workload] = {
    # batch 1, one query, n=4096, fp32, k=256, L=4, 8 q-heads / 2 kv-heads, d=64
    "tiny": Workload("tiny"),
    # batch 1 at 32K, bf16, k=2048, L=16, 32/8 heads, d=128, 1% planted tokens
    "decode32k": Workload("decode32k", n_max=32768, d_idx=128, k=2048, L=16, Hq=32,
                          Hkv=8, d=128, dtype="bf16", plant=0.01),
    # batch 1 at 128K, L=24: the headline decode workload
    "decode128k": Workload("decode128k", n_max=131072, d_idx=128, k=2048, L=24, Hq=32,
                           Hkv=8, d=128, dtype="bf16", plant=0.01),
    # 16 sequences, ragged lengths U[16384, 131072]
    "ragged16": Workload("ragged16", B=16, n_max=131072, lens=(16384, 131072), d_idx=128,
                         k=2048, L=24, Hq=32, Hkv=8, d=128, dtype="bf16"),
    # 4096 new rows appended to a 126976-token cache (n = 131072), causal
    "prefill4k": Workload("prefill4k", mode="prefill", n_max=131072, d_idx=128, k=2048,
                          L=24, Hq=32, Hkv=8, d=128, dtype="bf16", T=4096),
    # the same with consecutive rows' index queries correlated (rho = 0.95): neighbouring
    # rows select overlapping token sets, as consecutive tokens of real text tend to
    "prefill4k_corr": Workload("prefill4k_corr", mode="prefill", n_max=131072, d_idx=128, k=2048,
                               L=24, Hq=32, Hkv=8, d=128, dtype="bf16", T=4096, q_corr=0.95),
}

# stream ids, in the order the tensors are described
_S_QIDX, _S_KIDX, _S_PLANT, _S_K, _S_V, _S_Q, _S_LENS = range(7)

# --------------------------------------------------------------------------
# counter-based N(0,1)
# --------------------------------------------------------------------------

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK_PAIRS = 1 << 22
_POOL: Optional[ThreadPoolExecutor] = None


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z ^ (z >> np.uint64(30))
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def _stream_base(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([((seed & 0xFFFFFFFF) * 0x100000001 + stream * 0x1000193 + 1) % (1 << 64)],
                     dtype=np.uint64)
        return _mix64(_mix64(s))[0]


def _normal_pairs(base: np.uint64, pair0: int, npairs: int, out: np.ndarray) -> None:
    i = np.arange(pair0, pair0 + npairs, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = _mix64(i * _GAMMA + base)
    hi = (z >> np.uint64(40)).astype(np.float32)
    lo = ((z >> np.uint64(8)) & np.uint64(0xFFFFFF)).astype(np.float32)
    u1 = (hi + np.float32(1.0)) * np.float32(2.0 ** -24)     # (0, 1]
    u2 = lo * np.float32(2.0 ** -24)                          # [0, 1)
    r = np.sqrt(np.float32(-2.0) * np.log(u1))
    t = np.float32(2.0 * math.pi) * u2
    v = np.empty(2 * npairs, dtype=np.float32)
    v[0::2] = r * np.cos(t)
    v[1::2] = r * np.sin(t)
    if out.dtype == np.uint16:
        out[:] = f32_to_bf16_bits(v)[: out.size]
    else:
        out[:] = v[: out.size]


def counter_normal(seed: int, stream: int, start: int, count: int,
                   bf16: bool = False) -> np.ndarray:
    """N(0,1) values for counter positions [start, start+count) of a stream.

    Returns float32, or (``bf16=True``) the values rounded to bf16 as uint16 bits.
    ``start`` must be even (values come in Box-Muller pairs).
    """
    global _POOL
    if start % 2:
        raise ValueError("start must be even")
    npairs = (count + 1) // 2
    out = np.empty(2 * npairs, dtype=np.uint16 if bf16 else np.float32)
    base = _stream_base(seed, stream)
    p0 = start // 2
    jobs = [(c, min(_CHUNK_PAIRS, npairs - c)) for c in range(0, npairs, _CHUNK_PAIRS)]
    if len(jobs) == 1:
        _normal_pairs(base, p0, npairs, out)
    else:
        if _POOL is None:
            _POOL = ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1)))
        list(_POOL.map(lambda j: _normal_pairs(base, p0 + j[0], j[1],
                                               out[2 * j[0]: 2 * (j[0] + j[1])]), jobs))
    return out[:count]


# --------------------------------------------------------------------------
# bf16 storage
# --------------------------------------------------------------------------


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# inputs
# --------------------------------------------------------------------------


@dataclass
class Inputs:
    """Host arrays for one workload, in storage form.

    Shapes (decode):  q_idx [B][d_idx], k_idx [B][n_max][d_idx],
                      K, V [B][n_max][Hkv][d], Q [L][B][Hq][d], seq_lens int32 [B]
    Shapes (prefill): q_idx [T][d_idx], k_idx [n][d_idx], K, V [n][Hkv][d],
                      Q [L][T][Hq][d], seq_lens = [n]
    bf16 tensors are uint16 bit arrays; f32 tensors are float32 arrays.
    Rows j >= seq_lens[b] of the caches are zero.
    """

    workload: Workload
    q_idx: np.ndarray
    k_idx: np.ndarray
    K: np.ndarray
    V: np.ndarray
    Q: np.ndarray
    seq_lens: np.ndarray
    planted: list = field(default_factory=list)

    def f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a

    def nbytes(self) -> int:
        return sum(getattr(self, n).nbytes for n in ("q_idx", "k_idx", "K", "V", "Q"))


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if dtype == "bf16" else x.astype(np.float32, copy=False)


def _fill_rows(seed: int, stream: int, shape, lens, dtype: str) -> np.ndarray:
    """[B][n_max][...] tensor; only the first lens[b] rows of sequence b are drawn."""
    B, n_max = shape[0], shape[1]
    row = int(np.prod(shape[2:]))
    out = np.zeros(shape, dtype=np.uint16 if dtype == "bf16" else np.float32)
    flat = out.reshape(B, n_max * row)
    per_seq = n_max * row + (n_max * row) % 2
    for b in range(B):
        cnt = int(lens[b]) * row
        if cnt:
            flat[b, :cnt] = counter_normal(seed, stream, b * per_seq, cnt, bf16=dtype == "bf16")
    return out


def make_inputs(w: Workload, seed: Optional[int] = None) -> Inputs:
    """Draw every tensor of workload ``w``; identical bits on every call."""
    seed = w.seed if seed is None else seed
    rng_small = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    if w.mode == "decode":
        B, n = w.B, w.n_max
        if w.lens is None:
            lens = np.full(B, n, dtype=np.int32)
        else:
            lo, hi = w.lens
            lens = np.random.Generator(np.random.PCG64(np.random.SeedSequence(
                [seed, _S_LENS]))).integers(lo, hi, size=B, endpoint=True).astype(np.int32)
        q32 = counter_normal(seed, _S_QIDX, 0, B * w.d_idx).reshape(B, w.d_idx)
        q_st = _store(q32, w.dtype)
        q_val = bf16_bits_to_f32(q_st) if w.dtype == "bf16" else q_st
        kidx32 = np.zeros((B, n, w.d_idx), dtype=np.float32)
        per_seq = n * w.d_idx
        for b in range(B):
            cnt = int(lens[b]) * w.d_idx
            kidx32[b].reshape(-1)[:cnt] = counter_normal(seed, _S_KIDX, b * per_seq, cnt)
        planted = []
        if w.plant > 0:
            prng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _S_PLANT])))
            for b in range(B):
                m = int(math.floor(w.plant * int(lens[b])))
                js = np.sort(prng.choice(int(lens[b]), size=m, replace=False)) if m else np.zeros(0, int)
                u = q_val[b] / np.float32(np.linalg.norm(q_val[b].astype(np.float64)))
                kidx32[b, js] += np.float32(3.0) * u.astype(np.float32)
                planted.append(js.astype(np.int64))
        k_st = _store(kidx32, w.dtype)
        del kidx32
        K = _fill_rows(seed, _S_K, (B, n, w.Hkv, w.d), lens, w.dtype)
        V = _fill_rows(seed, _S_V, (B, n, w.Hkv, w.d), lens, w.dtype)
        Q = counter_normal(seed, _S_Q, 0, w.L * B * w.Hq * w.d,
                           bf16=w.dtype == "bf16").reshape(w.L, B, w.Hq, w.d)
        return Inputs(w, q_st, k_st, K, V, Q, lens, planted)
    if w.mode == "prefill":
        n, T = w.n_max, w.T
        if not (1 <= T <= n):
            raise ValueError("prefill needs 1 <= T <= n")
        qz = counter_normal(seed, _S_QIDX, 0, T * w.d_idx).reshape(T, w.d_idx)
        if w.q_corr:
            if not 0.0 < w.q_corr < 1.0:
                raise ValueError("q_corr must lie in [0, 1)")
            rho, tail = np.float32(w.q_corr), np.float32(math.sqrt(1.0 - w.q_corr ** 2))
            for t in range(1, T):  # in float32, row by row
                qz[t] = rho * qz[t - 1] + tail * qz[t]
        q = _store(qz, w.dtype)
        kidx = _store(counter_normal(seed, _S_KIDX, 0, n * w.d_idx).reshape(n, w.d_idx), w.dtype)
        lens = np.array([n], dtype=np.int32)
        K = _fill_rows(seed, _S_K, (1, n, w.Hkv, w.d), lens, w.dtype)[0]
        V = _fill_rows(seed, _S_V, (1, n, w.Hkv, w.d), lens, w.dtype)[0]
        Q = counter_normal(seed, _S_Q, 0, w.L * T * w.Hq * w.d,
                           bf16=w.dtype == "bf16").reshape(w.L, T, w.Hq, w.d)
        return Inputs(w, q, kidx, K, V, Q, lens, [])
    raise ValueError(f"unknown mode {w.mode!r}")


def scaled(name: str, **overrides) -> Workload:
    """A named workload with some fields replaced (smaller parity cases)."""
    return replace(WORKLOADS[name], **overrides)
