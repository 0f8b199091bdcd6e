"""The allocation-free TopK entry point, clsa_topk_noalloc.

Some callers cannot call cudaMalloc (they run inside another runtime's memory
pool, or on a path that must not synchronise the device), so they cannot hand
clsa_topk a workspace.  clsa_topk_noalloc keeps its scratch in a fixed array
inside the library.  This file checks, through the C ABI, that two calls in a
row return exactly what clsa_topk returns on the same scores and what the
oracle's TopK returns (TopK indices are integers: the tolerance is bit-exact),
that each call is one kernel launch, and that a size is refused exactly when
its scratch would exceed the fixed array.  It is named to be collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_clsa_b200 import clsa
from oracle import clsa_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from long_context_sparse_clsa_b200.build import build
    build()
    return clsa.load_library()


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("B,n,k,kind", [(1, 131072, 2048, "normal"), (16, 60000, 2048, "ragged"),
                                        (3, 5000, 700, "ties"), (300, 2000, 64, "normal")])
def test_noalloc_matches_workspace_topk_twice(lib, B, n, k, kind):
    rng = np.random.default_rng(B + n + k)
    if kind == "ties":
        s = rng.integers(-9, 9, size=(B, n)).astype(np.float32)
    else:
        s = (rng.standard_normal((B, n)) * 11).astype(np.float32)
    lens = np.full(B, n, dtype=np.int32)
    if kind == "ragged":
        lens = rng.integers(1, n + 1, size=B).astype(np.int32)
    scores = torch.tensor(s, device="cuda")
    L = torch.tensor(lens, device="cuda")
    ref_idx, ref_cnt = clsa.topk(scores, L, k)
    want_idx, want_cnt = O.topk_select(s.astype(np.float64), lens, k)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for _ in range(2):
        idx = torch.full((B, k), 7, dtype=torch.int32, device="cuda")
        cnt = torch.full((B,), 7, dtype=torch.int32, device="cuda")
        st = lib.clsa_topk_noalloc(_ptr(scores), _ptr(L), B, n, k, _ptr(idx), _ptr(cnt), stream)
        assert st == 0, clsa.STATUS.get(st)
        assert lib.clsa_last_launch_count() == 1
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)
        np.testing.assert_array_equal(idx.cpu().numpy(), want_idx)
        np.testing.assert_array_equal(cnt.cpu().numpy(), want_cnt)


@pytest.mark.parametrize("B", [16, 64, 512])
def test_noalloc_refuses_exactly_beyond_its_scratch(lib, B):
    """Refused iff clsa_topk's workspace for the size exceeds the 2 MiB array: at
    n = 128K a middle range of B (rows that still get several CTAs each) is refused;
    with more rows than CTAs every row runs alone and needs no inter-CTA scratch."""
    n, k = 131072, 2048
    scores = torch.randn(B, n, device="cuda") * 11
    L = torch.full((B,), n, dtype=torch.int32, device="cuda")
    idx = torch.empty(B, k, dtype=torch.int32, device="cuda")
    cnt = torch.empty(B, dtype=torch.int32, device="cuda")
    need = lib.clsa_topk_workspace_size(B, n, k)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = lib.clsa_topk_noalloc(_ptr(scores), _ptr(L), B, n, k, _ptr(idx), _ptr(cnt), stream)
    if need > (2 << 20):
        assert clsa.STATUS[st] == "CLSA_ERR_UNSUPPORTED"
    else:
        assert st == 0
        ref_idx, ref_cnt = clsa.topk(scores, L, k)
        torch.cuda.synchronize()
        assert torch.equal(idx, ref_idx) and torch.equal(cnt, ref_cnt)
