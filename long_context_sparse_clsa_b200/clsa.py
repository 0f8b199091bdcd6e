"""Thin Python binding of libclsa.so (include/clsa.h): argument marshalling only.

Every function takes torch CUDA tensors, passes their device pointers and the
current torch stream to the C ABI and raises ``ClsaError`` on a non-OK status.
All arithmetic happens in the library's CUDA kernels; there is no fallback.  If
the library has not been built, the first call raises ``RuntimeError`` naming
the build command.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libclsa.so")

CLSA_F32, CLSA_BF16 = 0, 1
STATUS = {0: "CLSA_OK", 1: "CLSA_ERR_INVALID_ARG", 2: "CLSA_ERR_UNSUPPORTED", 3: "CLSA_ERR_WORKSPACE",
          4: "CLSA_ERR_CUDA", 5: "CLSA_ERR_TIMEOUT", 6: "CLSA_ERR_BAD_INDEX"}

# every symbol include/clsa.h declares
EXPORTS = [
    "clsa_index_scores", "clsa_topk_workspace_size", "clsa_topk", "clsa_topk_noalloc",
    "clsa_gather_kv_workspace_size",
    "clsa_gather_kv", "clsa_sparse_attn_workspace_size", "clsa_sparse_attn",
    "clsa_distill_workspace_size", "clsa_distill_target", "clsa_attention_mass_workspace_size",
    "clsa_attention_mass",
    "clsa_decode_workspace_size", "clsa_decode_step", "clsa_prefill_workspace_size",
    "clsa_prefill_chunk", "clsa_prefill_attention", "clsa_workspace_size", "clsa_workspace_init", "clsa_read_device_status", "clsa_status_string",
    "clsa_selftest_timeout", "clsa_version", "clsa_last_launch_count", "clsa_time_next_call",
    "clsa_timed_event_count",
]


class ClsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code
        self.status = STATUS.get(code, str(code))


_vp, _i, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float


class DecodeArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("B", _i), ("n_max", _i), ("d_idx", _i), ("k", _i), ("L", _i),
                ("Hq", _i), ("Hkv", _i), ("d", _i), ("scale", _f),
                ("q_idx", _vp), ("k_idx", _vp), ("K", _vp), ("V", _vp), ("Q", _vp),
                ("seq_lens", _vp), ("O", _vp), ("idx", _vp), ("count", _vp), ("scores", _vp),
                ("lse", _vp), ("K_S", _vp), ("V_S", _vp)]


class PrefillArgs(ctypes.Structure):
    _fields_ = [("dtype", _i), ("n", _i), ("T", _i), ("d_idx", _i), ("k", _i), ("L", _i),
                ("Hq", _i), ("Hkv", _i), ("d", _i), ("scale", _f),
                ("q_idx", _vp), ("k_idx", _vp), ("K", _vp), ("V", _vp), ("Q", _vp),
                ("O", _vp), ("idx", _vp), ("count", _vp), ("lse", _vp)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libclsa.so (once).  Raises RuntimeError if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m long_context_sparse_clsa_b200.build`")
    lib = ctypes.CDLL(path)
    S = ctypes.c_int
    sig = {
        "clsa_index_scores": (S, [_vp, _vp, _vp, _i, _i, _i, _i, _vp, _vp]),
        "clsa_topk_workspace_size": (_sz, [_i, _i, _i]),
        "clsa_topk": (S, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
        "clsa_topk_noalloc": (S, [_vp, _vp, _i, _i, _i, _vp, _vp, _vp]),
        "clsa_gather_kv_workspace_size": (_sz, []),
        "clsa_gather_kv": (S, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz, _vp]),
        "clsa_sparse_attn_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
        "clsa_sparse_attn": (S, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp,
                                 _sz, _vp]),
        "clsa_distill_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
        "clsa_attention_mass_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
        "clsa_attention_mass": (S, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp]),
        "clsa_distill_target": (S, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz, _vp]),
        "clsa_decode_workspace_size": (_sz, [ctypes.POINTER(DecodeArgs)]),
        "clsa_decode_step": (S, [ctypes.POINTER(DecodeArgs), _vp, _sz, _vp]),
        "clsa_prefill_workspace_size": (_sz, [ctypes.POINTER(PrefillArgs)]),
        "clsa_prefill_chunk": (S, [ctypes.POINTER(PrefillArgs), _vp, _sz, _vp]),
        "clsa_prefill_attention": (S, [ctypes.POINTER(PrefillArgs), _i, _vp, _sz, _vp]),
        "clsa_workspace_size": (_sz, [_i, _vp]),
        "clsa_workspace_init": (S, [_vp, _sz, _vp]),
        "clsa_read_device_status": (S, [_vp, _vp, ctypes.POINTER(ctypes.c_int64)]),
        "clsa_status_string": (ctypes.c_char_p, [S]),
        "clsa_selftest_timeout": (S, [_i, _vp, _sz, _vp]),
        "clsa_version": (_i, []),
        "clsa_last_launch_count": (_i, []),
        "clsa_time_next_call": (S, [ctypes.POINTER(ctypes.c_void_p), _i]),
        "clsa_timed_event_count": (_i, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


# ---------------------------------------------------------------------------- helpers

def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return CLSA_BF16
    if t.dtype == torch.float32:
        return CLSA_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise ClsaError(code, where)


def last_launch_count() -> int:
    """Kernel launches made by the most recent library call on this thread."""
    return load_library().clsa_last_launch_count()


class LaunchTimer:
    """Per-launch device times of one library call: arm() before the call; after the
    stream has synchronized, times_ms() gives each launch's duration (events the library
    records before its first launch and after each launch, on the call's stream)."""

    def __init__(self, max_launches: int = 16):
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(max_launches + 1)]
        for e in self.events:  # torch creates the CUDA event on its first record
            e.record()
        torch.cuda.synchronize()
        self._handles = (ctypes.c_void_p * len(self.events))(*[e.cuda_event for e in self.events])

    def arm(self):
        _check(load_library().clsa_time_next_call(self._handles, len(self.events)), "clsa_time_next_call")

    def times_ms(self):
        n = load_library().clsa_timed_event_count()
        return [self.events[i].elapsed_time(self.events[i + 1]) for i in range(n - 1)]


class Workspace:
    """A zero-initialised device workspace of at least ``nbytes`` bytes."""

    def __init__(self, nbytes: int, device=None):
        self.nbytes = max(int(nbytes), 256)
        self.buf = torch.empty(self.nbytes, dtype=torch.uint8, device=device or "cuda")
        _check(load_library().clsa_workspace_init(_p(self.buf), self.nbytes, _stream()), "workspace_init")

    @property
    def ptr(self):
        return _p(self.buf)

    def ensure(self, nbytes: int) -> "Workspace":
        return self if nbytes <= self.nbytes else Workspace(nbytes, self.buf.device)

    def status(self, stream=None):
        """(status name, detail) of the first device-detected error; clears it."""
        detail = ctypes.c_int64(0)
        code = load_library().clsa_read_device_status(self.ptr, _stream(stream), ctypes.byref(detail))
        return STATUS.get(code, str(code)), detail.value


def fused_decode_trace(ws: Workspace):
    """Diagnostics of the fused decode step: the per-CTA phase stamps the last step wrote into
    ``ws`` when the library ran with CLSA_TRACE=1 in the environment (int64 [256][64]:
    globaltimer ns per phase; a row whose slot 0 is 0 belongs to no CTA of that step).
    Slot 31 holds the CTA's candidate slot count, plus 2^32 when the candidate windows decided
    the TopK (0 there: the group took the whole-row selection)."""
    return ws.buf[256:256 + 256 * 64 * 8].view(torch.int64).view(256, 64).cpu()


# ---------------------------------------------------------------------------- calls

def index_scores(q_idx, k_idx, seq_lens, scores=None):
    lib = load_library()
    B, n_max, d_idx = k_idx.shape
    if scores is None:
        scores = torch.empty(B, n_max, dtype=torch.float32, device=k_idx.device)
    _check(lib.clsa_index_scores(_p(q_idx), _p(k_idx), _p(seq_lens), B, n_max, d_idx, _dt(k_idx),
                                 _p(scores), _stream()), "clsa_index_scores")
    return scores


def topk(scores, seq_lens, k, ws: Optional[Workspace] = None, idx=None, count=None):
    lib = load_library()
    B, n_max = scores.shape
    need = lib.clsa_topk_workspace_size(B, n_max, k)
    ws = (ws or Workspace(need)).ensure(need)
    idx = idx if idx is not None else torch.empty(B, k, dtype=torch.int32, device=scores.device)
    count = count if count is not None else torch.empty(B, dtype=torch.int32, device=scores.device)
    _check(lib.clsa_topk(_p(scores), _p(seq_lens), B, n_max, k, _p(idx), _p(count), ws.ptr, ws.nbytes,
                         _stream()), "clsa_topk")
    return idx, count


def topk_noalloc(scores, seq_lens, k, idx=None, count=None):
    """clsa_topk without a workspace (scratch inside the library; see clsa.h)."""
    lib = load_library()
    B, n_max = scores.shape
    idx = idx if idx is not None else torch.empty(B, k, dtype=torch.int32, device=scores.device)
    count = count if count is not None else torch.empty(B, dtype=torch.int32, device=scores.device)
    _check(lib.clsa_topk_noalloc(_p(scores), _p(seq_lens), B, n_max, k, _p(idx), _p(count), _stream()),
           "clsa_topk_noalloc")
    return idx, count


def gather_kv(K, V, idx, count, ws: Optional[Workspace] = None, K_S=None, V_S=None):
    lib = load_library()
    B, n_max, Hkv, d = K.shape
    k = idx.shape[1]
    ws = ws or Workspace(lib.clsa_gather_kv_workspace_size())
    K_S = K_S if K_S is not None else torch.zeros(B, k, Hkv, d, dtype=K.dtype, device=K.device)
    V_S = V_S if V_S is not None else torch.zeros(B, k, Hkv, d, dtype=K.dtype, device=K.device)
    _check(lib.clsa_gather_kv(_p(K), _p(V), _p(idx), _p(count), B, n_max, k, Hkv, d, _dt(K), _p(K_S),
                              _p(V_S), ws.ptr, ws.nbytes, _stream()), "clsa_gather_kv")
    return K_S, V_S


def sparse_attn(Q, K_S, V_S, count, scale: float = 0.0, ws: Optional[Workspace] = None, O=None,
                lse=None, want_lse: bool = True):
    """Q [L][B][Hq][d] (or [B][Hq][d] for one layer); K_S/V_S [B][k][Hkv][d]."""
    lib = load_library()
    squeeze = Q.dim() == 3
    Qv = Q.unsqueeze(0) if squeeze else Q
    L, B, Hq, d = Qv.shape
    _, k, Hkv, _ = K_S.shape
    need = lib.clsa_sparse_attn_workspace_size(B, k, L, Hq, Hkv, d)
    ws = (ws or Workspace(need)).ensure(need)
    O = O if O is not None else torch.empty_like(Qv)
    if want_lse and lse is None:
        lse = torch.empty(L, B, Hq, dtype=torch.float32, device=Q.device)
    _check(lib.clsa_sparse_attn(_p(Qv), _p(K_S), _p(V_S), _p(count), B, k, L, Hq, Hkv, d, scale, _dt(Qv),
                                _p(O), _p(lse), ws.ptr, ws.nbytes, _stream()), "clsa_sparse_attn")
    if squeeze:
        return O[0], (lse[0] if lse is not None else None)
    return O, lse


def decode_args(q_idx, k_idx, K, V, Q, seq_lens, k, O, idx, count, scores=None, lse=None, K_S=None,
                V_S=None, scale: float = 0.0) -> DecodeArgs:
    B, n_max, d_idx = k_idx.shape
    L, _, Hq, d = Q.shape
    Hkv = K.shape[2]
    return DecodeArgs(_dt(K), B, n_max, d_idx, k, L, Hq, Hkv, d, scale, _p(q_idx), _p(k_idx), _p(K),
                      _p(V), _p(Q), _p(seq_lens), _p(O), _p(idx), _p(count), _p(scores), _p(lse),
                      _p(K_S), _p(V_S))


def decode_workspace_size(args: DecodeArgs) -> int:
    return load_library().clsa_decode_workspace_size(ctypes.byref(args))


def attention_mass(Q, K, lse_sparse, seq_lens, scale: float = 0.0, ws: Optional[Workspace] = None,
                   mass=None, lse_all=None, want_lse_all: bool = True):
    """Share of the dense softmax mass on the selection (see clsa.h): returns (mass, lse_all),
    both fp32 [L][B][Hq]; lse_sparse is the decode step's lse output."""
    lib = load_library()
    L, B, Hq, d = Q.shape
    _, n_max, Hkv, _ = K.shape
    need = lib.clsa_attention_mass_workspace_size(B, n_max, L, Hq, Hkv, d)
    ws = (ws or Workspace(need)).ensure(need)
    if mass is None:
        mass = torch.empty(L, B, Hq, dtype=torch.float32, device=Q.device)
    if lse_all is None and want_lse_all:
        lse_all = torch.empty(L, B, Hq, dtype=torch.float32, device=Q.device)
    _check(lib.clsa_attention_mass(_p(Q), _p(K), _p(lse_sparse), _p(seq_lens), B, n_max, L, Hq, Hkv, d, scale,
                                   _dt(K), _p(mass), _p(lse_all), ws.ptr, ws.nbytes, _stream()), "clsa_attention_mass")
    return mass, lse_all


def distill_target(Q, K, scores, seq_lens, scale: float = 0.0, ws: Optional[Workspace] = None,
                   want_abar: bool = True, abar=None, kl=None):
    """Distillation target (forward): Abar [B][n_max] (or None) and kl [B] (see clsa.h).
    abar / kl: optional preallocated outputs (fp32 [B][n_max] / [B])."""
    lib = load_library()
    L, B, Hq, d = Q.shape
    _, n_max, Hkv, _ = K.shape
    need = lib.clsa_distill_workspace_size(B, n_max, L, Hq, Hkv, d)
    ws = (ws or Workspace(need)).ensure(need)
    if abar is None and want_abar:
        abar = torch.empty(B, n_max, dtype=torch.float32, device=Q.device)
    if kl is None:
        kl = torch.empty(B, dtype=torch.float32, device=Q.device)
    _check(lib.clsa_distill_target(_p(Q), _p(K), _p(scores), _p(seq_lens), B, n_max, L, Hq, Hkv, d, scale, _dt(Q),
                                   _p(abar), _p(kl), ws.ptr, ws.nbytes, _stream()), "clsa_distill_target")
    return abar, kl, ws


def selftest_timeout(which: int, ws: Optional[Workspace] = None):
    """Launch the failure-detection self-test (see clsa.h); returns its workspace, whose
    status() then reads CLSA_ERR_TIMEOUT with detail 900 + which."""
    ws = ws or Workspace(512)
    _check(load_library().clsa_selftest_timeout(which, ws.ptr, ws.nbytes, _stream()), "clsa_selftest_timeout")
    return ws


def decode_step_args(args: DecodeArgs, ws: Workspace, stream=None):
    """Run one decode step on prepared arguments (no allocation)."""
    _check(load_library().clsa_decode_step(ctypes.byref(args), ws.ptr, ws.nbytes, _stream(stream)),
           "clsa_decode_step")


def decode_step(q_idx, k_idx, K, V, Q, seq_lens, k, scale: float = 0.0, ws: Optional[Workspace] = None,
                compact: bool = False, want_scores: bool = False, want_lse: bool = True):
    """One CLSA decode step.  Returns dict(O, idx, count, lse, scores, K_S, V_S)."""
    B, n_max, _ = k_idx.shape
    L, _, Hq, d = Q.shape
    Hkv = K.shape[2]
    dev = K.device
    out = {
        "O": torch.empty_like(Q),
        "idx": torch.empty(B, k, dtype=torch.int32, device=dev),
        "count": torch.empty(B, dtype=torch.int32, device=dev),
        "lse": torch.empty(L, B, Hq, dtype=torch.float32, device=dev) if want_lse else None,
        "scores": torch.empty(B, n_max, dtype=torch.float32, device=dev) if want_scores else None,
        "K_S": torch.zeros(B, k, Hkv, d, dtype=K.dtype, device=dev) if compact else None,
        "V_S": torch.zeros(B, k, Hkv, d, dtype=K.dtype, device=dev) if compact else None,
    }
    a = decode_args(q_idx, k_idx, K, V, Q, seq_lens, k, out["O"], out["idx"], out["count"], out["scores"],
                    out["lse"], out["K_S"], out["V_S"], scale)
    need = decode_workspace_size(a)
    if need == 0:
        raise ClsaError(1, "clsa_decode_workspace_size")
    ws = (ws or Workspace(need)).ensure(need)
    decode_step_args(a, ws)
    out["ws"] = ws
    return out


def prefill_args(q_idx, k_idx, K, V, Q, k, O, idx, count, lse=None, scale: float = 0.0) -> PrefillArgs:
    T, d_idx = q_idx.shape
    n = k_idx.shape[0]
    L, _, Hq, d = Q.shape
    Hkv = K.shape[1]
    return PrefillArgs(_dt(K), n, T, d_idx, k, L, Hq, Hkv, d, scale, _p(q_idx), _p(k_idx), _p(K), _p(V),
                       _p(Q), _p(O), _p(idx), _p(count), _p(lse))


def prefill_workspace_size(args: PrefillArgs) -> int:
    return load_library().clsa_prefill_workspace_size(ctypes.byref(args))


def prefill_chunk(q_idx, k_idx, K, V, Q, k, scale: float = 0.0, ws: Optional[Workspace] = None,
                  want_lse: bool = True):
    """Causal prefill of T = q_idx.shape[0] rows at the end of an n-token cache."""
    T = q_idx.shape[0]
    L, _, Hq, d = Q.shape
    dev = K.device
    out = {
        "O": torch.empty_like(Q),
        "idx": torch.empty(T, k, dtype=torch.int32, device=dev),
        "count": torch.empty(T, dtype=torch.int32, device=dev),
        "lse": torch.empty(L, T, Hq, dtype=torch.float32, device=dev) if want_lse else None,
    }
    a = prefill_args(q_idx, k_idx, K, V, Q, k, out["O"], out["idx"], out["count"], out["lse"], scale)
    need = prefill_workspace_size(a)
    if need == 0:
        raise ClsaError(1, "clsa_prefill_workspace_size")
    ws = (ws or Workspace(need)).ensure(need)
    _check(load_library().clsa_prefill_chunk(ctypes.byref(a), ws.ptr, ws.nbytes, _stream()),
           "clsa_prefill_chunk")
    out["ws"] = ws
    return out


def prefill_attention(q_idx, k_idx, K, V, Q, k, idx, count, mode: int = 0, scale: float = 0.0,
                      ws: Optional[Workspace] = None, O=None, lse=None, want_lse: bool = True):
    """The attention stage of a prefill chunk over a selection already in idx / count (as
    prefill_chunk returns it).  mode 0: per row; mode 1: key-centric row pairs."""
    T = q_idx.shape[0]
    L, _, Hq, d = Q.shape
    O = O if O is not None else torch.empty_like(Q)
    if want_lse and lse is None:
        lse = torch.empty(L, T, Hq, dtype=torch.float32, device=K.device)
    a = prefill_args(q_idx, k_idx, K, V, Q, k, O, idx, count, lse, scale)
    need = prefill_workspace_size(a)
    ws = (ws or Workspace(need)).ensure(need)
    _check(load_library().clsa_prefill_attention(ctypes.byref(a), int(mode), ws.ptr, ws.nbytes, _stream()),
           "clsa_prefill_attention")
    return O, lse


def to_device(inp, device="cuda"):
    """Copy an ``inputs.Inputs`` bundle to the device as torch tensors (bf16 or fp32)."""
    import numpy as np

    def conv(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)
    return {"q_idx": conv(inp.q_idx), "k_idx": conv(inp.k_idx), "K": conv(inp.K), "V": conv(inp.V),
            "Q": conv(inp.Q), "seq_lens": torch.from_numpy(inp.seq_lens.astype(np.int32)).to(device)}
