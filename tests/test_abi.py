"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol include/clsa.h declares, and rejects bad arguments before any launch."""
import ctypes
import os
import re

import pytest

from long_context_sparse_clsa_b200 import clsa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "clsa.h")


def header_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"CLSA_API\s+[\w\s\*]+?\b(clsa_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_clsa_b200.build import build
    build()
    return clsa.load_library()


def test_header_declares_the_six_calls():
    syms = header_symbols()
    for name in ("clsa_index_scores", "clsa_topk", "clsa_gather_kv", "clsa_sparse_attn",
                 "clsa_decode_step", "clsa_prefill_chunk"):
        assert name in syms


def test_library_exports_every_header_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
    assert sorted(clsa.EXPORTS) == header_symbols()


def test_status_strings_and_version(lib):
    for code, name in clsa.STATUS.items():
        assert lib.clsa_status_string(code).decode() == name
    assert lib.clsa_version() >= 100


NULL = None


def test_index_scores_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    assert lib.clsa_index_scores(NULL, p, p, 1, 16, 64, 0, p, NULL) == 1
    assert lib.clsa_index_scores(p, p, p, 0, 16, 64, 0, p, NULL) == 1
    assert lib.clsa_index_scores(p, p, p, 1, 16, 96, 0, p, NULL) == 2       # d_idx not 64/128
    assert lib.clsa_index_scores(ctypes.c_void_p(18), p, p, 1, 16, 64, 0, p, NULL) == 1  # misaligned


def test_topk_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    assert lib.clsa_topk(p, p, 1, 16, 0, p, p, p, 1 << 20, NULL) == 1      # k = 0
    assert lib.clsa_topk(p, p, 1, 16, 5000, p, p, p, 1 << 20, NULL) == 2   # k > 4096
    assert lib.clsa_topk(p, p, 1, 16, 4, p, p, NULL, 0, NULL) == 3         # no workspace


def test_sparse_attn_rejects_bad_shapes(lib):
    p = ctypes.c_void_p(16)
    ws = ctypes.c_void_p(256)
    args = dict(B=1, k=8, L=1, Hq=8, Hkv=3, d=64)
    assert lib.clsa_sparse_attn(p, p, p, p, 1, 8, 1, 8, 3, 64, 0.0, 1, p, NULL, ws, 1 << 30, NULL) == 2
    assert lib.clsa_sparse_attn(p, p, p, p, 1, 8, 1, 8, 2, 80, 0.0, 1, p, NULL, ws, 1 << 30, NULL) == 2
    assert lib.clsa_sparse_attn(p, p, p, p, 1, 8, 1, 8, 2, 64, 0.0, 7, p, NULL, ws, 1 << 30, NULL) == 1
    # fp32 path holds at most 32 query heads per KV head
    assert lib.clsa_sparse_attn(p, p, p, p, 1, 8, 1, 64, 1, 64, 0.0, 0, p, NULL, ws, 1 << 30, NULL) == 2
    del args


def test_decode_step_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    a = clsa.DecodeArgs(1, 1, 1024, 128, 64, 2, 8, 2, 128, 0.0, p, p, p, p, p, p, p, p, p, NULL, NULL,
                        p, NULL)  # K_S without V_S
    assert lib.clsa_decode_step(ctypes.byref(a), p, 1 << 30, NULL) == 1
    a.V_S = p
    a.d = 96
    assert lib.clsa_decode_step(ctypes.byref(a), p, 1 << 30, NULL) == 2
    assert lib.clsa_decode_workspace_size(ctypes.byref(a)) == 0
    assert lib.clsa_decode_step(None, p, 0, NULL) == 1


def test_prefill_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    a = clsa.PrefillArgs(1, 100, 200, 128, 16, 1, 8, 2, 64, 0.0, p, p, p, p, p, p, p, p, NULL)  # T > n
    assert lib.clsa_prefill_chunk(ctypes.byref(a), p, 1 << 30, NULL) == 1
    a.T, a.dtype = 50, 0
    assert lib.clsa_prefill_chunk(ctypes.byref(a), p, 1 << 30, NULL) == 2   # fp32 prefill unsupported


def test_prefill_attention_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    a = clsa.PrefillArgs(1, 100, 50, 128, 16, 1, 8, 2, 64, 0.0, p, p, p, p, p, p, p, p, NULL)
    assert lib.clsa_prefill_attention(None, 0, p, 1 << 30, NULL) == 1
    assert lib.clsa_prefill_attention(ctypes.byref(a), 2, p, 1 << 30, NULL) == 1    # no mode 2
    assert lib.clsa_prefill_attention(ctypes.byref(a), 1, p, 1 << 30, NULL) == 2    # key-centric: d = 128 only
    a.T = 200                                                                         # T > n
    assert lib.clsa_prefill_attention(ctypes.byref(a), 0, p, 1 << 30, NULL) == 1


def test_gather_kv_rejects_bad_args(lib):
    p, q = ctypes.c_void_p(16), ctypes.c_void_p(18)
    ws = ctypes.c_void_p(256)
    ok = [p, p, p, p, 1, 64, 8, 2, 128, 1, p, p, ws, 1 << 20, NULL]

    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return lib.clsa_gather_kv(*a)
    assert call(a0=NULL) == 1                  # no K
    assert call(a4=0) == 1                     # B = 0
    assert call(a9=7) == 1                     # no such dtype
    assert call(a8=96) == 2                    # d not 64 / 128
    assert call(a6=5000) == 2                  # k above 4096
    assert call(a0=q) == 1                     # K not 16-byte aligned
    assert call(a2=ctypes.c_void_p(18)) == 1   # idx not 4-byte aligned
    assert call(a12=NULL) == 3                 # no workspace
    assert call(a13=8) == 3                    # workspace below its header


@pytest.mark.parametrize("name", ["clsa_distill_target", "clsa_attention_mass"])
def test_distill_and_mass_reject_bad_args(lib, name):
    p, q = ctypes.c_void_p(16), ctypes.c_void_p(18)
    ws = ctypes.c_void_p(256)
    # Q, K, scores | lse_sparse, seq_lens, B, n_max, L, Hq, Hkv, d, scale, dt, out, out2, ws, ws_bytes, stream
    ok = [p, p, p, p, 1, 1024, 2, 8, 2, 128, 0.0, 1, p, p, ws, 1 << 30, NULL]
    fn = getattr(lib, name)

    def call(**kw):
        a = list(ok)
        for i, v in kw.items():
            a[int(i[1:])] = v
        return fn(*a)
    assert call(a4=0) == 1                     # B = 0
    assert call(a11=7) == 1                    # no such dtype
    assert call(a8=3) == 2                     # Hq not a multiple of Hkv
    assert call(a9=80) == 2                    # d not 64 / 128
    assert call(a0=NULL) == 1                  # no Q
    assert call(a1=q) == 1                     # K not 16-byte aligned
    assert call(a3=ctypes.c_void_p(18)) == 1   # seq_lens not 4-byte aligned


def test_topk_noalloc_rejects_bad_args(lib):
    p = ctypes.c_void_p(16)
    assert lib.clsa_topk_noalloc(NULL, p, 1, 16, 4, p, p, NULL) == 1                  # no scores
    assert lib.clsa_topk_noalloc(p, p, 1, 16, 0, p, p, NULL) == 1                     # k = 0
    assert lib.clsa_topk_noalloc(p, p, 0, 16, 4, p, p, NULL) == 1                     # B = 0
    assert lib.clsa_topk_noalloc(p, p, 1, 16, 5000, p, p, NULL) == 2                  # k above 4096
    assert lib.clsa_topk_noalloc(p, p, 1, 16, 4, ctypes.c_void_p(18), p, NULL) == 1   # idx misaligned


def test_oracle_is_not_imported_by_the_product():
    pkg = os.path.join(ROOT, "long_context_sparse_clsa_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle|clsa_oracle|#include.*oracle",
                                     text, re.M), f


def test_selftest_rejects_bad_args(lib):
    ws = ctypes.create_string_buffer(1024 + 16)
    base = (ctypes.addressof(ws) + 15) & ~15
    assert lib.clsa_selftest_timeout(2, base, 1024, None) == 1      # CLSA_ERR_INVALID_ARG
    assert lib.clsa_selftest_timeout(0, None, 1024, None) == 3      # CLSA_ERR_WORKSPACE
    assert lib.clsa_selftest_timeout(1, base, 300, None) == 3       # under 512 bytes
    assert lib.clsa_selftest_timeout(0, base + 4, 1000, None) == 3  # not 16-byte aligned


def test_generic_workspace_size_dispatches_by_op(lib):
    a = clsa.DecodeArgs(dtype=1, B=1, n_max=4096, d_idx=128, k=256, L=2, Hq=8, Hkv=2, d=128)
    for i, f in enumerate(["q_idx", "k_idx", "K", "V", "Q", "seq_lens", "O", "idx", "count"]):
        setattr(a, f, 0x100000 * (i + 1))  # aligned placeholders: the size calls never dereference
    p = clsa.PrefillArgs(dtype=1, n=4096, T=64, d_idx=128, k=256, L=2, Hq=8, Hkv=2, d=128)
    for i, f in enumerate(["q_idx", "k_idx", "K", "V", "Q", "O", "idx", "count"]):
        setattr(p, f, 0x100000 * (i + 1))
    dec, pre = lib.clsa_decode_workspace_size(ctypes.byref(a)), lib.clsa_prefill_workspace_size(ctypes.byref(p))
    assert dec > 0 and pre > 0
    assert lib.clsa_workspace_size(0, ctypes.byref(a)) == dec  # CLSA_OP_DECODE_STEP
    assert lib.clsa_workspace_size(1, ctypes.byref(p)) == pre  # CLSA_OP_PREFILL_CHUNK
    assert lib.clsa_workspace_size(2, ctypes.byref(p)) == 0
    assert lib.clsa_workspace_size(0, None) == 0
    a.k = 0  # rejected arguments: size 0, as from the op's own call
    assert lib.clsa_workspace_size(0, ctypes.byref(a)) == 0 == lib.clsa_decode_workspace_size(ctypes.byref(a))


def test_header_is_c99_and_a_c_program_links_and_calls(lib, tmp_path):
    """The boundary is a C ABI: clsa.h compiles as strict C99 and a C program links
    libclsa.so and calls it (here only calls that need no GPU)."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    src = tmp_path / "use_clsa.c"
    src.write_text(r"""
#include <stdio.h>
#include "clsa.h"
int main(void) {
  static char ws[1024];
  clsa_decode_args a = {0};
  if (clsa_version() < 100) return 1;
  printf("%s\n", clsa_status_string(CLSA_ERR_TIMEOUT));
  /* argument errors are returned before any device work */
  if (clsa_selftest_timeout(7, ws, sizeof ws, NULL) != CLSA_ERR_INVALID_ARG) return 2;
  if (clsa_workspace_size(CLSA_OP_PREFILL_CHUNK, NULL) != 0) return 3;
  if (clsa_decode_step(&a, NULL, 0, NULL) == CLSA_OK) return 4;
  return 0;
}
""")
    exe = tmp_path / "use_clsa"
    libdir = os.path.dirname(clsa.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.dirname(HEADER),
                    str(src), "-o", str(exe), "-L", libdir, "-l:libclsa.so", "-Wl,-rpath," + libdir], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, (out.returncode, out.stderr)
    assert out.stdout.strip() == "CLSA_ERR_TIMEOUT"
