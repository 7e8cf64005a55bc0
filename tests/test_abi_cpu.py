"""The C-ABI library without a GPU: it builds, loads, exports every symbol
include/mla.h declares, and rejects bad arguments before any CUDA call."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def M():
    from head_latent_attention_10_b200 import build
    build.build()
    import head_latent_attention_10_b200 as M
    M.load_library()
    return M


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "mla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_0-9]+)\s*\(", text)))


def test_library_exports_every_declared_symbol(M):
    decl = declared_symbols()
    assert len(decl) >= 8
    lib = M.load_library()
    for name in decl:
        assert hasattr(lib, name), name
    assert set(decl) == set(M.EXPORTED)


def test_library_has_no_libcuda_or_torch_dependency():
    import subprocess
    from head_latent_attention_10_b200 import LIB_PATH
    out = subprocess.run(["ldd", LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda" not in out and "torch" not in out and "libcudart" not in out


def test_status_strings(M):
    for code in range(6):
        assert M.mla_status_string(code).startswith("MLA_")
    assert "unknown" in M.mla_status_string(99)


def _raw(M):
    return M.load_library()


def test_unsupported_shapes_are_rejected(M):
    lib = _raw(M)
    p = ctypes.c_void_p(16)
    for bad in (M.dims(8), M.dims(136), M.dims(24), M.dims(128, d_c=256), M.dims(128, block_size=32)):
        st = lib.mla_decode(ctypes.byref(bad), p, p, 1, p, 1, p, 1, 1, p, None, p, 1 << 30, 0, None)
        assert st == M.MLA_ERR_UNSUPPORTED
        assert lib.mla_decode_workspace_size(ctypes.byref(bad), 1, 1, 64) == 0


def test_argument_errors(M):
    lib = _raw(M)
    d = M.dims(128)
    p = ctypes.c_void_p(256)
    assert lib.mla_decode(None, p, p, 1, p, 1, p, 1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode(ctypes.byref(d), None, p, 1, p, 1, p, 1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode(ctypes.byref(d), p, p, 1, p, 1, p, -1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode(ctypes.byref(d), p, p, 1, p, 1, p, 1, 0, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    # misaligned
    q = ctypes.c_void_p(258)
    assert lib.mla_decode(ctypes.byref(d), q, p, 1, p, 1, p, 1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    # workspace missing or too small
    assert lib.mla_decode(ctypes.byref(d), p, p, 1, p, 1, p, 1, 1, p, None, None, 0, 0, None) == M.MLA_ERR_WORKSPACE
    assert lib.mla_decode(ctypes.byref(d), p, p, 1, p, 1, p, 1, 1, p, None, p, 16, 0, None) == M.MLA_ERR_WORKSPACE
    # empty batch is a no-op that succeeds without touching the GPU
    assert lib.mla_decode(ctypes.byref(d), None, None, 0, None, 0, None, 0, 1, None, None, None, 0, 0, None) == M.MLA_OK
    assert lib.mla_absorb_q(ctypes.byref(d), p, p, None, p, 0, p, None) == M.MLA_OK
    assert lib.mla_absorb_q(ctypes.byref(d), None, p, None, p, 4, p, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_up_v(ctypes.byref(d), p, 4, p, p, 100, p, p, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_up_v(ctypes.byref(d), p, 4, None, None, 0, p, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_cache(ctypes.byref(d), p, 4, 100, p, p, p, p, p, 1, 1, p, 1, None, 0.0, None, None) == M.MLA_ERR_UNSUPPORTED
    assert lib.mla_append_latent(ctypes.byref(d), p, p, -1, p, p, p, 1, 1, p, 1, None, 0.0, None, None) == M.MLA_ERR_INVALID_ARG
    # a misaligned norm weight, a negative eps, a YaRN ramp with beta <= alpha
    q = ctypes.c_void_p(258)
    assert lib.mla_append_latent(ctypes.byref(d), p, p, 1, p, p, p, 1, 1, p, 1, q, 1e-6, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_latent(ctypes.byref(d), p, p, 1, p, p, p, 1, 1, p, 1, p, -1.0, None, None) == M.MLA_ERR_INVALID_ARG
    bad = M.dims(128, rope_scaling=40.0, rope_yarn_alpha=32.0, rope_yarn_beta=1.0)
    assert lib.mla_append_latent(ctypes.byref(bad), p, p, 1, p, p, p, 1, 1, p, 1, None, 0.0, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode_error(None, None, 0, None) == M.MLA_ERR_INVALID_ARG


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "mla.h"

int main(void)
{
    mla_dims_t d;
    memset(&d, 0, sizeof d);
    d.num_heads = 128; d.d_c = 512; d.d_rope = 64; d.d_head = 128; d.block_size = 64;
    d.softmax_scale = 0.f; d.rope_base = 0.f;
    size_t ws = mla_decode_workspace_size(&d, 128, 1, 4096);
    /* argument errors come back before any device work */
    mla_status_t e1 = mla_decode(NULL, NULL, NULL, 0, NULL, 0, NULL, 1, 1, NULL, NULL, NULL, 0, 0u, NULL);
    mla_status_t e2 = mla_decode(&d, (const void *)256, (const void *)256, 1, (const int32_t *)256, 1,
                                 (const int32_t *)256, 1, 1, (void *)256, NULL, NULL, 0, MLA_SYNC_CHECK, NULL);
    mla_status_t e3 = mla_decode(&d, NULL, NULL, 0, NULL, 0, NULL, 0, 1, NULL, NULL, NULL, 0, 0u, NULL);
    printf("%zu %d %d %d %s\n", ws, (int)e1, (int)e2, (int)e3, mla_status_string(MLA_ERR_WORKSPACE));
    return 0;
}
"""


def test_plain_c_caller_builds_links_and_runs(M, tmp_path):
    """A C11 program (no C++, no torch) compiles against include/mla.h, links
    the library and gets its argument checks without a GPU."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(M.LIB_PATH)
    libname = os.path.basename(M.LIB_PATH)
    subprocess.run([gcc, "-std=c11", "-Wall", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    str(src), "-o", str(exe), os.path.join(libdir, libname), f"-Wl,-rpath,{libdir}"],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    lib = _raw(M)
    d = M.dims(128)
    assert int(out[0]) == lib.mla_decode_workspace_size(ctypes.byref(d), 128, 1, 4096) > 0
    assert [int(x) for x in out[1:4]] == [M.MLA_ERR_INVALID_ARG, M.MLA_ERR_WORKSPACE, M.MLA_OK]
    assert len(out[4]) > 0


def test_workspace_size_grows_with_batch(M):
    lib = _raw(M)
    d = M.dims(128)
    a = lib.mla_decode_workspace_size(ctypes.byref(d), 1, 1, 4096)
    b = lib.mla_decode_workspace_size(ctypes.byref(d), 128, 1, 4096)
    c = lib.mla_decode_workspace_size(ctypes.byref(d), 128, 2, 4096)
    assert 0 < a < b <= c and a % 256 == 0


def test_missing_library_fails_loudly(tmp_path):
    import head_latent_attention_10_b200 as M
    saved = M._LIB
    M._LIB = None
    try:
        with pytest.raises(RuntimeError):
            M.load_library(str(tmp_path / "nope.so"))
    finally:
        M._LIB = saved


def test_product_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "head_latent_attention_10_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "mla_oracle" not in text, f


def test_every_entry_point_has_a_full_ctypes_signature(M):
    """A missing argtypes list makes ctypes pass 64-bit pointers as C ints."""
    import re
    lib = M.load_library()
    header = open(os.path.join(ROOT, "include", "mla.h")).read()
    for name in M.EXPORTED:
        f = getattr(lib, name)
        assert f.argtypes is not None, name
        decl = re.search(r"\b" + name + r"\(([^)]*)\)", header).group(1).strip()
        nargs = 0 if decl in ("", "void") else decl.count(",") + 1
        assert len(f.argtypes) == nargs, (name, len(f.argtypes), nargs)


def test_decode_rejects_an_empty_cache_for_a_non_empty_batch(M):
    """B > 0 with no cache block (or no block-table column) is an argument
    error, reported before any device work."""
    lib = _raw(M)
    d = M.dims(128)
    p = ctypes.c_void_p(256)
    n0 = lib.mla_kernel_launches()
    assert lib.mla_decode(ctypes.byref(d), p, p, 0, p, 1, p, 1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_decode(ctypes.byref(d), p, p, 1, p, 0, p, 1, 1, p, None, p, 1 << 30, 0, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_kernel_launches() == n0


@pytest.mark.parametrize("H,s", [(128, 200), (128, 96), (16, 900)])
def test_noalloc_rejects_tensor_core_shapes_beyond_its_scratch(M, H, s):
    """The tensor-core decode keeps two fp32 partial slots of s*H latent rows
    per range; once s*H outgrows the fixed scratch the call must fail with
    MLA_ERR_WORKSPACE before touching the device (no launch, no CUDA call:
    this runs without a GPU)."""
    lib = _raw(M)
    d = M.dims(H)
    p = ctypes.c_void_p(256)
    n0 = lib.mla_kernel_launches()
    st = lib.mla_decode_noalloc(ctypes.byref(d), p, p, 1, p, 1, p, 1, s, p, None, 0, None)
    assert st == M.MLA_ERR_WORKSPACE
    assert lib.mla_kernel_launches() == n0
    # the size the call refused is indeed beyond the scratch
    assert lib.mla_decode_workspace_size(ctypes.byref(d), 1, s, 64) > M.MLA_NOALLOC_SCRATCH_BYTES


def test_prefill_argument_errors_and_workspace(M):
    """mla_prefill rejects bad arguments before any device work, and its
    workspace grows with the sequences it expands."""
    lib = _raw(M)
    d = M.dims(128)
    p = ctypes.c_void_p(256)
    big = 1 << 40
    n0 = lib.mla_kernel_launches()
    call = lambda dd, qn=p, B=1, s=4, msl=64, ws=p, wsb=big, nb=1, mb=1: lib.mla_prefill(
        dd, qn, p, None, p, p, p, nb, p, mb, p, B, s, msl, p, None, ws, wsb, 0, None)
    assert call(None) == M.MLA_ERR_INVALID_ARG
    assert call(ctypes.byref(d), qn=None) == M.MLA_ERR_INVALID_ARG
    assert call(ctypes.byref(d), qn=ctypes.c_void_p(258)) == M.MLA_ERR_INVALID_ARG   # misaligned
    assert call(ctypes.byref(d), s=0) == M.MLA_ERR_INVALID_ARG
    assert call(ctypes.byref(d), s=65, msl=64) == M.MLA_ERR_INVALID_ARG             # max_seq_len < s
    assert call(ctypes.byref(d), nb=0) == M.MLA_ERR_INVALID_ARG
    assert call(ctypes.byref(d), mb=0) == M.MLA_ERR_INVALID_ARG
    assert call(ctypes.byref(d), ws=None) == M.MLA_ERR_WORKSPACE
    assert call(ctypes.byref(d), wsb=4096) == M.MLA_ERR_WORKSPACE
    assert call(ctypes.byref(M.dims(24))) == M.MLA_ERR_UNSUPPORTED
    assert lib.mla_prefill(ctypes.byref(d), None, None, None, None, None, None, 0, None, 0, None, 0, 1, 1,
                           None, None, None, 0, 0, None) == M.MLA_OK               # B = 0
    assert lib.mla_kernel_launches() == n0
    a = lib.mla_prefill_workspace_size(ctypes.byref(d), 1, 128, 1000)
    b = lib.mla_prefill_workspace_size(ctypes.byref(d), 1, 128, 1024)   # same 128-row padding
    c = lib.mla_prefill_workspace_size(ctypes.byref(d), 2, 128, 1000)
    assert 0 < a == b < c and a % 256 == 0
    # K^C and V^C dominate: 2 x rows x H x 128 bf16
    assert a >= 2 * 1024 * 128 * 128 * 2
    assert lib.mla_prefill_workspace_size(ctypes.byref(d), 1, 129, 128) == 0


def test_fp8_argument_errors(M):
    """The FP8 writer and decode reject bad arguments before any device work."""
    lib = _raw(M)
    d = M.dims(128)
    p = ctypes.c_void_p(256)
    n0 = lib.mla_kernel_launches()
    # writer: negative T, misaligned codes or scales, bad norm arguments; T = 0 is a no-op
    assert lib.mla_append_latent_fp8(ctypes.byref(d), p, p, -1, p, p, p, 1, 1, p, p, 1, None, 0.0, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_latent_fp8(ctypes.byref(d), p, p, 1, p, p, p, 1, 1, ctypes.c_void_p(264), p, 1, None, 0.0, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_latent_fp8(ctypes.byref(d), p, p, 1, p, p, p, 1, 1, p, ctypes.c_void_p(260), 1, None, 0.0, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_latent_fp8(ctypes.byref(d), p, p, 1, p, p, p, 1, 1, p, p, 1, p, -1.0, None, None) == M.MLA_ERR_INVALID_ARG
    assert lib.mla_append_latent_fp8(ctypes.byref(d), p, p, 0, p, p, p, 1, 1, p, p, 1, None, 0.0, None, None) == M.MLA_OK
    # decode: the CUDA-core path does not read FP8; bad sizes; misaligned scales; workspace
    big = 1 << 40
    dec = lambda flags=0, B=1, s=1, nb=1, mb=1, sc=p, ws=p, wsb=big: lib.mla_decode_fp8(
        ctypes.byref(d), p, p, sc, nb, p, mb, p, B, s, p, None, ws, wsb, flags, None)
    assert dec(flags=M.MLA_FORCE_SIMPLE) == M.MLA_ERR_UNSUPPORTED
    assert dec(s=0) == M.MLA_ERR_INVALID_ARG
    assert dec(nb=0) == M.MLA_ERR_INVALID_ARG
    assert dec(sc=ctypes.c_void_p(264)) == M.MLA_ERR_INVALID_ARG
    assert dec(ws=None) == M.MLA_ERR_WORKSPACE
    assert dec(wsb=16) == M.MLA_ERR_WORKSPACE
    assert dec(B=0) == M.MLA_OK
    assert lib.mla_kernel_launches() == n0
