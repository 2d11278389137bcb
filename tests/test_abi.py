"""The C ABI loads and rejects bad arguments before touching the GPU.

These run without a GPU: every call below fails validation (NULL or
misaligned pointers, bad shapes, unsupported head size, non-finite scale),
which happens on the host before any CUDA call.  The pointers passed are
plain integers that are never dereferenced.
"""
import ctypes
import math
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def fa():
    from exact_attention_144_b200 import build
    build.build()
    import exact_attention_144_b200 as fa
    return fa


def test_every_declared_symbol_is_exported(fa):
    names = fa.declared_functions()
    assert set(names) >= {"fa_fwd", "fa_fwd_f16", "fa_bwd", "fa_bwd_f16", "fa_status_string",
                          "fa_get_device_status", "fa_selftest_bounded_wait", "fa_version",
                          "fa_set_kernel_events", "fa_kernel_launches", "fa_bwd_noalloc",
                          "fa_last_cuda_error"}
    lib = fa.lib()
    for n in names:
        assert hasattr(lib, n), n
    # and the dynamic symbol table holds exactly those fa_* functions
    out = subprocess.check_output(["nm", "-D", "--defined-only", fa.LIB_PATH], text=True)
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {n for n in exported if n.startswith("fa_")} == set(names)


def test_library_targets_sm100a_only(fa):
    from exact_attention_144_b200 import build
    assert "arch=compute_100a,code=sm_100a" in build.NVCC_FLAGS


def test_status_strings(fa):
    for code in range(0, -10, -1):
        s = fa.fa_status_string(code)
        assert s and s != "unknown status"
    assert fa.fa_status_string(-100) == "unknown status"
    assert fa.fa_version() >= 100


A = 0x10000          # a 16-byte aligned fake address (never dereferenced)
MIS = 0x10008        # an 8-byte aligned one


def _fwd(fa, ptrs, B=1, H=1, N=8, d=64, scale=0.125):
    return fa.lib().fa_fwd(*ptrs, B, H, N, d, ctypes.c_float(scale), None)


def _bwd(fa, ptrs, B=1, H=1, N=8, d=64, scale=0.125):
    return fa.lib().fa_bwd(*ptrs, B, H, N, d, ctypes.c_float(scale), None)


def test_forward_validation(fa):
    ok = [A] * 5
    for i in range(5):
        p = list(ok)
        p[i] = None
        assert _fwd(fa, p) == fa.FA_ERR_NULL
        p[i] = MIS
        assert _fwd(fa, p) == fa.FA_ERR_ALIGN
    assert _fwd(fa, ok, B=0) == fa.FA_ERR_SHAPE
    assert _fwd(fa, ok, H=0) == fa.FA_ERR_SHAPE
    assert _fwd(fa, ok, N=0) == fa.FA_ERR_SHAPE
    assert _fwd(fa, ok, B=1 << 10, N=1 << 16, H=1, d=64) == fa.FA_ERR_SHAPE  # 2^32 elements
    for d in (0, 32, 80, 100, 160, 512):
        assert _fwd(fa, ok, d=d) == fa.FA_ERR_HEADDIM
    assert _fwd(fa, ok, scale=math.nan) == fa.FA_ERR_SCALE
    assert _fwd(fa, ok, scale=math.inf) == fa.FA_ERR_SCALE
    assert fa.lib().fa_fwd_f16(*ok, 1, 1, 8, 80, ctypes.c_float(1.0), None) == fa.FA_ERR_HEADDIM


def test_backward_validation(fa):
    ok = [A] * 9
    for i in range(9):
        p = list(ok)
        p[i] = None
        assert _bwd(fa, p) == fa.FA_ERR_NULL
        p[i] = MIS
        assert _bwd(fa, p) == fa.FA_ERR_ALIGN
    assert _bwd(fa, ok, N=-3) == fa.FA_ERR_SHAPE
    for d in (32, 80, 160, 512):
        assert _bwd(fa, ok, d=d) == fa.FA_ERR_HEADDIM
    assert _bwd(fa, ok, scale=-math.inf) == fa.FA_ERR_SCALE


def test_status_queries_reject_null(fa):
    lib = fa.lib()
    assert lib.fa_get_device_status(None, 0) == fa.FA_ERR_NULL
    assert lib.fa_selftest_bounded_wait(1000, None) == fa.FA_ERR_NULL


def test_binding_fails_loudly_without_library(tmp_path):
    # A copy of the package without the .so must refuse to import.
    import shutil
    pkg = tmp_path / "exact_attention_144_b200"
    shutil.copytree(os.path.join(ROOT, "exact_attention_144_b200"), pkg,
                    ignore=shutil.ignore_patterns("*.so", "csrc", "__pycache__"))
    (tmp_path / "include").mkdir()
    code = "import exact_attention_144_b200 as fa; fa.lib()"
    r = subprocess.run([sys.executable, "-c", code], cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "no fallback" in (r.stderr + r.stdout)


def test_product_package_does_not_touch_the_oracle():
    pkg = os.path.join(ROOT, "exact_attention_144_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "oracle" not in text.lower(), f


def test_ex_entry_points_reject_bad_flags_and_types():
    import ctypes
    import exact_attention_144_b200 as fa
    lib = fa.lib()
    buf = (ctypes.c_char * 4096)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    args = [p] * 5 + [1, 1, 8, 64, ctypes.c_float(0.125)]
    assert lib.fa_fwd_ex(*args, 0, 2, None) == fa.FA_ERR_FLAGS
    assert lib.fa_fwd_ex(*args, 7, 0, None) == fa.FA_ERR_DTYPE
    bargs = [p] * 9 + [1, 1, 8, 64, ctypes.c_float(0.125)]
    assert lib.fa_bwd_ex(*bargs, 0, 0x80, None) == fa.FA_ERR_FLAGS
    assert lib.fa_bwd_ex(*bargs, -1, 1, None) == fa.FA_ERR_DTYPE
    assert fa.fa_status_string(fa.FA_ERR_FLAGS) == "unknown flag bits"


def test_fp8_entry_validates_before_any_cuda_call():
    import ctypes
    import exact_attention_144_b200 as fa
    lib = fa.lib()
    buf = (ctypes.c_char * 4096)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    mis = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256 + 8)
    one = ctypes.c_float(1.0)

    def call(ptrs=None, d=128, scale=0.125, dq=1.0, dk=1.0, dv=1.0, flags=0, B=1):
        ptrs = ptrs or [p] * 5
        return lib.fa_fwd_fp8(*ptrs, B, 1, 8, d, ctypes.c_float(scale), ctypes.c_float(dq),
                              ctypes.c_float(dk), ctypes.c_float(dv), flags, None)
    for i in range(5):
        ptrs = [p] * 5
        ptrs[i] = None
        assert call(ptrs) == fa.FA_ERR_NULL
        ptrs[i] = mis
        assert call(ptrs) == fa.FA_ERR_ALIGN
    for d in (64, 96, 256):  # the 8-bit path is built for d = 128 only
        assert call(d=d) == fa.FA_ERR_HEADDIM
    assert call(B=0) == fa.FA_ERR_SHAPE
    assert call(dq=math.nan) == fa.FA_ERR_SCALE
    assert call(dv=math.inf) == fa.FA_ERR_SCALE
    assert call(scale=1e30, dq=1e30) == fa.FA_ERR_SCALE  # the folded score scale overflows
    assert call(flags=2) == fa.FA_ERR_FLAGS
    del one


def test_fp8_binding_checks_types():
    import torch
    import exact_attention_144_b200 as fa
    x = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16)
    with pytest.raises((TypeError, ValueError)):
        fa.fa_fwd_fp8(x, x, x)


def test_varlen_bounds_clamp_every_input_into_range():
    # the rule the varlen kernels apply to cu_seqlens: whatever the contents,
    # each sequence lies inside [0, total) and holds at most max_seqlen tokens
    import exact_attention_144_b200 as fa
    total, ms = 1000, 300
    assert fa.fa_varlen_bounds([0, 100, 400, 1000], 0, ms, total) == (0, 100)
    assert fa.fa_varlen_bounds([0, 100, 400, 1000], 1, ms, total) == (100, 300)
    assert fa.fa_varlen_bounds([0, 100, 400, 1000], 2, ms, total) == (400, 300)  # 600 clamped to 300
    rng = __import__("numpy").random.default_rng(3)
    for _ in range(2000):
        cu = [int(x) for x in rng.integers(-2000, 3000, size=5)]
        for b in range(4):
            t0, n = fa.fa_varlen_bounds(cu, b, ms, total)
            assert 0 <= t0 <= total and 0 <= n <= ms and t0 + n <= total


def test_size_limit_is_exact():
    # every tensor must hold fewer than 2^31 elements: at 2^31 the call is
    # refused before any CUDA call; one token fewer passes validation (and
    # then, without a GPU, fails in the CUDA runtime instead)
    import ctypes
    import exact_attention_144_b200 as fa
    lib = fa.lib()
    buf = (ctypes.c_char * 4096)()
    p = ctypes.c_void_p((ctypes.addressof(buf) + 255) // 256 * 256)
    s = ctypes.c_float(0.1)
    n_max = 1 << 25  # with H = 1, d = 64: 2^31 elements
    assert lib.fa_fwd(p, p, p, p, p, 1, 1, n_max, 64, s, None) == fa.FA_ERR_SHAPE
    assert lib.fa_fwd(p, p, p, p, p, 1, 1, n_max - 1, 64, s, None) not in (
        fa.FA_ERR_SHAPE, fa.FA_OK)
    assert lib.fa_bwd(*([p] * 9), 1, 1, n_max, 64, s, None) == fa.FA_ERR_SHAPE
    assert lib.fa_bwd(*([p] * 9), 1, 1, n_max - 1, 64, s, None) not in (fa.FA_ERR_SHAPE, fa.FA_OK)
    # packed: the [B, N, 3, H, d] tensor counts three times the tokens' elements
    n3 = (1 << 31) // (3 * 64) + 1
    assert lib.fa_fwd_qkvpacked(p, p, p, 1, 1, n3, 64, s, 0, 0, None) == fa.FA_ERR_SHAPE
    assert lib.fa_fwd_qkvpacked(p, p, p, 1, 1, n3 - 1, 64, s, 0, 0, None) not in (
        fa.FA_ERR_SHAPE, fa.FA_OK)
    # 8-bit: the same element limit
    one = ctypes.c_float(1.0)
    assert lib.fa_fwd_fp8(p, p, p, p, p, 1, 1, 1 << 24, 128, s, one, one, one, 0,
                          None) == fa.FA_ERR_SHAPE
