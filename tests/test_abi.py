"""The C-ABI library: builds, loads, exports every symbol include/fa.h declares, and rejects
bad arguments before touching the GPU. CPU only: no compute call reaches a kernel here."""

from __future__ import annotations

import ctypes
import os
import re

import pytest

from exact_io_aware_66_b200 import build as fa_build
from exact_io_aware_66_b200 import fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fa_build.build()
    return fa.lib()


def _header_functions():
    src = open(os.path.join(ROOT, "include", "fa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(lib):
    names = _header_functions()
    assert "fa_fwd" in names and "fa_bwd" in names
    for name in names:
        assert hasattr(lib, name), f"{name} declared in include/fa.h but not exported"
    assert set(names) <= set(fa.SIGNATURES), "binding lacks a signature for a header function"


def test_exports_via_nm():
    fa_build.build()
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", fa.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (fa_[a-z0-9_]+)", out))
    assert set(_header_functions()) <= exported


def test_version(lib):
    assert "sm_100a" in fa.fa_version()


def test_workspace_size(lib):
    rows = 2 * 3 * 100
    ws = fa.fa_bwd_workspace_size(2, 3, 100, 64)
    assert ws >= rows * 64 * 4 + rows * 4
    assert ws % 16 == 0
    assert fa.fa_bwd_workspace_size(2, 3, 100, 80) == 0
    assert fa.fa_bwd_workspace_size(2, 3, 100, 96) >= rows * 96 * 4 + rows * 4
    assert fa.fa_bwd_workspace_size(0, 3, 100, 64) == 0


def _fwd_raw(lib, q=16, k=32, v=48, o=1 << 20, lse=2 << 20, B=1, H=1, N=128, d=64, scale=0.125,
             causal=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, None)


def test_fwd_validation_without_gpu(lib):
    # every one of these is rejected by the argument checks, before any CUDA call
    assert _fwd_raw(lib, d=80) == 2
    assert "head dim" in fa.fa_last_error_string()
    assert _fwd_raw(lib, N=0) == 1
    assert _fwd_raw(lib, B=-1) == 1
    assert _fwd_raw(lib, scale=0.0) == 1
    assert _fwd_raw(lib, scale=float("nan")) == 1
    assert _fwd_raw(lib, q=0) == 1
    assert _fwd_raw(lib, q=8) == 3  # not 16-byte aligned
    assert _fwd_raw(lib, B=1 << 16, H=1 << 8, N=1 << 8) == 2  # B*H*N >= 2^31
    # output aliasing an input
    assert _fwd_raw(lib, o=32) == 1


def test_bwd_validation_without_gpu(lib):
    base = dict(q=1 << 20, k=2 << 20, v=3 << 20, o=4 << 20, do=5 << 20, lse=6 << 20,
                dq=7 << 20, dk=8 << 20, dv=9 << 20, ws=10 << 20)

    def call(ws_bytes=1 << 20, d=64, N=128, **kw):
        a = dict(base, **kw)
        return lib.fa_bwd(a["q"], a["k"], a["v"], a["o"], a["do"], a["lse"], a["dq"], a["dk"],
                          a["dv"], a["ws"], ws_bytes, 1, 1, N, d, 0.125, 0, None)

    assert call(d=80) == 2
    assert call(ws=0) == 6
    assert call(ws_bytes=16) == 6
    assert call(dq=0) == 1
    assert call(dk=(8 << 20) + 4) == 3
    assert call(dv=1 << 20) == 1  # dv aliases q


def test_check_status_without_gpu(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("GPU present")
    assert lib.fa_check_status(None) == 4  # FA_ERR_CUDA: no device
    with pytest.raises(fa.FaError):
        fa.fa_check_status(0)


def test_no_cpu_fallback_in_product_package():
    """The product package never imports the oracle (no CPU fallback path exists)."""
    pkg = os.path.join(ROOT, "exact_io_aware_66_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            src = open(os.path.join(pkg, fn)).read()
            assert not re.search(r"^\s*(from|import)\s+oracle", src, flags=re.M), fn


def test_selftest_timeout_rejects_bad_limit_without_gpu(lib):
    assert lib.fa_selftest_timeout(0, None) == 1
    assert lib.fa_selftest_timeout(10 ** 8, None) == 1


def _fwd_ex_raw(lib, B=1, H=2, H_kv=1, N_q=100, N_kv=300, d=64, scale=0.125, mask=2, o=1 << 20,
                lse=2 << 20):
    s = fa.FaAttnShape(B, H, H_kv, N_q, N_kv, d, scale, mask)
    return lib.fa_fwd_ex(16, 1 << 16, 2 << 16, o, lse, ctypes.byref(s), None, None)


def test_fwd_ex_validation_without_gpu(lib):
    assert lib.fa_fwd_ex(16, 32, 48, 1 << 20, 2 << 20, None, None, None) == 1  # null shape
    assert _fwd_ex_raw(lib, H=3, H_kv=2) == 1  # H not a multiple of H_kv
    assert "multiple" in fa.fa_last_error_string()
    assert _fwd_ex_raw(lib, mask=3) == 1
    assert _fwd_ex_raw(lib, N_kv=0) == 1
    assert _fwd_ex_raw(lib, d=80) == 2
    # o (B*H*N_q*d*2 = 25600 bytes from 1<<16 - 25600 + 16) would overlap k at 1<<16
    assert _fwd_ex_raw(lib, o=(1 << 16) - 1024) == 1
    # k and v are B*H_kv*N_kv*d*2 = 38400 bytes: an lse placed inside v overlaps it
    assert _fwd_ex_raw(lib, lse=(2 << 16) + 1024) == 1


def test_bwd_ex_workspace_size(lib):
    s = fa.FaAttnShape(2, 4, 2, 100, 300, 64, 0.125, 1)
    ws = lib.fa_bwd_ex_workspace_size(ctypes.byref(s))
    # the workspace scales with the query rows B*H*N_q, not with the keys
    assert ws == fa.fa_bwd_workspace_size(2, 4, 100, 64)
    assert fa.fa_bwd_ex_workspace_size(2, 4, 2, 100, 300, 64, True) == ws
    assert fa.fa_bwd_ex_workspace_size(2, 4, 3, 100, 300, 64, True) == 0
    assert lib.fa_bwd_ex_workspace_size(None) == 0


def test_mask_code():
    assert fa.mask_code(False) == 0 and fa.mask_code("none") == 0
    assert fa.mask_code(True) == 1 and fa.mask_code("top_left") == 1
    assert fa.mask_code("bottom_right") == 2
    with pytest.raises(ValueError):
        fa.mask_code("diagonal")


def test_dropout_validation_without_gpu(lib):
    s = fa.FaAttnShape(1, 2, 1, 100, 300, 64, 0.125, 2)
    for p in (1.0, -0.1, float("nan")):
        d = fa.FaDropout(p, 1, 0)
        assert lib.fa_fwd_ex(16, 1 << 16, 2 << 16, 1 << 20, 2 << 20, ctypes.byref(s),
                             ctypes.byref(d), None) == 1
        assert "dropout" in fa.fa_last_error_string()


def test_sources_hash_covers_every_library_source():
    """bench.py's roofline traffic is trusted only while the ncu captures match the sources hash,
    so the hash must cover every file the library is compiled from."""
    import bench

    csrc = os.path.join(ROOT, "exact_io_aware_66_b200", "csrc")
    compiled = {f"exact_io_aware_66_b200/csrc/{fn}" for fn in os.listdir(csrc)
                if fn.endswith((".cu", ".cuh"))}
    assert compiled <= set(bench.KERNEL_SOURCES), sorted(compiled - set(bench.KERNEL_SOURCES))


def test_debug_stall_hook_validation_without_gpu(lib):
    assert lib.fa_debug_stall_next(1, 0, 1000) == 1  # only the forward (0) and backward main (2)
    assert lib.fa_debug_stall_next(0, -1, 1000) == 1
    assert lib.fa_debug_stall_next(2, 0, 0) == 1
    assert lib.fa_debug_stall_next(2, 0, 10 ** 8) == 1
    assert lib.fa_debug_stall_next(0, 3, 20000) == 0
    assert lib.fa_debug_stall_next(-1, 0, 0) == 0  # disarm


def test_noalloc_d256_over_builtin_scratch_rejected_without_gpu(lib):
    """At d = 256 the scratch fa_bwd_noalloc needs is sized like fa_bwd's workspace for d = 256
    (fp32 dQ accumulator of 256 columns): sizes beyond the built-in 64 MiB are refused before any
    CUDA call."""
    B, H, N = 4, 16, 4096
    assert fa.fa_bwd_workspace_size(B, H, N, 256) >= B * H * N * 256 * 4 > 64 << 20
    fake = 1 << 24
    st = lib.fa_bwd_noalloc(fake, fake * 2, fake * 3, fake * 4, fake * 5, fake * 6, fake * 7,
                            fake * 8, fake * 9, B, H, N, 256, 0.0625, 1, None)
    assert st == 2
    assert "built into the library" in fa.fa_last_error_string()


def test_d256_backward_workspace_without_gpu(lib):
    s = fa.FaAttnShape(2, 4, 2, 100, 300, 256, 0.0625, 1)
    ws = lib.fa_bwd_ex_workspace_size(ctypes.byref(s))
    assert ws == fa.fa_bwd_workspace_size(2, 4, 100, 256) > 2 * 4 * 100 * 256 * 4
