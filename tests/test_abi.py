"""The C-ABI library without a GPU: it builds for sm_100a, loads, exports every function that
include/fa.h declares, sizes workspaces on the host, and rejects bad arguments with the
documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

import exact_io_aware_98_b200 as fa
from exact_io_aware_98_b200 import build as fabuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, INVALID, UNSUPPORTED, ALIGN, CUDA, TIMEOUT, WORKSPACE = 0, -1, -2, -3, -4, -5, -6
A = 0x100000  # a 16-byte-aligned fake device address; never dereferenced by these calls


@pytest.fixture(scope="module")
def lib():
    fabuild.build()
    return fa.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_get_last_error",
                     "fa_device_status"):
        assert required in names


def test_binding_constants_match_header():
    text = open(HEADER).read()
    vals = {k: int(v) for k, v in re.findall(r"\b(FA_TILE_[A-Z0-9_]+)\s*=\s*(\d+)", text)}
    assert vals == {"FA_TILE_REVERSE": fa.TILE_REVERSE, "FA_TILE_L_ROUNDED": fa.TILE_L_ROUNDED,
                    "FA_TILE_TENSOR_CORE": fa.TILE_TENSOR_CORE, "FA_TILE_O_F32": fa.TILE_O_F32}
    vals = {k: int(v) for k, v in re.findall(r"\b(FA_BWD_DKDV_[A-Z]+)\s*=\s*(\d+)", text)}
    assert vals == {"FA_BWD_DKDV_PAIR": fa.BWD_DKDV_PAIR, "FA_BWD_DKDV_SINGLE": fa.BWD_DKDV_SINGLE}


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in fa.SIGNATURES, f"binding lacks {name}"


def test_workspace_sizes_on_host(lib):
    B, H, N, d = 2, 3, 300, 64
    npad = 384
    r256 = lambda x: (x + 255) // 256 * 256
    expect = r256(B * H * npad * 4) * 2 + r256(B * H * N * d * 4)
    assert lib.fa_bwd_workspace_size(B, H, N, d) == expect
    assert lib.fa_bwd_workspace_size(0, 1, 1, 64) == 0
    assert lib.fa_naive_workspace_size(B, H, N) == B * H * N * N * 2


def _fwd(lib, q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, scale=0.125, causal=0,
         dtype=0):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, None, None, dtype, None)


def test_fwd_validation_codes(lib):
    assert _fwd(lib, q=None) == INVALID
    assert "null" in lib.fa_get_last_error().decode()
    assert _fwd(lib, N=0) == INVALID
    assert _fwd(lib, B=-1) == INVALID
    assert _fwd(lib, scale=0.0) == INVALID
    assert _fwd(lib, scale=float("nan")) == INVALID
    assert _fwd(lib, scale=-1.0) == INVALID
    assert _fwd(lib, q=A + 8) == ALIGN
    assert _fwd(lib, lse=A + 4) == ALIGN
    assert _fwd(lib, d=96) == UNSUPPORTED
    assert _fwd(lib, d=256, dtype=1) == UNSUPPORTED
    assert _fwd(lib, dtype=7) == INVALID


def test_bwd_validation_codes(lib):
    def bwd(d=64, dtype=0, ws=A, wsb=1 << 30, dq=A, wsaddr=None):
        return lib.fa_bwd(A, A, A, A, A, A, dq, A, A, 1, 2, 256, d, 0.125, 1, None, None, dtype,
                          ws if wsaddr is None else wsaddr, wsb, None)
    assert bwd(dq=None) == INVALID
    assert bwd(dq=A + 2) == ALIGN
    assert bwd(dtype=1, d=256) == UNSUPPORTED
    assert bwd(dtype=3) == INVALID
    assert bwd(d=32) == UNSUPPORTED
    assert bwd(ws=None) == WORKSPACE
    assert bwd(wsb=10) == WORKSPACE
    assert bwd(wsaddr=A + 16) == WORKSPACE
    assert "256-byte" in lib.fa_get_last_error().decode()


def test_gqa_validation_codes(lib):
    def fwd(H=4, H_kv=2):
        return lib.fa_fwd_gqa(A, A, A, A, A, 1, H, H_kv, 128, 64, 0.125, 1, None, None, 0, None)

    def bwd(H=4, H_kv=2, wsb=1 << 30):
        return lib.fa_bwd_gqa(A, A, A, A, A, A, A, A, A, 1, H, H_kv, 256, 64, 0.125, 1, None,
                              None, 0, A, wsb, None)
    for H, H_kv in ((4, 3), (4, 0), (4, 8), (6, -2)):
        assert fwd(H, H_kv) == INVALID
        assert "H_kv" in lib.fa_get_last_error().decode()
        assert bwd(H, H_kv) == INVALID
    assert bwd(wsb=10) == WORKSPACE

    def det(H=4, H_kv=2, wsb=1 << 30, dtype=0, d=64):
        return lib.fa_bwd_deterministic(A, A, A, A, A, A, A, A, A, 1, H, H_kv, 256, d, 0.125, 1,
                                        None, None, dtype, A, wsb, None)
    assert det(H_kv=3) == INVALID
    assert det(wsb=10) == WORKSPACE
    assert det(d=96) == UNSUPPORTED
    assert det(dtype=1, d=256) == UNSUPPORTED
    assert det(dtype=5) == INVALID


def test_aux_entry_validation(lib):
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 64, 0.125, 0, None, None, 48, 0,
                                     None) == INVALID
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 192, 0.125, 0, None, None, 64, 0,
                                     None) == UNSUPPORTED
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 64, 0.125, 0, None, None, 64, 16,
                                     None) == INVALID
    assert "flags" in lib.fa_get_last_error().decode()
    # the tensor-core sweep: d = 64 and bc in {64, 128} only, no reverse / rounded-l variant
    tc = fa.TILE_TENSOR_CORE
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 64, 0.125, 0, None, None, 64,
                                     tc | fa.TILE_REVERSE, None) == INVALID
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 128, 0.125, 0, None, None, 64, tc,
                                     None) == UNSUPPORTED
    assert lib.fa_fwd_tile_reference(A, A, A, A, A, 1, 1, 64, 64, 0.125, 0, None, None, 96, tc,
                                     None) == UNSUPPORTED
    assert lib.fa_naive_fwd(A, A, A, A, A, 1, 1, 64, 64, 0.125, 0, None, None, A, 16,
                            None) == WORKSPACE


def test_binding_fails_loudly_without_gpu_tensors():
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(fa.FaError):
        fa.fwd(q, q, q)


def test_binding_raises_when_library_missing(tmp_path):
    saved = fa._lib
    fa._lib = None
    try:
        with pytest.raises(fa.FaError):
            fa.load(str(tmp_path / "nope.so"))
    finally:
        fa._lib = saved


def test_measurement_diagnostics_without_a_gpu(lib):
    """The launch counter and the kernel-timing switch work on the host: no launch has been
    made in this process, so nothing is counted or recorded; a null output is rejected."""
    assert lib.fa_launch_count() == 0
    assert lib.fa_kernel_timing(1) == OK
    n, ms = ctypes.c_int(-1), ctypes.c_double(-1.0)
    assert lib.fa_kernel_timing_read(b"", ctypes.byref(n), ctypes.byref(ms)) == OK
    assert n.value == 0 and ms.value == 0.0
    assert lib.fa_kernel_timing(0) == OK
    assert lib.fa_kernel_timing_read(b"fa_", None, ctypes.byref(ms)) == INVALID


def test_deterministic_ex_rejects_unknown_options(lib):
    """Unknown option bits, or both dK/dV kernels at once, are refused before any launch."""
    for opt in (3, 4, 1 << 30):
        rc = lib.fa_bwd_deterministic_ex(A, A, A, A, A, A, A, A, A, 1, 2, 2, 256, 128, 0.088,
                                         1, None, None, 0, A, 1 << 20, opt, None)
        assert rc == INVALID
        assert "option" in lib.fa_get_last_error().decode()
