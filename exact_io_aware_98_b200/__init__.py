"""Python binding of libfa (exact IO-aware attention on B200, sm_100a).

Argument marshalling only: every step of the attention computation runs in the
CUDA kernels behind the C ABI declared in ``include/fa.h``.  PyTorch supplies
device memory and the current stream.  There is no CPU fallback: if the
library is missing or no GPU is present, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfa.so")

FA_BF16, FA_F32 = 0, 1
BWD_DKDV_PAIR, BWD_DKDV_SINGLE = 1, 2   # fa.h FA_BWD_DKDV_*
_STATUS = {0: "FA_OK", -1: "FA_ERR_INVALID", -2: "FA_ERR_UNSUPPORTED", -3: "FA_ERR_ALIGN",
           -4: "FA_ERR_CUDA", -5: "FA_ERR_TIMEOUT", -6: "FA_ERR_WORKSPACE"}

# exported symbol -> (restype, argtypes)
_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "fa_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _i, _vp]),
    "fa_fwd_gqa": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _i, _vp]),
    "fa_bwd_workspace_size": (_sz, [_i, _i, _i, _i]),
    "fa_bwd_gqa": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f, _i,
                        _vp, _vp, _i, _vp, _sz, _vp]),
    "fa_bwd_deterministic": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                  _f, _i, _vp, _vp, _i, _vp, _sz, _vp]),
    "fa_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp,
                    _vp, _i, _vp, _sz, _vp]),
    "fa_bwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i,
                            _vp, _vp, _i, _vp]),
    "fa_bwd_deterministic_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i,
                                     _i, _f, _i, _vp, _vp, _i, _vp, _sz, _i, _vp]),
    "fa_fwd_tile_reference": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp,
                                   _i, _i, _vp]),
    "fa_naive_workspace_size": (_sz, [_i, _i, _i]),
    "fa_naive_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp, _sz,
                          _vp]),
    "fa_diag_exp2": (_i, [_vp, _vp, _vp, _vp, _i, _vp]),
    "fa_diag_wait_timeout": (_i, [_i, _vp]),
    "fa_launch_count": (ctypes.c_ulonglong, []),
    "fa_kernel_timing": (_i, [_i]),
    "fa_kernel_timing_read": (_i, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_int),
                                   ctypes.POINTER(ctypes.c_double)]),
    "fa_get_last_error": (ctypes.c_char_p, []),
    "fa_device_status": (_i, [ctypes.POINTER(ctypes.c_uint)]),
}

_lib = None


class FaError(RuntimeError):
    pass


def load(path: str = LIB_PATH):
    """Load libfa.so (built by ``exact_io_aware_98_b200.build``); raises if absent."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise FaError(f"libfa.so not found at {path}: build it first "
                          "(python -m exact_io_aware_98_b200.build)")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = load().fa_get_last_error().decode(errors="replace")
        raise FaError(f"{what}: {_STATUS.get(rc, rc)}: {msg}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _require(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise FaError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise FaError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise FaError(f"{name} must be {dtype}, got {t.dtype}")


def _masks(block_mask, kv_len):
    if block_mask is not None:
        _require(block_mask, "block_mask", torch.uint8)
    if kv_len is not None:
        _require(kv_len, "kv_len", torch.int32)
    return _ptr(block_mask), _ptr(kv_len)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float32:
        return FA_F32
    raise FaError(f"unsupported dtype {t.dtype}")


def default_scale(d: int) -> float:
    return float(torch.tensor(1.0 / math.sqrt(d), dtype=torch.float32).item())


def _kv_heads(q, k, v) -> int:
    """K/V head count; k and v are [B, H_kv, N, d] with H a multiple of H_kv."""
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    for t, n in ((k, "k"), (v, "v")):
        if t.dim() != 4 or (t.shape[0], t.shape[2], t.shape[3]) != (B, N, d) or t.shape[1] != H_kv:
            raise FaError(f"{n} shape {tuple(t.shape)} does not match q {tuple(q.shape)}")
    if H_kv < 1 or H % H_kv != 0:
        raise FaError(f"H = {H} is not a multiple of H_kv = {H_kv}")
    return H_kv


def fwd(q, k, v, scale: Optional[float] = None, causal: bool = False, block_mask=None,
        kv_len=None, out=None, lse=None):
    """O, lse = fa_fwd(q, k, v); q [B, H, N, d], k and v [B, H_kv, N, d] (bf16 or fp32) on the
    GPU.  H_kv < H is grouped-query attention (fa_fwd_gqa): query head h reads K/V head
    h // (H / H_kv)."""
    lib = load()
    B, H, N, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, q.dtype)
    H_kv = _kv_heads(q, k, v)
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device) if lse is None else lse
    _require(o, "out", q.dtype)
    _require(l, "lse", torch.float32)
    bm, kl = _masks(block_mask, kv_len)
    s = default_scale(d) if scale is None else float(scale)
    if H_kv == H:
        rc = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, N, d, s, int(causal),
                        bm, kl, _dtype_code(q), _stream())
        _check(rc, "fa_fwd")
    else:
        rc = lib.fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, H_kv, N, d, s,
                            int(causal), bm, kl, _dtype_code(q), _stream())
        _check(rc, "fa_fwd_gqa")
    return o, l


def bwd_workspace_size(B: int, H: int, N: int, d: int) -> int:
    return int(load().fa_bwd_workspace_size(B, H, N, d))


def _bwd_operands(q, k, v, o, lse, do, dq, dk, dv):
    """Checks shared by every backward call: dtypes, contiguity, and the shapes of o, do, lse
    and of caller-supplied gradients against q, k and v (so that no kernel is ever handed a
    buffer smaller than the tensor maps it builds from q's sizes).  Returns H_kv and dq, dk, dv
    (allocated here when not supplied)."""
    B, H, N, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (do, "do")):
        _require(t, n, q.dtype)
    H_kv = _kv_heads(q, k, v)
    for t, n in ((o, "o"), (do, "do")):
        if t.shape != q.shape:
            raise FaError(f"{n} shape {tuple(t.shape)} does not match q {tuple(q.shape)}")
    _require(lse, "lse", torch.float32)
    if tuple(lse.shape) != (B, H, N):
        raise FaError(f"lse shape {tuple(lse.shape)} must be {(B, H, N)}")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    for t, n in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        _require(t, n, q.dtype)
    if dq.shape != q.shape or dk.shape != k.shape or dv.shape != v.shape:
        raise FaError("gradient shapes must match q, k and v")
    return H_kv, dq, dk, dv


def bwd(q, k, v, o, lse, do, scale: Optional[float] = None, causal: bool = False,
        block_mask=None, kv_len=None, workspace=None, dq=None, dk=None, dv=None,
        deterministic: bool = False, dkdv_pair: Optional[bool] = None):
    """dQ, dK, dV = fa_bwd(...); tensors on the GPU, q/o/do [B, H, N, d], k/v and dK/dV
    [B, H_kv, N, d] (fa_bwd_gqa when H_kv < H).  ``deterministic`` calls fa_bwd_deterministic:
    bit-reproducible gradients, dQ without atomics; with it, ``dkdv_pair`` True / False picks
    the 2-CTA or the single-CTA dK/dV kernel at d = 128 (fa_bwd_deterministic_ex), None the
    library's default."""
    lib = load()
    B, H, N, d = q.shape
    H_kv, dq, dk, dv = _bwd_operands(q, k, v, o, lse, do, dq, dk, dv)
    need = bwd_workspace_size(B, H, N, d)
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    _require(ws, "workspace", torch.uint8)
    bm, kl = _masks(block_mask, kv_len)
    s = default_scale(d) if scale is None else float(scale)
    if deterministic and dkdv_pair is not None:
        opt = BWD_DKDV_PAIR if dkdv_pair else BWD_DKDV_SINGLE
        rc = lib.fa_bwd_deterministic_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                                         _ptr(dq), _ptr(dk), _ptr(dv), B, H, H_kv, N, d, s,
                                         int(causal), bm, kl, _dtype_code(q), _ptr(ws),
                                         ws.numel(), opt, _stream())
        _check(rc, "fa_bwd_deterministic_ex")
    elif deterministic:
        rc = lib.fa_bwd_deterministic(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do),
                                      _ptr(dq), _ptr(dk), _ptr(dv), B, H, H_kv, N, d, s,
                                      int(causal), bm, kl, _dtype_code(q), _ptr(ws), ws.numel(),
                                      _stream())
        _check(rc, "fa_bwd_deterministic")
    elif H_kv == H:
        rc = lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                        _ptr(dk), _ptr(dv), B, H, N, d, s, int(causal), bm, kl, _dtype_code(q),
                        _ptr(ws), ws.numel(), _stream())
        _check(rc, "fa_bwd")
    else:
        rc = lib.fa_bwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, H, H_kv, N, d, s, int(causal), bm, kl,
                            _dtype_code(q), _ptr(ws), ws.numel(), _stream())
        _check(rc, "fa_bwd_gqa")
    return dq, dk, dv


def bwd_noalloc(q, k, v, o, lse, do, scale: Optional[float] = None, causal: bool = False,
                block_mask=None, kv_len=None, dq=None, dk=None, dv=None):
    """fa_bwd without a workspace, for callers that cannot allocate device memory: the
    library's own fixed 32 MiB scratch is used instead, and calls on one device must not
    overlap.  Ordinary attention only (k and v have q's H heads).  dq, dk and dv may be passed
    in; otherwise this wrapper allocates them with torch, which a caller that cannot allocate
    avoids by passing its own."""
    lib = load()
    B, H, N, d = q.shape
    H_kv, dq, dk, dv = _bwd_operands(q, k, v, o, lse, do, dq, dk, dv)
    if H_kv != H:
        raise FaError(f"fa_bwd_noalloc takes ordinary attention only (k/v have {H_kv} heads, "
                      f"q has {H})")
    bm, kl = _masks(block_mask, kv_len)
    s = default_scale(d) if scale is None else float(scale)
    rc = lib.fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq),
                            _ptr(dk), _ptr(dv), B, H, N, d, s, int(causal), bm, kl,
                            _dtype_code(q), _stream())
    _check(rc, "fa_bwd_noalloc")
    return dq, dk, dv


TILE_REVERSE = 1          # fa.h FA_TILE_REVERSE: key tiles visited last to first
TILE_L_ROUNDED = 2        # fa.h FA_TILE_L_ROUNDED: l sums the bf16-rounded P
TILE_TENSOR_CORE = 4      # fa.h FA_TILE_TENSOR_CORE: the tcgen05 forward with bc-key tiles
TILE_O_F32 = 8            # fa.h FA_TILE_O_F32: fp32 O/l before its bf16 rounding


def fwd_tile_reference(q, k, v, bc: int, scale: Optional[float] = None, causal: bool = False,
                       block_mask=None, kv_len=None, reverse: bool = False,
                       l_rounded: bool = False, tensor_core: bool = False, o_f32: bool = False):
    """bf16 forward that rescales after every `bc` keys (deviation study): the CUDA-core
    reference (`reverse` visits the key tiles last to first, `l_rounded` sums l over the
    bf16-rounded P) or, with `tensor_core`, the tcgen05 forward with bc-key tiles (d = 64,
    bc 64 or 128).  `o_f32` returns the fp32 O/l before its bf16 rounding."""
    lib = load()
    B, H, N, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, torch.bfloat16)
    o = torch.empty(q.shape, dtype=torch.float32 if o_f32 else torch.bfloat16, device=q.device)
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    bm, kl = _masks(block_mask, kv_len)
    s = default_scale(d) if scale is None else float(scale)
    flags = ((TILE_REVERSE if reverse else 0) | (TILE_L_ROUNDED if l_rounded else 0) |
             (TILE_TENSOR_CORE if tensor_core else 0) | (TILE_O_F32 if o_f32 else 0))
    rc = lib.fa_fwd_tile_reference(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, N, d, s,
                                   int(causal), bm, kl, int(bc), flags, _stream())
    _check(rc, "fa_fwd_tile_reference")
    return o, l


def naive_fwd(q, k, v, scale: Optional[float] = None, causal: bool = False, block_mask=None,
              kv_len=None, workspace=None):
    """Materialised baseline: S and P go through HBM in bf16."""
    lib = load()
    B, H, N, d = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n, torch.bfloat16)
    need = int(lib.fa_naive_workspace_size(B, H, N))
    ws = torch.empty(need, dtype=torch.uint8, device=q.device) if workspace is None else workspace
    o = torch.empty_like(q)
    l = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    bm, kl = _masks(block_mask, kv_len)
    s = default_scale(d) if scale is None else float(scale)
    rc = lib.fa_naive_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(l), B, H, N, d, s,
                          int(causal), bm, kl, _ptr(ws), ws.numel(), _stream())
    _check(rc, "fa_naive_fwd")
    return o, l


def diag_exp2(x):
    """(FMA-pipe 2^x, ex2.approx, exp2f) of a float32 CUDA tensor; diagnostic only."""
    lib = load()
    _require(x, "x", torch.float32)
    y = [torch.empty_like(x) for _ in range(3)]
    rc = lib.fa_diag_exp2(_ptr(x), _ptr(y[0]), _ptr(y[1]), _ptr(y[2]), x.numel(), _stream())
    _check(rc, "fa_diag_exp2")
    return tuple(y)


def diag_wait_timeout(site: int):
    """Launch the bounded-wait diagnostic (gives up after ~2 s); read it with device_status()."""
    _check(load().fa_diag_wait_timeout(int(site), _stream()), "fa_diag_wait_timeout")


def device_status() -> int:
    """Synchronise; return the bounded-wait status code (0 = no wait gave up) and clear it."""
    code = ctypes.c_uint(0)
    rc = load().fa_device_status(ctypes.byref(code))
    if rc not in (0, -5):
        _check(rc, "fa_device_status")
    return int(code.value)


def launch_count() -> int:
    """Kernels this library has launched in the process (fa_launch_count)."""
    return int(load().fa_launch_count())


def kernel_timing(enable: bool):
    """Start (True) or stop (False) bracketing each tensor-core launch with CUDA events."""
    _check(load().fa_kernel_timing(int(bool(enable))), "fa_kernel_timing")


def kernel_timing_read(name: str = ""):
    """(launches, total ms) of the recorded launches of kernels whose name contains ``name``;
    waits for them and forgets them."""
    n = ctypes.c_int(0)
    ms = ctypes.c_double(0.0)
    _check(load().fa_kernel_timing_read(name.encode(), ctypes.byref(n), ctypes.byref(ms)),
           "fa_kernel_timing_read")
    return int(n.value), float(ms.value)
