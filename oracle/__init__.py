"""FP64 CPU oracle for exact scaled-dot-product attention (forward and backward).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import this package.  The CUDA library
never calls into it and it never calls into the CUDA library.

Two independent implementations live here:

* ``attn_oracle.c`` (loaded through ctypes): the definition written out with
  S and A materialised, OpenMP over rows.  Used at every size.
* ``brute_force.py``: pure-Python double loops, for tiny inputs only.  It is a
  second, separately written statement of the same definition used to pin the
  C oracle.

Inputs are the kernel's own bf16/fp32 values widened exactly to float64, and
the kernel's float32 scale widened exactly, so input rounding is never counted
as kernel error.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_u8p = ctypes.POINTER(ctypes.c_uint8)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
               "-fno-fast-math", "-ffp-contract=off", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        lib.oracle_attn_fwd.restype = ctypes.c_int
        lib.oracle_attn_fwd.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_double, ctypes.c_int, _u8p,
                                        ctypes.c_int, _i32p, _dp, _dp]
        lib.oracle_attn_fwd_rows.restype = ctypes.c_int
        lib.oracle_attn_fwd_rows.argtypes = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                             ctypes.c_int, _u8p, ctypes.c_int, _i32p, _i64p,
                                             ctypes.c_int, _dp, _dp]
        lib.oracle_attn_bwd.restype = ctypes.c_int
        lib.oracle_attn_bwd.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                        ctypes.c_int, _u8p, ctypes.c_int, _i32p, _i32p,
                                        ctypes.c_int, _dp, _dp, _dp]
        lib.oracle_attn_probs.restype = None
        lib.oracle_attn_probs.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                          ctypes.c_int, _u8p, ctypes.c_int, ctypes.c_int,
                                          _dp, _dp]
        lib.oracle_softmax_av.restype = None
        lib.oracle_softmax_av.argtypes = [_dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          _dp, _dp, _dp]
        lib.oracle_attn_bwd_dq_rows.restype = ctypes.c_int
        lib.oracle_attn_bwd_dq_rows.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                                ctypes.c_int, _u8p, ctypes.c_int, _i32p, _i64p,
                                                ctypes.c_int, _dp]
        lib.oracle_attn_bwd_kv_rows.restype = ctypes.c_int
        lib.oracle_attn_bwd_kv_rows.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_int, ctypes.c_int, ctypes.c_double,
                                                ctypes.c_int, _u8p, ctypes.c_int, _i32p, _i64p,
                                                ctypes.c_int, _dp, _dp]
        lib.oracle_num_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # torch tensor: widen exactly to float64
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: Optional[np.ndarray], typ):
    if a is None:
        return ctypes.cast(None, typ)
    return a.ctypes.data_as(typ)


def _masks(block_mask, kv_len):
    bm = None if block_mask is None else np.ascontiguousarray(
        block_mask.numpy() if hasattr(block_mask, "numpy") else block_mask, dtype=np.uint8)
    kl = None if kv_len is None else np.ascontiguousarray(
        kv_len.numpy() if hasattr(kv_len, "numpy") else kv_len, dtype=np.int32)
    return bm, kl


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def attn_fwd(q, k, v, scale: float, causal: bool = False, block_mask=None, kv_len=None,
             block: int = 128):
    """O [B,H,N,d] and lse [B,H,N] in float64 for every head."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    bm, kl = _masks(block_mask, kv_len)
    o = np.zeros_like(q)
    lse = np.zeros((B, H, N), np.float64)
    rc = lib.oracle_attn_fwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, N, d,
                             float(scale), int(bool(causal)), _ptr(bm, _u8p), block,
                             _ptr(kl, _i32p), _ptr(o, _dp), _ptr(lse, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd failed ({rc})")
    return o, lse


def attn_fwd_rows(q, k, v, scale: float, rows: Sequence[int], causal: bool = False,
                  block_mask=None, kv_len=None, block: int = 128):
    """O and lse of selected rows; ``rows`` are flat indices (b*H + h)*N + i."""
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    bm, kl = _masks(block_mask, kv_len)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((len(r), d), np.float64)
    lse = np.zeros(len(r), np.float64)
    rc = lib.oracle_attn_fwd_rows(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, N, d,
                                  float(scale), int(bool(causal)), _ptr(bm, _u8p), block,
                                  _ptr(kl, _i32p), _ptr(r, _i64p), len(r), _ptr(o, _dp),
                                  _ptr(lse, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_fwd_rows failed ({rc})")
    return o, lse


def attn_bwd(q, k, v, do, scale: float, causal: bool = False, block_mask=None, kv_len=None,
             block: int = 128, heads: Optional[Sequence[int]] = None):
    """dQ, dK, dV [B,H,N,d] float64.  With ``heads`` (flat b*H + h) only those are filled."""
    lib = _load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    bm, kl = _masks(block_mask, kv_len)
    hs = None if heads is None else np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    rc = lib.oracle_attn_bwd(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(do, _dp),
                             B, H, N, d, float(scale), int(bool(causal)), _ptr(bm, _u8p),
                             block, _ptr(kl, _i32p), _ptr(hs, _i32p),
                             0 if hs is None else len(hs),
                             _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd failed ({rc})")
    return dq, dk, dv


def attn_bwd_dq_rows(q, k, v, do, scale: float, rows: Sequence[int], causal: bool = False,
                     block_mask=None, kv_len=None, block: int = 128):
    """dQ of selected rows (flat (b*H + h)*N + i), float64 [len(rows), d]."""
    lib = _load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    bm, kl = _masks(block_mask, kv_len)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dq = np.zeros((len(r), d), np.float64)
    rc = lib.oracle_attn_bwd_dq_rows(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(do, _dp),
                                     B, H, N, d, float(scale), int(bool(causal)),
                                     _ptr(bm, _u8p), block, _ptr(kl, _i32p), _ptr(r, _i64p),
                                     len(r), _ptr(dq, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_dq_rows failed ({rc})")
    return dq


def attn_bwd_kv_rows(q, k, v, do, scale: float, rows: Sequence[int], causal: bool = False,
                     block_mask=None, kv_len=None, block: int = 128):
    """dK and dV of selected key rows (flat (b*H + h)*N + j), float64 [len(rows), d] each.
    Every query row that may attend to a selected key is materialised in full (its softmax
    normaliser and its sum over k are needed), so the cost is that of the full backward of
    the heads that hold a selected key, without the N x N storage."""
    lib = _load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    bm, kl = _masks(block_mask, kv_len)
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    dk = np.zeros((len(r), d), np.float64)
    dv = np.zeros((len(r), d), np.float64)
    rc = lib.oracle_attn_bwd_kv_rows(_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), _ptr(do, _dp),
                                     B, H, N, d, float(scale), int(bool(causal)),
                                     _ptr(bm, _u8p), block, _ptr(kl, _i32p), _ptr(r, _i64p),
                                     len(r), _ptr(dk, _dp), _ptr(dv, _dp))
    if rc != 0:
        raise RuntimeError(f"oracle_attn_bwd_kv_rows failed ({rc})")
    return dk, dv


def kv_group(H: int, H_kv: int) -> int:
    """Query heads per K/V head; H must be a multiple of H_kv."""
    if H_kv < 1 or H % H_kv != 0:
        raise ValueError(f"H = {H} is not a multiple of H_kv = {H_kv}")
    return H // H_kv


def attn_fwd_gqa(q, k, v, scale: float, causal: bool = False, block_mask=None, kv_len=None,
                 block: int = 128):
    """Grouped-query attention, the MQA/GQA of the tcdigital FA-2 ROI article (section
    "MQA/GQA ... との相乗効果"): q is [B,H,N,d], k and v are [B,H_kv,N,d], and query head h
    reads K/V head h // (H / H_kv) (contiguous groups; H_kv = 1 is multi-query attention).
    Written as the definition: ordinary attention with every K/V head repeated for the query
    heads of its group."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    G = kv_group(q.shape[1], k.shape[1])
    return attn_fwd(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), scale, causal,
                    block_mask, kv_len, block)


def attn_bwd_gqa(q, k, v, do, scale: float, causal: bool = False, block_mask=None,
                 kv_len=None, block: int = 128, kv_heads: Optional[Sequence[int]] = None):
    """dQ [B,H,N,d] and dK, dV [B,H_kv,N,d] of grouped-query attention.  A K/V head enters the
    output of every query head of its group, so by the chain rule through the repetition its
    gradient is the sum of the per-query-head gradients.  With ``kv_heads`` (flat b*H_kv + j)
    only those K/V heads and the query heads of their groups are filled."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    B, H, N, d = q.shape
    H_kv = k.shape[1]
    G = kv_group(H, H_kv)
    heads = None
    if kv_heads is not None:
        heads = [(j // H_kv) * H + (j % H_kv) * G + g for j in kv_heads for g in range(G)]
    dq, dk, dv = attn_bwd(q, np.repeat(k, G, axis=1), np.repeat(v, G, axis=1), do, scale,
                          causal, block_mask, kv_len, block, heads)
    return (dq, dk.reshape(B, H_kv, G, N, d).sum(axis=2),
            dv.reshape(B, H_kv, G, N, d).sum(axis=2))


def attn_probs(q, k, scale: float, causal: bool = False, block_mask=None, kv_len_b: int = -1,
               block: int = 128):
    """A (N x N) and lse (N) of one head; q, k are [N, d]."""
    lib = _load()
    q, k = _f64(q), _f64(k)
    N, d = q.shape
    bm, _ = _masks(block_mask, None)
    A = np.zeros((N, N), np.float64)
    lse = np.zeros(N, np.float64)
    lib.oracle_attn_probs(_ptr(q, _dp), _ptr(k, _dp), N, d, float(scale), int(bool(causal)),
                          _ptr(bm, _u8p), block, int(kv_len_b), _ptr(A, _dp), _ptr(lse, _dp))
    return A, lse


def softmax_av(S, v):
    """O = softmax(S) V from given logits S (rows x cols, -inf = masked); also lse and A."""
    lib = _load()
    S, v = _f64(S), _f64(v)
    rows, cols = S.shape
    dv = v.shape[1]
    o = np.zeros((rows, dv), np.float64)
    lse = np.zeros(rows, np.float64)
    A = np.zeros((rows, cols), np.float64)
    lib.oracle_softmax_av(_ptr(S, _dp), _ptr(v, _dp), rows, cols, dv, _ptr(o, _dp),
                          _ptr(lse, _dp), _ptr(A, _dp))
    return o, lse, A
