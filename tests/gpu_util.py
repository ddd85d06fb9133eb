"""Helpers shared by the GPU parity tests: move seeded inputs to the GPU, run the CUDA path
through the C ABI, run the oracle on the same values, compare with the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

import oracle

# Tolerances (stated for unit-normal bf16 inputs): absolute on O, relative to max|ref| on
# gradients; lse (natural log) absolute.
BF16_O_MAX, BF16_O_MEAN = 2e-2, 2e-3
BF16_LSE_MAX = 1e-3
F32_TOL = 1e-5
GRAD_MAX, GRAD_MEAN = 2e-2, 2e-3


def to_gpu(x: dict) -> dict:
    g = dict(x)
    for key in ("q", "k", "v", "do", "kv_len", "block_mask"):
        if x.get(key) is not None:
            g[key] = x[key].cuda().contiguous()
    return g


def compare_o(o_gpu: np.ndarray, o_ref: np.ndarray, dtype: str = "bf16"):
    err = np.abs(o_gpu.astype(np.float64) - o_ref)
    if dtype == "f32":
        assert err.max() <= F32_TOL, f"fp32 O max err {err.max():.3e}"
    else:
        assert err.max() <= BF16_O_MAX, f"O max err {err.max():.3e}"
        assert err.mean() <= BF16_O_MEAN, f"O mean err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def compare_lse(l_gpu: np.ndarray, l_ref: np.ndarray, tol: float = BF16_LSE_MAX):
    l_gpu = l_gpu.astype(np.float64)
    fin = np.isfinite(l_ref)
    assert np.array_equal(fin, np.isfinite(l_gpu)), "masked-row pattern of lse differs"
    assert np.all(l_gpu[~fin] == -np.inf)
    if fin.any():
        err = np.abs(l_gpu[fin] - l_ref[fin]).max()
        assert err <= tol, f"lse max err {err:.3e}"
        return float(err)
    return 0.0


def compare_grad(g_gpu: np.ndarray, g_ref: np.ndarray, name: str, floor: float = 0.0):
    """Max and mean error relative to max |reference|.  Where the reference gradient vanishes
    identically (a single visible key makes dS = P (dP - Dvec) exactly 0 in exact arithmetic,
    while the kernel's dP and Dvec, summed in different orders, leave rounding of the size of
    dP), "relative to max |reference|" is undefined; such a reference is measured against
    ``floor``, the largest reference gradient of the same call, as the fp32 backward test does."""
    ref_max = float(np.abs(g_ref).max())
    scale = max(ref_max if ref_max > 0.0 else floor, 1e-30)
    err = np.abs(g_gpu.astype(np.float64) - g_ref) / scale
    assert err.max() <= GRAD_MAX, f"{name} max rel err {err.max():.3e}"
    assert err.mean() <= GRAD_MEAN, f"{name} mean rel err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def oracle_fwd(x: dict):
    return oracle.attn_fwd(x["q"], x["k"], x["v"], x["scale"], x["causal"], x["block_mask"],
                           x["kv_len"])


def oracle_bwd(x: dict, heads=None):
    return oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], x["causal"],
                           x["block_mask"], x["kv_len"], heads=heads)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()
