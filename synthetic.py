"""Seeded synthetic inputs for the attention workloads.

This module only draws numbers and builds masks; it holds none of the
attention arithmetic.  It is the one module shared by the CPU oracle side
(tests, the CPU baseline) and the CUDA side (tests, bench), so both always
see bit-identical inputs.

Recipe (one independent generator per tensor):
  * values: ``numpy.random.default_rng(seed + tensor_id).standard_normal``
    in float64, times the workload's amplitude, rounded once to float32 and
    then (bf16 workloads) to bfloat16 with round-to-nearest-even.
    tensor ids: q=0, k=1, v=2, dO=3, key lengths=4.
  * key lengths (padding workload): integers uniform in [lo, hi] inclusive
    from generator ``seed + 4``.
  * block mask (block-sparse workload): 128x128 blocks; query block I keeps
    key block J when |I-J| <= 1 (a band of three blocks around the
    diagonal), or J in {0, 1} (two global key blocks every query sees), or
    I in {0, 1} (two global query blocks that see every key).
  * scale: float32(1/sqrt(d)); the same float32 value goes to both sides.

Shapes follow the workloads the attention pages measure on: GPT-2 small
(12 heads, seq 1K, d 64), BERT-large (16 heads, seq 512, d 64), long
context (seq 16K) and block-sparse attention (seq 4K).  No dataset is read.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

BLOCK = 128  # block-mask granularity (rows and columns)

T_Q, T_K, T_V, T_DO, T_LEN = 0, 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str            # "bf16" or "f32"
    causal: bool
    mask: str             # "none" | "causal" | "padding" | "block"
    seed: int
    qk_amp: float = 1.0   # Q and K are amp * N(0,1)
    backward: bool = True
    kv_lo: int = 128
    kv_hi: int = 512
    description: str = ""


WORKLOADS = {
    "fp32_single_head": Workload(
        "fp32_single_head", 1, 1, 128, 64, "f32", False, "none", 1001,
        backward=False,
        description="single-head exact attention in fp32, B1 H1 N128 d64, no mask"),
    "gpt2_causal": Workload(
        "gpt2_causal", 8, 12, 1024, 64, "bf16", True, "causal", 1002,
        description="GPT-2-small-shaped causal self-attention, B8 H12 N1024 d64"),
    "bert_padding": Workload(
        "bert_padding", 16, 16, 512, 64, "bf16", False, "padding", 1003,
        description="BERT-large-shaped attention with key padding, B16 H16 N512 d64, "
                    "valid key length uniform in [128,512]"),
    "long_causal": Workload(
        "long_causal", 1, 16, 16384, 128, "bf16", True, "causal", 1004, qk_amp=2.0,
        description="long-context causal attention, B1 H16 N16384 d128, Q,K ~ 2*N(0,1)"),
    "block_sparse": Workload(
        "block_sparse", 2, 16, 4096, 64, "bf16", False, "block", 1005,
        description="block-sparse attention, B2 H16 N4096 d64, 128x128 blocks: "
                    "band of 3 + 2 global key blocks + 2 global query blocks"),
}


def scale_for(d: int) -> float:
    """float32(1/sqrt(d)) returned as a Python float holding that float32 value."""
    return float(np.float32(1.0 / math.sqrt(d)))


def _normal(seed: int, shape, amp: float) -> np.ndarray:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal(size=int(np.prod(shape)), dtype=np.float64)
    if amp != 1.0:
        x = x * amp
    return x.astype(np.float32).reshape(shape)


def _to_dtype(x32: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(x32)
    if dtype == "bf16":
        return t.to(torch.bfloat16)  # round-to-nearest-even
    if dtype == "f32":
        return t.clone()
    raise ValueError(dtype)


def block_mask_band_global(N: int, band: int = 1, n_global_k: int = 2,
                           n_global_q: int = 2) -> np.ndarray:
    """uint8 [nb, nb] block mask: band of 2*band+1 blocks, global key and query blocks."""
    nb = (N + BLOCK - 1) // BLOCK
    I = np.arange(nb)[:, None]
    J = np.arange(nb)[None, :]
    keep = (np.abs(I - J) <= band) | (J < n_global_k) | (I < n_global_q)
    return keep.astype(np.uint8)


def key_lengths(seed: int, B: int, lo: int, hi: int) -> np.ndarray:
    rng = np.random.default_rng(seed + T_LEN)
    return rng.integers(lo, hi + 1, size=B, dtype=np.int64).astype(np.int32)


def make_inputs(B: int, H: int, N: int, d: int, dtype: str = "bf16", seed: int = 0,
                qk_amp: float = 1.0, causal: bool = False,
                kv_len: Optional[np.ndarray] = None,
                block_mask: Optional[np.ndarray] = None,
                with_grad: bool = True, H_kv: Optional[int] = None) -> dict:
    """Seeded CPU tensors in [B, H, N, d] layout (contiguous).  With ``H_kv`` (grouped-query
    attention) K and V are [B, H_kv, N, d]."""
    shape = (B, H, N, d)
    kv_shape = shape if H_kv is None else (B, H_kv, N, d)
    out = {
        "B": B, "H": H, "N": N, "d": d, "dtype": dtype, "seed": seed,
        "H_kv": H if H_kv is None else H_kv,
        "scale": scale_for(d), "causal": bool(causal),
        "q": _to_dtype(_normal(seed + T_Q, shape, qk_amp), dtype),
        "k": _to_dtype(_normal(seed + T_K, kv_shape, qk_amp), dtype),
        "v": _to_dtype(_normal(seed + T_V, kv_shape, 1.0), dtype),
        "kv_len": None if kv_len is None else torch.from_numpy(np.asarray(kv_len, np.int32)),
        "block_mask": None if block_mask is None else torch.from_numpy(
            np.ascontiguousarray(block_mask, dtype=np.uint8)),
    }
    if with_grad:
        out["do"] = _to_dtype(_normal(seed + T_DO, shape, 1.0), dtype)
    return out


def workload_inputs(name: str, with_grad: Optional[bool] = None, H: Optional[int] = None) -> dict:
    """Inputs of a named workload.  ``H`` may shrink the head count (same per-head recipe)."""
    w = WORKLOADS[name]
    heads = w.H if H is None else H
    kv = key_lengths(w.seed, w.B, w.kv_lo, w.kv_hi) if w.mask == "padding" else None
    bm = block_mask_band_global(w.N) if w.mask == "block" else None
    wg = w.backward if with_grad is None else with_grad
    x = make_inputs(w.B, heads, w.N, w.d, w.dtype, w.seed, w.qk_amp, w.causal, kv, bm, wg)
    x["workload"] = name
    return x


def allowed_pairs(N: int, causal: bool, kv_len: Optional[np.ndarray], B: int,
                  block_mask: Optional[np.ndarray]) -> np.ndarray:
    """Number of unmasked (i, j) pairs per batch entry (one head), int64 [B].

    Counting only: used for FLOP accounting, never for attention values.
    """
    out = np.zeros(B, np.int64)
    i = np.arange(N)
    for b in range(B):
        L = N if kv_len is None else int(min(kv_len[b], N))
        if block_mask is None:
            if causal:
                cnt = np.minimum(i + 1, L).sum()
            else:
                cnt = N * L
        else:
            nb = block_mask.shape[0]
            cnt = 0
            for I in range(nb):
                rows = np.arange(I * BLOCK, min((I + 1) * BLOCK, N))
                for J in range(nb):
                    if not block_mask[I, J]:
                        continue
                    c0, c1 = J * BLOCK, min((J + 1) * BLOCK, L)
                    if c1 <= c0:
                        continue
                    if causal:
                        cnt += np.clip(np.minimum(rows + 1, c1) - c0, 0, None).sum()
                    else:
                        cnt += len(rows) * (c1 - c0)
        out[b] = cnt
    return out
