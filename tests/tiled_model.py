"""CPU model of the tiled online-softmax recurrence (test artefact, not the oracle).

It walks one head tile by tile the way the CUDA kernel does -- Br query rows
against Bc keys at a time, keeping a running row maximum m and row sum l on
chip and rescaling the output accumulator -- so that the recurrence itself
(stages 3-4 of the five-stage map in "What is FlashAttention? Why smarter
memory use speeds up transformers", and the "partial softmax statistics
accumulated on-chip, tile by tile" of mdooai Ch.04) can be checked against
the materialised oracle before any GPU code runs.

Options mirror the kernel's choices:
  * ``lazy_threshold``: the reference maximum is only raised when a tile's
    maximum exceeds it by more than this many log2 units (0 = always).
    The final division by l uses the same reference, so the result is exact.
  * ``round_p_bf16``: round P to bfloat16 before the P.V product (the tensor
    core consumes bf16 P); l is summed from the unrounded fp32-or-fp64 P unless
    ``l_rounded`` is set, in which case l sums the rounded P that enters P.V.
  * ``reverse``: visit the key tiles from the last to the first.  In exact
    arithmetic the order does not matter; in floating point it is one of the
    axes of the deviation study in "Is Flash Attention Stable?".
  * ``dtype``: float64 (exactness check) or float32 (kernel-like arithmetic).
"""
from __future__ import annotations

import numpy as np
import torch

LOG2E = 1.4426950408889634


def _bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).to(torch.float32).numpy()


def tiled_forward_head(q, k, v, scale, causal=False, L=None, block_mask=None, block=128,
                       Br=128, Bc=128, lazy_threshold=0.0, round_p_bf16=False,
                       dtype=np.float64, reverse=False, l_rounded=False):
    q = np.asarray(q, dtype)
    k = np.asarray(k, dtype)
    v = np.asarray(v, dtype)
    N, d = q.shape
    L = N if L is None else min(int(L), N)
    scale2 = dtype(scale * LOG2E) if dtype is np.float32 else scale * LOG2E
    O = np.zeros((N, v.shape[1]), np.float64)
    lse = np.full(N, -np.inf)
    for r0 in range(0, N, Br):
        rows = np.arange(r0, min(r0 + Br, N))
        m = np.full(len(rows), -np.inf, dtype)
        l = np.zeros(len(rows), dtype)
        acc = np.zeros((len(rows), v.shape[1]), dtype)
        starts = list(range(0, N, Bc))
        for c0 in (starts[::-1] if reverse else starts):
            cols = np.arange(c0, min(c0 + Bc, N))
            allowed = (cols[None, :] < L) & np.ones((len(rows), 1), bool)
            if causal:
                allowed &= cols[None, :] <= rows[:, None]
            if block_mask is not None:
                allowed &= np.asarray(block_mask, bool)[rows[:, None] // block,
                                                        cols[None, :] // block]
            if not allowed.any():
                continue  # whole tile skipped
            s = (q[rows] @ k[cols].T).astype(dtype) * scale2   # log2 domain
            s = np.where(allowed, s, -np.inf)
            tile_max = s.max(axis=1)
            m_new = m.copy()
            raise_ = tile_max > m + lazy_threshold
            raise_ |= np.isneginf(m) & np.isfinite(tile_max)
            m_new[raise_] = tile_max[raise_]
            alpha = np.where(np.isneginf(m_new), 1.0, np.exp2(np.where(
                np.isneginf(m), -np.inf, m - m_new))).astype(dtype)
            alpha = np.where(np.isneginf(m), 0.0, alpha).astype(dtype)
            base = np.where(np.isneginf(m_new), 0.0, m_new)
            p = np.exp2(s - base[:, None]).astype(dtype)
            p = np.where(allowed, p, 0.0).astype(dtype)
            pv = _bf16(p) if round_p_bf16 else p
            l = alpha * l + (pv if l_rounded else p).sum(axis=1, dtype=dtype)
            acc = alpha[:, None] * acc + (pv @ v[cols]).astype(dtype)
            m = m_new
        ok = l > 0
        O[rows[ok]] = (acc[ok] / l[ok, None]).astype(np.float64)
        lse[rows[ok]] = (m[ok].astype(np.float64) + np.log2(l[ok].astype(np.float64))) / LOG2E
    return O, lse
