"""The tiled online-softmax recurrence equals the materialised definition (CPU, fp64).

FlashAttention computes exactly the same attention as the dense form, only
tile by tile ("What is FlashAttention?", definition section; mdooai Ch.04).
In fp64 the tiled model must agree with the oracle to 1e-12 for every tile
shape of the deviation sweep, every mask, and with lazy rescaling on.
"""
import numpy as np
import pytest

import oracle
from tiled_model import tiled_forward_head

R = np.random.default_rng(7)


@pytest.mark.parametrize("Br,Bc", [(64, 64), (64, 128), (64, 256), (128, 64), (128, 128),
                                   (128, 256)])
@pytest.mark.parametrize("mask", ["none", "causal", "padding", "block"])
@pytest.mark.parametrize("lazy", [0.0, 8.0])
def test_tiled_equals_oracle(Br, Bc, mask, lazy):
    N, d = 300, 16
    q, k, v = (R.standard_normal((N, d)) * a for a in (2.0, 2.0, 1.0))
    scale = 0.25
    causal = mask == "causal"
    L = 211 if mask == "padding" else None
    bm, block = None, 128
    if mask == "block":
        block = 32
        nb = (N + block - 1) // block
        I, J = np.meshgrid(np.arange(nb), np.arange(nb), indexing="ij")
        bm = ((np.abs(I - J) <= 1) | (J < 2) | (I < 2)).astype(np.uint8)
    o_ref, lse_ref = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], scale,
                                     causal, bm, None if L is None else np.array([L]), block)
    o, lse = tiled_forward_head(q, k, v, scale, causal, L, bm, block, Br, Bc, lazy)
    assert np.max(np.abs(o - o_ref[0, 0])) < 1e-12
    assert np.max(np.abs(lse - lse_ref[0, 0])) < 1e-12


def test_lazy_rescale_threshold_is_exact_for_large_jumps():
    """Logits that jump by far more than the threshold between tiles stay exact."""
    N, d = 256, 8
    q = R.standard_normal((N, d))
    k = R.standard_normal((N, d))
    k[200:] *= 30.0   # late keys dominate
    v = R.standard_normal((N, d))
    o_ref, lse_ref = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], 0.35)
    o, lse = tiled_forward_head(q, k, v, 0.35, Br=64, Bc=64, lazy_threshold=8.0)
    assert np.max(np.abs(o - o_ref[0, 0])) < 1e-12
    assert np.max(np.abs(lse - lse_ref[0, 0])) < 1e-12


def test_bf16_p_rounding_stays_inside_tolerance():
    """fp32 arithmetic with bf16 P on the long-context value scale (Q,K ~ 2N(0,1), d=128)."""
    N, d = 1024, 128
    q, k = (R.standard_normal((N, d)) * 2.0 for _ in range(2))
    v = R.standard_normal((N, d))
    qb, kb, vb = (np.asarray(__import__("torch").from_numpy(x.astype(np.float32)).to(
        __import__("torch").bfloat16).float()) for x in (q, k, v))
    scale = float(np.float32(1 / np.sqrt(d)))
    o_ref, _ = oracle.attn_fwd(qb[None, None], kb[None, None], vb[None, None], scale, True)
    o, _ = tiled_forward_head(qb, kb, vb, scale, True, Br=128, Bc=128, lazy_threshold=8.0,
                              round_p_bf16=True, dtype=np.float32)
    err = np.abs(o - o_ref[0, 0])
    assert err.max() < 2e-2 and err.mean() < 2e-3


@pytest.mark.parametrize("Bc", [64, 128, 256])
@pytest.mark.parametrize("mask", ["none", "causal", "padding"])
def test_reverse_tile_order_is_exact(Bc, mask):
    """Visiting the key tiles last to first changes nothing in exact arithmetic: the tile-order
    axis of "Is Flash Attention Stable?" (aibr.jp summary, section 3) only moves rounding."""
    N, d = 333, 16
    q, k, v = (R.standard_normal((N, d)) * a for a in (2.0, 2.0, 1.0))
    causal = mask == "causal"
    L = 250 if mask == "padding" else None
    o_ref, lse_ref = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], 0.25, causal,
                                     None, None if L is None else np.array([L]))
    for lazy in (0.0, 8.0):
        o, lse = tiled_forward_head(q, k, v, 0.25, causal, L, Bc=Bc, lazy_threshold=lazy,
                                    reverse=True)
        assert np.max(np.abs(o - o_ref[0, 0])) < 1e-12
        assert np.max(np.abs(lse - lse_ref[0, 0])) < 1e-12


def test_rounded_normaliser_makes_rows_sum_to_one():
    """With l summed over the same bf16-rounded P that multiplies V, the effective attention
    weights of a row sum to one: V = 1 gives O = 1 to fp64 rounding.  With l over the unrounded
    P the ratio sum(round(P)) / sum(P) is left in O (reading c-7 of the normaliser choice)."""
    N, d = 256, 8
    q, k = (R.standard_normal((N, d)) * 2.0 for _ in range(2))
    v = np.ones((N, 4))
    o_r, _ = tiled_forward_head(q, k, v, 0.35, True, Bc=64, round_p_bf16=True, l_rounded=True)
    assert np.max(np.abs(o_r - 1.0)) < 1e-13
    o_f, _ = tiled_forward_head(q, k, v, 0.35, True, Bc=64, round_p_bf16=True, l_rounded=False)
    dev = np.abs(o_f - 1.0)
    assert dev.max() > 1e-6            # the rounding of P shows
    assert dev.max() < 2.0 ** -8       # but stays within bf16's relative rounding of P


@pytest.mark.parametrize("reverse", [False, True])
@pytest.mark.parametrize("l_rounded", [False, True])
def test_deviation_axes_stay_inside_tolerance(reverse, l_rounded):
    """fp32 arithmetic, bf16 P, both tile orders and both normalisers, on the long-context value
    scale: every variant of the deviation sweep stays within the bf16 tolerance of the oracle."""
    N, d = 512, 64
    torch = __import__("torch")
    q, k = (R.standard_normal((N, d)) * 2.0 for _ in range(2))
    v = R.standard_normal((N, d))
    qb, kb, vb = (torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).float().numpy()
                  for x in (q, k, v))
    o_ref, _ = oracle.attn_fwd(qb[None, None], kb[None, None], vb[None, None], 0.125, True)
    o, _ = tiled_forward_head(qb, kb, vb, 0.125, True, Bc=64, round_p_bf16=True,
                              dtype=np.float32, reverse=reverse, l_rounded=l_rounded)
    err = np.abs(o - o_ref[0, 0])
    assert err.max() < 2e-2 and err.mean() < 2e-3
