"""Pins of the grouped-query oracle (CPU, fp64).

Grouped-query and multi-query attention are named on the tcdigital FA-2 ROI article (section
"MQA/GQA ... との相乗効果") without a formula; the reading used here is the one of the models it
names (Llama 2/3): query head h reads K/V head h // (H / H_kv).  The oracle writes that as the
ordinary attention over repeated K/V heads.  These tests fix the head mapping by a closed form
and the summed K/V gradients by finite differences, independently of that construction.
"""
import numpy as np
import pytest

import oracle

R = np.random.default_rng(11)


@pytest.mark.parametrize("H,H_kv", [(4, 2), (6, 3), (4, 1), (3, 3)])
def test_head_mapping_closed_form(H, H_kv):
    """V head j is the constant j + 1, so every output row of query head h is exactly
    h // (H / H_kv) + 1, whatever the scores are."""
    B, N, d = 2, 37, 8
    q = R.standard_normal((B, H, N, d))
    k = R.standard_normal((B, H_kv, N, d)) * 3.0
    v = np.broadcast_to(np.arange(1, H_kv + 1, dtype=np.float64)[None, :, None, None],
                        (B, H_kv, N, d)).copy()
    for causal in (False, True):
        o, lse = oracle.attn_fwd_gqa(q, k, v, 0.3, causal)
        G = H // H_kv
        for h in range(H):
            assert np.max(np.abs(o[:, h] - (h // G + 1))) < 1e-13


def _loss(q, k, v, do, scale, causal):
    o, _ = oracle.attn_fwd_gqa(q, k, v, scale, causal)
    return float(np.sum(do * o))


@pytest.mark.parametrize("causal", [False, True])
def test_gradients_by_finite_differences(causal):
    """dQ, dK, dV of L = sum(dO * O) by central differences (h = 1e-6): the K/V gradients must
    collect every query head of the group."""
    B, H, H_kv, N, d, scale = 1, 4, 2, 5, 3, 0.7
    q = R.standard_normal((B, H, N, d))
    k = R.standard_normal((B, H_kv, N, d))
    v = R.standard_normal((B, H_kv, N, d))
    do = R.standard_normal((B, H, N, d))
    dq, dk, dv = oracle.attn_bwd_gqa(q, k, v, do, scale, causal)
    assert dk.shape == k.shape and dv.shape == v.shape and dq.shape == q.shape
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, scale, causal)
            num[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(num - g)) / max(1.0, np.max(np.abs(g)))
        assert err < 1e-6, (name, err)


def test_multi_query_with_identical_heads_scales_the_kv_gradient():
    """H identical query heads over one K/V head: dK and dV are H times those of one head, and
    every query head gets the single-head dQ."""
    B, H, N, d = 1, 5, 40, 16
    q1 = R.standard_normal((B, 1, N, d))
    do1 = R.standard_normal((B, 1, N, d))
    k = R.standard_normal((B, 1, N, d))
    v = R.standard_normal((B, 1, N, d))
    dq1, dk1, dv1 = oracle.attn_bwd(q1, k, v, do1, 0.25, True)
    dq, dk, dv = oracle.attn_bwd_gqa(np.repeat(q1, H, 1), k, v, np.repeat(do1, H, 1), 0.25, True)
    assert np.max(np.abs(dk - H * dk1)) < 1e-12 * max(1, np.abs(dk).max())
    assert np.max(np.abs(dv - H * dv1)) < 1e-12 * max(1, np.abs(dv).max())
    for h in range(H):
        assert np.max(np.abs(dq[:, h] - dq1[:, 0])) < 1e-13


def test_kv_head_subset_matches_full():
    B, H, H_kv, N, d = 2, 6, 2, 50, 8
    q = R.standard_normal((B, H, N, d))
    k = R.standard_normal((B, H_kv, N, d))
    v = R.standard_normal((B, H_kv, N, d))
    do = R.standard_normal((B, H, N, d))
    full = oracle.attn_bwd_gqa(q, k, v, do, 0.35, True)
    part = oracle.attn_bwd_gqa(q, k, v, do, 0.35, True, kv_heads=[3])  # b = 1, j = 1
    for a, b_ in zip(full[1:], part[1:]):
        assert np.array_equal(a[1, 1], b_[1, 1])
    assert np.array_equal(full[0][1, 3:6], part[0][1, 3:6])


def test_group_size_must_divide():
    with pytest.raises(ValueError):
        oracle.kv_group(6, 4)
