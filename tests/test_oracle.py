"""Pins for the FP64 CPU oracle: checked against what the pages and the mathematics fix.

The attention pages print no worked numeric example, so every pin is a closed
form, an invariant, a special case with a known answer, an independent
pure-Python brute force, or finite differences.  Each is chosen so that a
plausible mistake (a dropped scale, a wrong sign, a transposed operand, the
wrong mask direction, a transposed block mask, a log base) fails one of them.
"""
import math

import numpy as np
import pytest

import oracle
from oracle import brute_force as bf

RNG = np.random.default_rng(12345)


def rand(*shape, amp=1.0):
    return RNG.standard_normal(shape) * amp


# ---------------------------------------------------------------- closed forms

def test_closed_form_two_keys():
    """Logits (0, ln 3) give weights (1/4, 3/4): softmax definition, mdooai Ch.04 core formula."""
    S = np.array([[0.0, math.log(3.0)]])
    V = np.array([[4.0, -1.0], [8.0, 3.0]])
    o, lse, A = oracle.softmax_av(S, V)
    assert np.allclose(A, [[0.25, 0.75]], rtol=0, atol=1e-15)
    assert np.allclose(o, [[7.0, 2.0]], rtol=0, atol=1e-14)
    assert abs(lse[0] - math.log(4.0)) < 1e-15


def test_single_token():
    """N = 1: the only weight is 1, O = v_0, lse = scale * q.k."""
    q, k, v = rand(1, 1, 1, 5), rand(1, 1, 1, 5), rand(1, 1, 1, 5)
    o, lse = oracle.attn_fwd(q, k, v, 0.37)
    assert np.allclose(o, v, rtol=0, atol=1e-15)
    assert abs(lse[0, 0, 0] - 0.37 * float(q.ravel() @ k.ravel())) < 1e-14


def test_scale_enters_logits():
    """Two keys, d = 1: A_00 = sigmoid(scale*q*(k0-k1)) -- fails if the scale is dropped."""
    q = np.array([[[[2.0], [0.0]]]])
    k = np.array([[[[1.5], [-0.5]]]])
    v = np.array([[[[1.0], [0.0]]]])
    for scale in (1.0, 0.125, 0.7):
        o, lse = oracle.attn_fwd(q, k, v, scale)
        x = scale * 2.0 * (1.5 - (-0.5))
        assert abs(o[0, 0, 0, 0] - 1.0 / (1.0 + math.exp(-x))) < 1e-15
        assert abs(o[0, 0, 1, 0] - 0.5) < 1e-15
        ref_lse = math.log(math.exp(scale * 3.0) + math.exp(scale * -1.0))
        assert abs(lse[0, 0, 0] - ref_lse) < 1e-14


def test_zero_queries_give_mean_of_allowed_values():
    """q = 0 makes every allowed logit 0: A is uniform on the allowed keys."""
    N, d = 9, 4
    q = np.zeros((1, 1, N, d))
    k, v = rand(1, 1, N, d), rand(1, 1, N, d)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=True)
    for i in range(N):
        assert np.allclose(o[0, 0, i], v[0, 0, :i + 1].mean(axis=0), rtol=0, atol=1e-14)
        assert abs(lse[0, 0, i] - math.log(i + 1)) < 1e-14


# ---------------------------------------------------------------- invariants

@pytest.mark.parametrize("causal,L,use_bm", [(False, None, False), (True, None, False),
                                             (False, 11, False), (True, 7, True)])
def test_rows_sum_to_one(causal, L, use_bm):
    """Each row of A sums to 1 over its allowed keys (mdooai Ch.04, formula key points)."""
    N, d = 24, 6
    q, k = rand(N, d), rand(N, d)
    bm = None
    if use_bm:
        bm = np.ones((3, 3), np.uint8)
        bm[2, 0] = 0
        bm[0, 2] = 0
    A, lse = oracle.attn_probs(q, k, 0.4, causal, bm, -1 if L is None else L, block=8)
    Lm = N if L is None else L
    i, j = np.meshgrid(np.arange(N), np.arange(N), indexing="ij")
    allowed = (j < Lm) & ((not causal) | (j <= i))
    if use_bm:
        allowed &= bm[i // 8, j // 8].astype(bool)
    has_key = allowed.any(axis=1)
    sums = A.sum(axis=1)
    assert np.all(np.abs(sums[has_key] - 1.0) < 1e-14)
    assert np.all(sums[~has_key] == 0.0) and np.all(np.isneginf(lse[~has_key]))
    assert np.all(A[~allowed] == 0.0) and np.all(A[allowed & has_key[:, None]] > 0)
    assert np.all(A[:, Lm:] == 0.0)
    if causal:
        assert np.all(np.triu(A, 1) == 0.0)
    if use_bm:
        assert np.all(A[16:24, 0:8] == 0.0) and np.all(A[0:8, 16:24] == 0.0)


def test_shift_invariance_per_row():
    """Adding c_i to row i of the logits leaves O unchanged and shifts lse by c_i."""
    S = rand(12, 15, amp=3.0)
    S[2, 4] = -np.inf
    S[5, :7] = -np.inf
    V = rand(15, 5)
    c = rand(12, 1, amp=50.0)
    o1, l1, _ = oracle.softmax_av(S, V)
    o2, l2, _ = oracle.softmax_av(S + c, V)
    assert np.max(np.abs(o1 - o2)) < 1e-13
    assert np.max(np.abs((l2 - l1) - c[:, 0])) < 1e-12


def test_identical_keys_average_values():
    """All k_j equal: O_i is the mean of the allowed v_j and lse_i = s_i + ln(n_i)."""
    N, d = 20, 8
    q = rand(1, 1, N, d)
    k = np.broadcast_to(rand(1, d), (N, d)).reshape(1, 1, N, d).copy()
    v = rand(1, 1, N, d)
    scale = 0.3
    for causal in (False, True):
        o, lse = oracle.attn_fwd(q, k, v, scale, causal=causal)
        for i in range(N):
            n = i + 1 if causal else N
            assert np.allclose(o[0, 0, i], v[0, 0, :n].mean(axis=0), rtol=0, atol=1e-13)
            s = scale * float(q[0, 0, i] @ k[0, 0, 0])
            assert abs(lse[0, 0, i] - (s + math.log(n))) < 1e-12


def test_dominant_logit_selects_its_value():
    """A logit 1000 above the rest makes O_i = v_j* (to 1e-12)."""
    S = rand(6, 10)
    V = rand(10, 4)
    jstar = [3, 0, 9, 5, 5, 1]
    for i, j in enumerate(jstar):
        S[i, j] += 1000.0
    o, _, _ = oracle.softmax_av(S, V)
    for i, j in enumerate(jstar):
        assert np.max(np.abs(o[i] - V[j])) < 1e-12
    # the same through the q.k path: q_i aligned with one key, scaled up
    N, d = 8, 3
    k = rand(1, 1, N, d)
    q = np.zeros((1, 1, N, d))
    js = [2, 7, 0, 5, 5, 1, 3, 6]
    for i, j in enumerate(js):
        q[0, 0, i] = k[0, 0, j] / np.dot(k[0, 0, j], k[0, 0, j]) * 4000.0
    k2 = k.copy()
    v = rand(1, 1, N, d)
    o, _ = oracle.attn_fwd(q, k2, v, 1.0)
    for i, j in enumerate(js):
        # logit of j* is 4000, others are 4000 * cos * |k_j|/|k_j*| < 4000 - large margin
        others = [4000.0 * float(k[0, 0, jj] @ k[0, 0, j]) / float(k[0, 0, j] @ k[0, 0, j])
                  for jj in range(N) if jj != j]
        if max(others) < 4000.0 - 60.0:
            assert np.max(np.abs(o[0, 0, i] - v[0, 0, j])) < 1e-12


def test_fully_masked_row_convention():
    """A row with no allowed key: O = 0, lse = -inf (block mask removes its only block)."""
    N, d = 8, 3
    q, k, v = rand(1, 1, N, d), rand(1, 1, N, d), rand(1, 1, N, d)
    bm = np.array([[0, 1], [1, 1]], np.uint8)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=True, block_mask=bm, block=4)
    # causal + block (0,0) removed: rows 0..3 see nothing
    assert np.all(o[0, 0, :4] == 0.0) and np.all(np.isneginf(lse[0, 0, :4]))
    assert np.all(np.isfinite(lse[0, 0, 4:]))
    dq, dk, dv = oracle.attn_bwd(q, k, v, rand(1, 1, N, d), 0.5, causal=True, block_mask=bm,
                                 block=4)
    assert np.all(dq[0, 0, :4] == 0.0)


# ---------------------------------------------------------------- brute force

def _case(N, d, causal, L, bm, block, seed):
    r = np.random.default_rng(seed)
    q, k, v, do = (r.standard_normal((N, d)) for _ in range(4))
    return q, k, v, do


CASES = [
    # N, d, causal, L, block_mask, block
    (1, 1, False, None, None, 4),
    (5, 3, False, None, None, 4),
    (7, 8, True, None, None, 4),
    (16, 8, False, 9, None, 4),
    (16, 5, True, 11, None, 4),
    (12, 4, False, None, [[1, 0, 1], [0, 1, 0], [1, 1, 0]], 4),
    (16, 6, True, 14, [[1, 0, 0, 1], [1, 1, 0, 0], [0, 1, 1, 1], [1, 0, 1, 1]], 4),
    (10, 2, False, None, [[0, 1, 1], [1, 0, 1], [1, 1, 1]], 4),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_forward_matches_brute_force(case):
    N, d, causal, L, bml, block = CASES[case]
    q, k, v, _ = _case(N, d, causal, L, bml, block, 100 + case)
    scale = 0.5 + 0.1 * case
    bm = None if bml is None else np.array(bml, np.uint8)
    O, lse, _ = bf.forward_head(q.tolist(), k.tolist(), v.tolist(), scale, causal, bml, block, L)
    o, l = oracle.attn_fwd(q[None, None], k[None, None], v[None, None], scale, causal,
                           block_mask=bm, kv_len=None if L is None else np.array([L], np.int32),
                           block=block)
    assert np.max(np.abs(o[0, 0] - np.array(O))) < 1e-12
    lse_bf = np.array(lse)
    fin = np.isfinite(lse_bf)
    assert np.array_equal(fin, np.isfinite(l[0, 0]))
    assert np.max(np.abs(l[0, 0][fin] - lse_bf[fin]), initial=0.0) < 1e-12
    # the rows-only entry computes the same rows
    rows = list(range(0, N, 2))
    o_r, l_r = oracle.attn_fwd_rows(q[None, None], k[None, None], v[None, None], scale, rows,
                                    causal, bm, None if L is None else np.array([L], np.int32),
                                    block)
    assert np.max(np.abs(o_r - o[0, 0, rows])) < 1e-15


@pytest.mark.parametrize("case", range(len(CASES)))
def test_backward_matches_brute_force(case):
    N, d, causal, L, bml, block = CASES[case]
    q, k, v, do = _case(N, d, causal, L, bml, block, 200 + case)
    scale = 0.3 + 0.05 * case
    bm = None if bml is None else np.array(bml, np.uint8)
    gq, gk, gv = bf.backward_head(q.tolist(), k.tolist(), v.tolist(), do.tolist(), scale,
                                  causal, bml, block, L)
    dq, dk, dv = oracle.attn_bwd(q[None, None], k[None, None], v[None, None], do[None, None],
                                 scale, causal, bm,
                                 None if L is None else np.array([L], np.int32), block)
    for got, ref in ((dq, gq), (dk, gk), (dv, gv)):
        ref = np.array(ref)
        assert np.max(np.abs(got[0, 0] - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_multi_head_batches_are_independent():
    """Heads and batch entries do not mix; kv_len applies per batch entry."""
    B, H, N, d = 2, 3, 6, 4
    q, k, v = rand(B, H, N, d), rand(B, H, N, d), rand(B, H, N, d)
    L = np.array([4, 6], np.int32)
    o, lse = oracle.attn_fwd(q, k, v, 0.6, causal=True, kv_len=L)
    for b in range(B):
        for h in range(H):
            O, ls, _ = bf.forward_head(q[b, h].tolist(), k[b, h].tolist(), v[b, h].tolist(),
                                       0.6, True, None, 128, int(L[b]))
            assert np.max(np.abs(o[b, h] - np.array(O))) < 1e-12


# ---------------------------------------------------------------- backward pins

def _loss(q, k, v, do, scale, causal, L):
    o, _ = oracle.attn_fwd(q, k, v, scale, causal, kv_len=L)
    return float(np.sum(o * do))


@pytest.mark.parametrize("causal,L", [(False, None), (True, np.array([5], np.int32))])
def test_backward_finite_differences(causal, L):
    """Central differences of L = sum(dO * O) in fp64 (h = 1e-6) agree to 1e-6 relative."""
    N, d = 7, 3
    q, k, v, do = (rand(1, 1, N, d) for _ in range(4))
    scale = 0.45
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, scale, causal, kv_len=L)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        num = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args = {"q": q, "k": k, "v": v}
            args[name] = xp
            lp = _loss(args["q"], args["k"], args["v"], do, scale, causal, L)
            args[name] = xm
            lm = _loss(args["q"], args["k"], args["v"], do, scale, causal, L)
            num[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(num - g)) / max(np.max(np.abs(g)), 1e-30)
        assert err < 1e-6, (name, err)


def test_backward_invariants():
    """sum_j dK_j = 0; sum_j dV_j = sum_i dO_i (rows with keys); padded keys get 0."""
    B, H, N, d = 2, 2, 40, 5
    q, k, v, do = (rand(B, H, N, d) for _ in range(4))
    L = np.array([23, 40], np.int32)
    for causal in (False, True):
        dq, dk, dv = oracle.attn_bwd(q, k, v, do, 0.35, causal, kv_len=L)
        assert np.max(np.abs(dk.sum(axis=2))) < 1e-12
        assert np.max(np.abs(dv.sum(axis=2) - do.sum(axis=2))) < 1e-12
        assert np.all(dk[0, :, 23:] == 0.0) and np.all(dv[0, :, 23:] == 0.0)


def test_backward_head_subset():
    B, H, N, d = 1, 3, 10, 4
    q, k, v, do = (rand(B, H, N, d) for _ in range(4))
    full = oracle.attn_bwd(q, k, v, do, 0.5, True)
    part = oracle.attn_bwd(q, k, v, do, 0.5, True, heads=[2])
    for a, b in zip(full, part):
        assert np.array_equal(a[0, 2], b[0, 2])
        assert np.all(b[0, :2] == 0.0)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_dq_rows_match_brute_force(case):
    """The row-restricted dQ equals the brute-force chain rule on the same rows."""
    N, d, causal, L, bml, block = CASES[case]
    q, k, v, do = _case(N, d, causal, L, bml, block, 300 + case)
    scale = 0.4
    bm = None if bml is None else np.array(bml, np.uint8)
    gq, _, _ = bf.backward_head(q.tolist(), k.tolist(), v.tolist(), do.tolist(), scale, causal,
                                bml, block, L)
    rows = list(range(N))[::-1]
    dq = oracle.attn_bwd_dq_rows(q[None, None], k[None, None], v[None, None], do[None, None],
                                 scale, rows, causal, bm,
                                 None if L is None else np.array([L], np.int32), block)
    ref = np.array(gq)[rows]
    assert np.max(np.abs(dq - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("case", range(len(CASES)))
def test_kv_rows_match_brute_force(case):
    """dK and dV of selected key rows equal the brute-force chain rule on the same keys (every
    mask kind, ragged lengths, keys listed out of order and one key twice)."""
    N, d, causal, L, bml, block = CASES[case]
    q, k, v, do = _case(N, d, causal, L, bml, block, 400 + case)
    scale = 0.55
    bm = None if bml is None else np.array(bml, np.uint8)
    _, gk, gv = bf.backward_head(q.tolist(), k.tolist(), v.tolist(), do.tolist(), scale, causal,
                                 bml, block, L)
    rows = list(range(N))[::-1] + [N // 2]
    dk, dv = oracle.attn_bwd_kv_rows(q[None, None], k[None, None], v[None, None],
                                     do[None, None], scale, rows, causal, bm,
                                     None if L is None else np.array([L], np.int32), block)
    for got, ref in ((dk, np.array(gk)[rows]), (dv, np.array(gv)[rows])):
        assert np.max(np.abs(got - ref)) < 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_kv_rows_match_full_backward_across_heads():
    """Across batch entries and heads (per-batch key lengths, a block mask with a fully masked
    query block), the key-row entry reproduces the full backward's dK and dV rows, and keys
    beyond a batch entry's length get exactly 0."""
    B, H, N, d = 2, 3, 48, 6
    q, k, v, do = (rand(B, H, N, d) for _ in range(4))
    L = np.array([37, 48], np.int32)
    bm = np.ones((3, 3), np.uint8)
    bm[1, :] = 0            # query rows 16..31 see no key
    bm[2, 0] = 0
    for causal in (False, True):
        _, dk, dv = oracle.attn_bwd(q, k, v, do, 0.4, causal, bm, L, block=16)
        rng = np.random.default_rng(5)
        rows = np.concatenate([rng.choice(B * H * N, 40, replace=False), [0, N - 1, B * H * N - 1]])
        gk, gv = oracle.attn_bwd_kv_rows(q, k, v, do, 0.4, rows, causal, bm, L, block=16)
        ref_k, ref_v = dk.reshape(-1, d)[rows], dv.reshape(-1, d)[rows]
        assert np.max(np.abs(gk - ref_k)) < 1e-13 * max(1.0, np.abs(ref_k).max())
        assert np.max(np.abs(gv - ref_v)) < 1e-13 * max(1.0, np.abs(ref_v).max())
        pad = [r for r in range(N) if r >= 37]       # batch 0, head 0, padded keys
        zk, zv = oracle.attn_bwd_kv_rows(q, k, v, do, 0.4, pad, causal, bm, L, block=16)
        assert np.all(zk == 0.0) and np.all(zv == 0.0)


def test_kv_rows_sum_invariants():
    """Summed over every key of a head, dK is 0 and dV is the sum of dO over rows with a key --
    the backward invariants, now through the key-row entry."""
    N, d = 30, 4
    q, k, v, do = (rand(1, 1, N, d) for _ in range(4))
    dk, dv = oracle.attn_bwd_kv_rows(q, k, v, do, 0.7, list(range(N)), True)
    assert np.max(np.abs(dk.sum(axis=0))) < 1e-12
    assert np.max(np.abs(dv.sum(axis=0) - do[0, 0].sum(axis=0))) < 1e-12
