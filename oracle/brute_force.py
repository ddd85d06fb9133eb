"""Pure-Python brute force of exact attention, for tiny inputs only (N <= 16, d <= 8).

TEST INFRASTRUCTURE ONLY.  A second, separately written statement of the
definition in "Attention optimisation: FlashAttention and sparse attention"
(mdooai, Ch.04), sections "core formula" and "formula key points":
S_ij = scale * q_i . k_j, -inf for keys outside the allowed set, A = row
softmax of S, O = A V; lse is the natural log of the row's sum of exp.
The backward follows the chain rule through each scalar, with no matrix
identities: dO_i.dO/dA_ij, then the softmax Jacobian sum_k dL/dA_ik *
A_ik (delta_kj - A_ij), then S = scale * q . k.
Everything is nested Python loops over lists of floats.
"""
from __future__ import annotations

import math


def _allowed(i, j, causal, block_mask, block, L):
    if j >= L:
        return False
    if causal and j > i:
        return False
    if block_mask is not None and not block_mask[i // block][j // block]:
        return False
    return True


def forward_head(q, k, v, scale, causal=False, block_mask=None, block=128, L=None):
    """q, k, v: lists of rows (lists of floats).  Returns (O rows, lse list, A rows)."""
    N = len(q)
    L = N if L is None else min(L, N)
    O, lse, A = [], [], []
    for i in range(N):
        logits = []
        for j in range(N):
            if _allowed(i, j, causal, block_mask, block, L):
                logits.append(scale * sum(q[i][c] * k[j][c] for c in range(len(q[i]))))
            else:
                logits.append(None)
        finite = [s for s in logits if s is not None]
        if not finite:
            A.append([0.0] * N)
            lse.append(-math.inf)
            O.append([0.0] * len(v[0]))
            continue
        m = max(finite)
        ex = [0.0 if s is None else math.exp(s - m) for s in logits]
        tot = sum(ex)
        a = [e / tot for e in ex]
        A.append(a)
        lse.append(m + math.log(tot))
        O.append([sum(a[j] * v[j][c] for j in range(N)) for c in range(len(v[0]))])
    return O, lse, A


def backward_head(q, k, v, do, scale, causal=False, block_mask=None, block=128, L=None):
    """Gradients of L = sum_ic dO_ic * O_ic with respect to q, k, v (lists of rows)."""
    N = len(q)
    d = len(q[0])
    dv_ = len(v[0])
    _, _, A = forward_head(q, k, v, scale, causal, block_mask, block, L)
    gq = [[0.0] * d for _ in range(N)]
    gk = [[0.0] * d for _ in range(N)]
    gv = [[0.0] * dv_ for _ in range(N)]
    for i in range(N):
        # dL/dA_ij = sum_c dO_ic v_jc ; dL/dv_jc += A_ij dO_ic
        gA = [sum(do[i][c] * v[j][c] for c in range(dv_)) for j in range(N)]
        for j in range(N):
            for c in range(dv_):
                gv[j][c] += A[i][j] * do[i][c]
        # softmax Jacobian: dA_ik/dS_ij = A_ik (delta_kj - A_ij)
        for j in range(N):
            gS = 0.0
            for kk in range(N):
                jac = A[i][kk] * ((1.0 if kk == j else 0.0) - A[i][j])
                gS += gA[kk] * jac
            if gS == 0.0:
                continue
            # S_ij = scale * q_i . k_j
            for c in range(d):
                gq[i][c] += gS * scale * k[j][c]
                gk[j][c] += gS * scale * q[i][c]
    return gq, gk, gv
