"""Grouped-query / multi-query attention on the GPU (fa_fwd_gqa, fa_bwd_gqa through the C ABI)
against the grouped-query oracle: query head h reads K/V head h // (H / H_kv), and the K/V
gradients sum over the query heads of a group."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import compare_grad, compare_lse, compare_o, f64, to_gpu

pytestmark = pytest.mark.gpu


def _inputs(B, H, H_kv, N, d, causal, L=None, use_bm=False, seed=0, dtype="bf16", grad=True):
    return syn.make_inputs(B, H, N, d, dtype, seed=seed, causal=causal,
                           kv_len=None if L is None else np.array(L, np.int32),
                           block_mask=syn.block_mask_band_global(N) if use_bm else None,
                           with_grad=grad, H_kv=H_kv)


def _fwd(fa, g):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return o, lse


def _fb(fa, g):
    o, lse = _fwd(fa, g)
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                        g["block_mask"], g["kv_len"])
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return o, lse, dq, dk, dv


CASES = [
    # B, H, H_kv, N, d, causal, kv_len, block mask
    (2, 4, 2, 700, 64, True, None, False),
    (1, 6, 2, 777, 128, False, None, False),
    (2, 4, 1, 513, 128, True, [513, 300], False),   # multi-query, key padding
    (1, 8, 2, 900, 64, False, None, True),          # band + global block mask
    (1, 3, 3, 300, 64, True, None, False),          # H_kv = H through the grouped entry
    (1, 4, 2, 129, 128, True, None, False),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_gqa_forward_and_backward(cuda_lib, case):
    B, H, H_kv, N, d, causal, L, use_bm = CASES[case]
    x = _inputs(B, H, H_kv, N, d, causal, L, use_bm, seed=1200 + case)
    o, lse, dq, dk, dv = _fb(cuda_lib, to_gpu(x))
    assert dk.shape == x["k"].shape and dv.shape == x["v"].shape
    o_ref, lse_ref = oracle.attn_fwd_gqa(x["q"], x["k"], x["v"], x["scale"], causal,
                                         x["block_mask"], x["kv_len"])
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], causal,
                                     x["block_mask"], x["kv_len"])
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")
    if L is not None:
        for b, Lb in enumerate(L):
            assert torch.all(dk[b, :, Lb:] == 0) and torch.all(dv[b, :, Lb:] == 0)


def test_gqa_forward_is_mha_on_repeated_kv(cuda_lib):
    """The grouped forward reads the same K/V values as the ordinary forward over repeated K/V
    heads, in the same order: O and lse are bit-identical."""
    x = _inputs(2, 8, 2, 1000, 128, True, seed=1300, grad=False)
    g = to_gpu(x)
    o, lse = _fwd(cuda_lib, g)
    G = 4
    o2, lse2 = cuda_lib.fwd(g["q"], g["k"].repeat_interleave(G, 1).contiguous(),
                            g["v"].repeat_interleave(G, 1).contiguous(), g["scale"], True)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(lse, lse2)


def test_gqa_fp32_forward(cuda_lib):
    x = _inputs(1, 4, 2, 200, 64, False, seed=1301, dtype="f32", grad=False)
    o, lse = _fwd(cuda_lib, to_gpu(x))
    o_ref, lse_ref = oracle.attn_fwd_gqa(x["q"], x["k"], x["v"], x["scale"], False)
    compare_o(f64(o), o_ref, "f32")
    compare_lse(f64(lse), lse_ref, 1e-5)


def test_gqa_llama_like_sampled(cuda_lib):
    """B1 H32 H_kv8 N2048 d128 causal (the grouping of Llama-class models): two K/V groups
    differentiated in full by the oracle, forward rows sampled."""
    x = _inputs(1, 32, 8, 2048, 128, True, seed=1302)
    o, lse, dq, dk, dv = _fb(cuda_lib, to_gpu(x))
    rows = np.unique(np.concatenate([np.random.default_rng(3).choice(32 * 2048, 300, replace=False),
                                     [0, 2047, 2048, 32 * 2048 - 1]]))
    qrep = lambda t: np.repeat(f64(t), 4, axis=1)
    o_ref, l_ref = oracle.attn_fwd_rows(f64(x["q"]), qrep(x["k"]), qrep(x["v"]), x["scale"], rows,
                                        True)
    compare_o(f64(o).reshape(-1, 128)[rows], o_ref)
    compare_lse(f64(lse).reshape(-1)[rows], l_ref)
    kv_heads = [0, 5]
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], True,
                                     kv_heads=kv_heads)
    for j in kv_heads:
        compare_grad(f64(dk[0, j]), rk[0, j], f"dK[{j}]")
        compare_grad(f64(dv[0, j]), rv[0, j], f"dV[{j}]")
        for h in range(4 * j, 4 * j + 4):
            compare_grad(f64(dq[0, h]), rq[0, h], f"dQ[{h}]")


def test_gqa_long_all_groups(cuda_lib):
    """B1 H32 H_kv8 N8192 d128 causal: the backward's CTAs run in groups of two K/V heads.  dK and
    dV of every K/V head equal the deterministic backward's bit for bit, and dQ rows sampled over
    all 32 query heads match the oracle (on K/V repeated per query head)."""
    fa = cuda_lib
    x = _inputs(1, 32, 8, 8192, 128, True, seed=1304)
    g = to_gpu(x)
    o, lse = _fwd(fa, g)
    args = (g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"], g["block_mask"],
            g["kv_len"])
    dq, dk, dv = fa.bwd(*args)
    _, dk2, dv2 = fa.bwd(*args, deterministic=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    N = 8192
    rows = np.unique(np.concatenate([np.random.default_rng(4).choice(32 * N, 200, replace=False),
                                     [0, N - 1, 31 * N, 32 * N - 1]]))
    rep = lambda t: np.repeat(f64(t), 4, axis=1)
    rq = oracle.attn_bwd_dq_rows(f64(x["q"]), rep(x["k"]), rep(x["v"]), f64(x["do"]), x["scale"],
                                 rows, True)
    got = f64(dq).reshape(-1, 128)[rows]
    scale = np.abs(rq).max()
    assert np.abs(got - rq).max() / scale <= 2e-2
    assert np.abs(got - rq).mean() / scale <= 2e-3


def test_gqa_dkdv_deterministic(cuda_lib):
    g = to_gpu(_inputs(1, 6, 2, 640, 64, True, seed=1303))
    _, _, _, dk1, dv1 = _fb(cuda_lib, g)
    _, _, _, dk2, dv2 = _fb(cuda_lib, g)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)
