"""fp32 backward on the GPU (CUDA-core kernels through fa_bwd with FA_F32) against the FP64
oracle: dQ, dK, dV within 1e-5 of max |reference|, and bit-identical across runs."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import f64, to_gpu

pytestmark = pytest.mark.gpu

F32_GRAD = 1e-5


def _fb(fa, g):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                        g["block_mask"], g["kv_len"])
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return dq, dk, dv


def _close(got, ref, name, floor=0.0):
    # relative to max|ref|.  With a single visible key dQ and dK vanish identically (dS = P
    # (dP - Dvec) = 0 in exact arithmetic) while dP and Dvec do not, so their fp32 difference
    # leaves rounding of the size of dP; such a reference is measured against ``floor``, the
    # largest reference gradient of the same call.
    scale = max(np.abs(ref).max(), floor, 1e-30)
    err = np.abs(got - ref).max() / scale
    assert err <= F32_GRAD, f"{name}: max err {err:.3e} of max|ref|"


CASES = [
    # B, H, H_kv, N, d, causal, kv_len, block mask
    (1, 1, 1, 128, 64, False, None, False),     # the fp32 single-head workload's shape
    (2, 2, 2, 300, 100, True, None, False),
    (1, 2, 2, 257, 7, False, None, False),
    (2, 2, 2, 400, 128, False, [400, 211], False),
    (1, 2, 2, 390, 64, False, None, True),
    (1, 4, 2, 200, 64, True, None, False),       # grouped-query
    (1, 1, 1, 1, 32, True, None, False),
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_f32_backward(cuda_lib, case):
    B, H, H_kv, N, d, causal, L, use_bm = CASES[case]
    x = syn.make_inputs(B, H, N, d, "f32", seed=1500 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=syn.block_mask_band_global(N) if use_bm else None,
                        H_kv=H_kv)
    dq, dk, dv = _fb(cuda_lib, to_gpu(x))
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], causal,
                                     x["block_mask"], x["kv_len"])
    top = max(np.abs(r).max() for r in (rq, rk, rv))
    _close(f64(dq), rq, "dQ", top if N == 1 else 0.0)
    _close(f64(dk), rk, "dK", top if N == 1 else 0.0)
    _close(f64(dv), rv, "dV")


def test_f32_workload_backward_and_determinism(cuda_lib):
    x = syn.workload_inputs("fp32_single_head", with_grad=True)
    g = to_gpu(x)
    a = _fb(cuda_lib, g)
    b = _fb(cuda_lib, g)
    for t1, t2 in zip(a, b):
        assert torch.equal(t1, t2)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], False)
    _close(f64(a[0]), rq, "dQ")
    _close(f64(a[1]), rk, "dK")
    _close(f64(a[2]), rv, "dV")
