"""Deterministic backward on the GPU (fa_bwd_deterministic): dQ from the query-stationary
tensor-core kernel without atomics, dK/dV from the double-buffered dK/dV kernel.  Parity with
the FP64 oracle, bit-identical repeats, and dV (and dK at d = 128) bit-identical to fa_bwd's."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import compare_grad, f64, to_gpu

pytestmark = pytest.mark.gpu


def _run(fa, g, deterministic):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    out = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                 g["block_mask"], g["kv_len"], deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return out


CASES = [
    # B, H, H_kv, N, d, causal, kv_len, block mask
    (2, 2, 2, 700, 64, True, None, False),
    (1, 2, 2, 1000, 128, True, None, False),
    (1, 2, 2, 777, 128, False, None, False),
    (3, 1, 1, 512, 64, False, [130, 512, 301], False),
    (2, 1, 1, 640, 128, True, [640, 333], False),
    (1, 2, 2, 1100, 128, True, None, True),
    (1, 2, 2, 900, 64, False, None, True),
    (1, 1, 1, 129, 128, True, None, False),
    (1, 1, 1, 1, 64, True, None, False),
    (1, 4, 2, 700, 128, True, None, False),     # grouped-query
    (2, 4, 1, 300, 64, False, [300, 77], False),  # multi-query with padding
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_deterministic_backward_parity(cuda_lib, case):
    B, H, H_kv, N, d, causal, L, use_bm = CASES[case]
    x = syn.make_inputs(B, H, N, d, "bf16", seed=1600 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=syn.block_mask_band_global(N) if use_bm else None, H_kv=H_kv)
    g = to_gpu(x)
    dq, dk, dv = _run(cuda_lib, g, True)
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], causal,
                                     x["block_mask"], x["kv_len"])
    floor = max(float(np.abs(r).max()) for r in (rq, rk, rv))
    compare_grad(f64(dq), rq, "dQ", floor)
    compare_grad(f64(dk), rk, "dK", floor)
    compare_grad(f64(dv), rv, "dV", floor)
    # the dK/dV kernel repeats fa_bwd's arithmetic: dV bit for bit; dK too at d = 128, where
    # both keep P in fp32 for dS (fa_bwd's d = 64 kernel reuses the bf16-rounded P there)
    _, dk2, dv2 = _run(cuda_lib, g, False)
    assert torch.equal(dv, dv2)
    if d == 128:
        assert torch.equal(dk, dk2)


def test_deterministic_backward_repeats_bit_identically(cuda_lib):
    x = syn.make_inputs(2, 4, 1500, 128, "bf16", seed=1650, causal=True)
    g = to_gpu(x)
    a = _run(cuda_lib, g, True)
    for _ in range(3):
        b = _run(cuda_lib, g, True)
        for t1, t2 in zip(a, b):
            assert torch.equal(t1, t2)


def test_deterministic_backward_long_causal_sampled(cuda_lib):
    """The long-context workload (B1 H16 N16384 d128 causal) in the launch configuration of the
    bench: dQ of sampled rows against the oracle, two runs bit-identical."""
    x = syn.workload_inputs("long_causal")
    g = to_gpu(x)
    dq, dk, dv = _run(cuda_lib, g, True)
    dq2, dk2, dv2 = _run(cuda_lib, g, True)
    assert torch.equal(dq, dq2) and torch.equal(dk, dk2) and torch.equal(dv, dv2)
    N, H, d = x["N"], x["q"].shape[1], x["d"]
    rows = np.unique(np.concatenate([np.random.default_rng(77).choice(H * N, 150, replace=False),
                                     [0, 127, 128, N - 1, H * N - 1]]))
    rq = oracle.attn_bwd_dq_rows(x["q"], x["k"], x["v"], x["do"], x["scale"], rows, True)
    got = f64(dq).reshape(-1, d)[rows]
    scale = np.abs(rq).max()
    assert np.abs(got - rq).max() / scale <= 2e-2
    assert np.abs(got - rq).mean() / scale <= 2e-3
    assert torch.isfinite(dq.float()).all()
