"""Backward parity on the GPU: dQ, dK, dV from the CUDA path (forward + backward through the
C ABI) against the FP64 oracle's explicit derivative, relative to max |reference|."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import compare_grad, f64, oracle_bwd, to_gpu

pytestmark = pytest.mark.gpu


def run_fb(fa, g):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                        g["block_mask"], g["kv_len"])
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return dq, dk, dv


SMALL = [
    # B, H, N, d, causal, kv_len, block mask
    (2, 2, 700, 64, False, None, False),
    (2, 2, 700, 64, True, None, False),
    (1, 2, 1000, 128, True, None, False),
    (1, 2, 777, 128, False, None, False),
    (3, 1, 512, 64, False, [130, 512, 301], False),
    (2, 1, 640, 128, True, [640, 333], False),
    (1, 2, 900, 64, False, None, True),
    (1, 2, 1100, 128, True, None, True),
    (1, 1, 8, 64, False, None, False),
    (1, 1, 129, 128, True, None, False),
    (1, 1, 1, 64, True, None, False),
    (2, 1, 3, 128, False, [2, 3], False),
    (1, 2, 257, 64, True, [200], True),
    (2, 1, 390, 128, True, [390, 260], True),
]


@pytest.mark.parametrize("case", range(len(SMALL)))
def test_bwd_small_elementwise(cuda_lib, case):
    B, H, N, d, causal, L, use_bm = SMALL[case]
    x = syn.make_inputs(B, H, N, d, "bf16", seed=900 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=syn.block_mask_band_global(N) if use_bm else None)
    dq, dk, dv = run_fb(cuda_lib, to_gpu(x))
    rq, rk, rv = oracle_bwd(x)
    floor = max(float(np.abs(r).max()) for r in (rq, rk, rv))
    compare_grad(f64(dq), rq, "dQ", floor)
    compare_grad(f64(dk), rk, "dK", floor)
    compare_grad(f64(dv), rv, "dV", floor)
    if L is not None:
        for b, Lb in enumerate(L):
            assert torch.all(dk[b, :, Lb:] == 0) and torch.all(dv[b, :, Lb:] == 0)


WORKLOAD_HEADS = {
    "gpt2_causal": [0, 13, 50, 95],
    "bert_padding": [0, 17, 100, 255],
    "block_sparse": [0, 3, 7, 12, 16, 21, 26, 31],   # both batch entries, 8 of 32 heads
    "long_causal": [0],
}


@pytest.mark.parametrize("name", list(WORKLOAD_HEADS))
def test_bwd_workload_heads(cuda_lib, name):
    """Full-size launch; the oracle differentiates a subset of heads in full."""
    x = syn.workload_inputs(name)
    dq, dk, dv = run_fb(cuda_lib, to_gpu(x))
    heads = WORKLOAD_HEADS[name]
    rq, rk, rv = oracle_bwd(x, heads=heads)
    B, H, N, d = x["q"].shape
    for h in heads:
        b, hh = divmod(h, H)
        compare_grad(f64(dq[b, hh]), rq[b, hh], f"dQ[{h}]")
        compare_grad(f64(dk[b, hh]), rk[b, hh], f"dK[{h}]")
        compare_grad(f64(dv[b, hh]), rv[b, hh], f"dV[{h}]")
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


def test_bwd_dkdv_deterministic(cuda_lib):
    x = to_gpu(syn.make_inputs(1, 2, 640, 64, "bf16", seed=5, causal=True))
    _, dk1, dv1 = run_fb(cuda_lib, x)
    _, dk2, dv2 = run_fb(cuda_lib, x)
    assert torch.equal(dk1, dk2) and torch.equal(dv1, dv2)


@pytest.mark.parametrize("name", ["gpt2_causal", "bert_padding"])
def test_bwd_overlapped_launches(cuda_lib, name):
    """At d = 64 the main backward kernel is launched to start under the preprocess kernel's tail,
    and the dQ convert under the main kernel's.  The workspace is filled with 0x7f bytes
    (~3.4e38 as fp32) before each of 12 back-to-back calls, so a read of lse2, Dvec or the dQ
    accumulator before the kernel that writes it had finished would give wrong or non-finite
    gradients: every call's dK and dV equal the first call's bit for bit, dQ agrees to within
    the rounding of its atomic sums, and the last call matches the oracle on one head."""
    fa = cuda_lib
    x = syn.workload_inputs(name)
    g = to_gpu(x)
    B, H, N, d = x["q"].shape
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    ws = torch.empty(fa.bwd_workspace_size(B, H, N, d), dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(12):
        ws.fill_(0x7f)
        outs.append(fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                           g["block_mask"], g["kv_len"], workspace=ws))
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    dq0, dk0, dv0 = outs[0]
    top = float(dq0.float().abs().max())
    for dq, dk, dv in outs:
        assert torch.isfinite(dq.float()).all()
        assert torch.equal(dk, dk0) and torch.equal(dv, dv0)
        assert float((dq.float() - dq0.float()).abs().max()) <= 1e-2 * top
    rq, rk, rv = oracle_bwd(x, heads=[0])
    dq, dk, dv = outs[-1]
    compare_grad(f64(dq[0, 0]), rq[0, 0], "dQ[0]")
    compare_grad(f64(dk[0, 0]), rk[0, 0], "dK[0]")
    compare_grad(f64(dv[0, 0]), rv[0, 0], "dV[0]")


def test_bwd_long_causal_all_heads(cuda_lib):
    """The long-context workload (B1 H16 N16384 d128 causal) in the bench's launch: its CTAs run
    in several L2-sized groups of heads and dQ is added by TMA reduce-adds.  Every head's dK and
    dV equal the deterministic backward's bit for bit (the same key-stationary sums), and dQ rows
    sampled over all heads match the oracle."""
    fa = cuda_lib
    x = syn.workload_inputs("long_causal")
    g = to_gpu(x)
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    args = (g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"], g["block_mask"],
            g["kv_len"])
    dq, dk, dv = fa.bwd(*args)
    _, dk2, dv2 = fa.bwd(*args, deterministic=True)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    assert torch.equal(dk, dk2) and torch.equal(dv, dv2)
    N, H, d = x["N"], x["q"].shape[1], x["d"]
    rows = np.unique(np.concatenate([np.random.default_rng(78).choice(H * N, 240, replace=False),
                                     [0, 63, 64, N - 1, N, H * N - 64, H * N - 1]]))
    rq = oracle.attn_bwd_dq_rows(x["q"], x["k"], x["v"], x["do"], x["scale"], rows, True)
    got = f64(dq).reshape(-1, d)[rows]
    scale = np.abs(rq).max()
    assert np.abs(got - rq).max() / scale <= 2e-2
    assert np.abs(got - rq).mean() / scale <= 2e-3
    assert torch.isfinite(dq.float()).all()
    # dK and dV of key rows in one head of every L2-sized group of heads (the CTAs run 4 heads at
    # a time here), against the oracle's definition: edge keys of the first, middle and last KV
    # tiles plus random keys
    rng = np.random.default_rng(79)
    keys = []
    for h in (0, 5, 10, 15):
        js = np.concatenate([[0, 1, 127, 128, N // 2, N - 129, N - 128, N - 1],
                             rng.choice(N, 8, replace=False)])
        keys.append(h * N + np.unique(js))
    keys = np.concatenate(keys)
    rk, rv = oracle.attn_bwd_kv_rows(x["q"], x["k"], x["v"], x["do"], x["scale"], keys, True)
    compare_grad(f64(dk).reshape(-1, d)[keys], rk, "dK key rows")
    compare_grad(f64(dv).reshape(-1, d)[keys], rv, "dV key rows")
