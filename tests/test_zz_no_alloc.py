"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers cannot pass fa_bwd a workspace: a plugin that a host framework hands only its input
and output buffers (the framework owns every device allocation), or code that must not call
cudaMalloc / cudaFree because those calls can synchronise the whole device.  fa_bwd_noalloc runs
fa_bwd's kernels on the library's own fixed 32 MiB scratch instead.

Each case calls it through the C ABI twice in a row, after a larger call has left the scratch
full of another problem's values, and checks
  * every gradient against the FP64 oracle within the parity tolerance (max 2e-2 and mean 2e-3
    relative to max |reference|), and
  * against fa_bwd with a caller-provided workspace: dK and dV bit for bit (both calls run the
    same deterministic key-stationary sums), and dQ bit for bit on the fp32 path; the bf16 dQ
    adds its key tiles' contributions in an order that varies, so it is held to the tolerance.
A partial leak of the previous call's scratch would break the bit equalities.
This file is collected last on purpose; it passes on its own in a fresh process as well as
after the other tests.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_98_b200 as fa
import oracle
import synthetic as syn
from gpu_util import compare_grad, f64, to_gpu

CASES = [
    # B, H, N, d, causal, kv_len, block mask, dtype
    (2, 3, 700, 64, True, None, False, "bf16"),
    (1, 2, 1000, 128, False, [1000], False, "bf16"),
    (3, 2, 512, 64, False, [130, 512, 301], True, "bf16"),
    (1, 2, 300, 100, True, None, False, "f32"),  # the fp32 backward on the same scratch
]


def _dirty_scratch(lib):
    """A larger backward (B4 H4 N2048 d128 needs ~16.1 MiB of scratch) through the same entry
    point, so that the checked calls start from another problem's leftovers."""
    x = to_gpu(syn.make_inputs(4, 4, 2048, 128, "bf16", seed=3199, causal=False))
    o, lse = lib.fwd(x["q"], x["k"], x["v"], x["scale"])
    lib.bwd_noalloc(x["q"], x["k"], x["v"], o, lse, x["do"], x["scale"])
    torch.cuda.synchronize()
    assert lib.device_status() == 0


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_oracle_and_workspace_backward(cuda_lib, case):
    B, H, N, d, causal, L, use_bm, dt = CASES[case]
    x = syn.make_inputs(B, H, N, d, dt, seed=3100 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=syn.block_mask_band_global(N) if use_bm else None)
    g = to_gpu(x)
    kw = dict(scale=g["scale"], causal=g["causal"], block_mask=g["block_mask"],
              kv_len=g["kv_len"])
    o, lse = cuda_lib.fwd(g["q"], g["k"], g["v"], **kw)
    ws_dq, ws_dk, ws_dv = cuda_lib.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
    torch.cuda.synchronize()
    ref = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], causal, x["block_mask"],
                          x["kv_len"])
    _dirty_scratch(cuda_lib)
    for _ in range(2):  # the second call runs on the scratch the first one left behind
        dq, dk, dv = cuda_lib.bwd_noalloc(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
        torch.cuda.synchronize()
        assert cuda_lib.device_status() == 0
        for name, got, r in zip(("dQ", "dK", "dV"), (dq, dk, dv), ref):
            if dt == "f32":
                err = np.abs(f64(got) - r).max() / max(np.abs(r).max(), 1e-30)
                assert err <= 1e-5, f"{name} fp32 max rel err {err:.3e}"
            else:
                compare_grad(f64(got), r, name)
        assert torch.equal(dk, ws_dk) and torch.equal(dv, ws_dv)
        if dt == "f32":
            assert torch.equal(dq, ws_dq)
        else:
            compare_grad(f64(dq), f64(ws_dq), "dQ vs fa_bwd")


@pytest.mark.gpu
def test_noalloc_binding_rejects_mismatched_buffers(cuda_lib):
    """The binding refuses what the C entry point cannot describe (grouped K/V heads) and
    buffers whose shapes differ from q's, before anything reaches the GPU."""
    x = to_gpu(syn.make_inputs(1, 4, 256, 64, "bf16", seed=3190, H_kv=2))
    o = torch.zeros_like(x["q"])
    lse = torch.zeros((1, 4, 256), dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FaError):
        cuda_lib.bwd_noalloc(x["q"], x["k"], x["v"], o, lse, x["do"])
    y = to_gpu(syn.make_inputs(1, 4, 256, 64, "bf16", seed=3191))
    with pytest.raises(fa.FaError):
        cuda_lib.bwd_noalloc(y["q"], y["k"], y["v"], o, lse[:, :2], y["do"])
    with pytest.raises(fa.FaError):
        cuda_lib.bwd_noalloc(y["q"], y["k"], y["v"], o, lse, y["do"],
                             dk=torch.empty((1, 2, 256, 64), dtype=torch.bfloat16, device="cuda"))


def test_noalloc_rejects_problems_larger_than_its_scratch():
    """B1 H16 N16384 d128 needs ~136 MB of scratch; the call refuses before touching the GPU."""
    lib = fa.load()
    A = 0x100000  # aligned fake address: the size check returns before any device access
    rc = lib.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 16, 16384, 128, 0.0883883, 1, None,
                            None, 0, None)
    assert rc == -6
    msg = lib.fa_get_last_error().decode()
    assert "scratch" in msg and str(32 << 20) in msg
