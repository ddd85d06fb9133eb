"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device memory.

Such callers (a plugin that is handed only its input and output buffers by a host framework
that owns all device memory, or code that must not call cudaMalloc/cudaFree because those can
synchronise the device) cannot pass fa_bwd a workspace.  fa_bwd_noalloc uses the library's own
fixed 32 MiB scratch instead.  These tests call it through the C ABI and check that two calls
in a row give the same gradients as fa_bwd with a caller-provided workspace, within the
gradient tolerance the parity tests use (max 2e-2 and mean 2e-3 relative to max |reference|).
This file is collected last on purpose, and it passes on its own in a fresh process as well as
after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_io_aware_98_b200 as fa
import synthetic as syn
from gpu_util import compare_grad, f64, to_gpu

CASES = [
    # B, H, N, d, causal, kv_len, block mask, dtype
    (2, 3, 700, 64, True, None, False, "bf16"),
    (1, 2, 1000, 128, False, [1000], False, "bf16"),
    (3, 2, 512, 64, False, [130, 512, 301], True, "bf16"),
    (1, 2, 300, 100, True, None, False, "f32"),  # the fp32 backward on the same scratch
]


@pytest.mark.gpu
@pytest.mark.parametrize("case", range(len(CASES)))
def test_noalloc_matches_workspace_backward(cuda_lib, case):
    B, H, N, d, causal, L, use_bm, dt = CASES[case]
    x = syn.make_inputs(B, H, N, d, dt, seed=3100 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=syn.block_mask_band_global(N) if use_bm else None)
    g = to_gpu(x)
    kw = dict(scale=g["scale"], causal=g["causal"], block_mask=g["block_mask"],
              kv_len=g["kv_len"])
    o, lse = cuda_lib.fwd(g["q"], g["k"], g["v"], **kw)
    ref = cuda_lib.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
    torch.cuda.synchronize()
    ref = [f64(t) for t in ref]
    for _ in range(2):  # the second call runs on the scratch the first one left behind
        got = cuda_lib.bwd_noalloc(g["q"], g["k"], g["v"], o, lse, g["do"], **kw)
        torch.cuda.synchronize()
        assert cuda_lib.device_status() == 0
        for name, a, b in zip(("dQ", "dK", "dV"), got, ref):
            compare_grad(f64(a), b, name)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    """B1 H16 N16384 d128 needs ~136 MB of scratch; the call refuses before touching the GPU."""
    lib = fa.load()
    A = 0x100000  # aligned fake address: the size check returns before any device access
    rc = lib.fa_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 16, 16384, 128, 0.0883883, 1, None,
                            None, 0, None)
    assert rc == -6
    msg = lib.fa_get_last_error().decode()
    assert "scratch" in msg and str(32 << 20) in msg
