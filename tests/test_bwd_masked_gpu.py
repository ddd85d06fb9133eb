"""Backward parity on the GPU for rows that see no key at all.

"Attention optimisation: FlashAttention and sparse attention" (mdooai Ch.04, sparse-masking
paragraph) sets the logit of every key outside a row's allowed set to -inf before the softmax.
A row whose allowed set is empty then has no softmax weights: O = 0, lse = -inf, and it takes no
part in any gradient (dQ of the row is 0 and it adds nothing to dK or dV).  These cases make such
rows with a block mask that removes a whole query block (alone and together with the causal
mask) and with a batch entry whose key length is 0, and run them through every backward entry
point: fa_bwd, fa_bwd_deterministic and fa_bwd_gqa, at d = 64 and 128."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import compare_grad, compare_lse, compare_o, f64, to_gpu

pytestmark = pytest.mark.gpu

MODES = {
    # name: (H, H_kv, deterministic)
    "fa_bwd": (2, 2, False),
    "fa_bwd_deterministic": (2, 2, True),
    "fa_bwd_gqa": (4, 2, False),
    "fa_bwd_deterministic_gqa": (4, 2, True),
}


def _run(fa, g, deterministic):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    dq, dk, dv = fa.bwd(g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"],
                        g["block_mask"], g["kv_len"], deterministic=deterministic)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return o, lse, dq, dk, dv


def _check_against_oracle(x, o, lse, dq, dk, dv):
    o_ref, lse_ref = oracle.attn_fwd_gqa(x["q"], x["k"], x["v"], x["scale"], x["causal"],
                                         x["block_mask"], x["kv_len"])
    compare_o(f64(o), o_ref)
    compare_lse(f64(lse), lse_ref)
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], x["causal"],
                                     x["block_mask"], x["kv_len"])
    compare_grad(f64(dq), rq, "dQ")
    compare_grad(f64(dk), rk, "dK")
    compare_grad(f64(dv), rv, "dV")
    return lse_ref


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_fully_masked_query_block(cuda_lib, mode, d, causal):
    """N = 350 (three query blocks, the last ragged); query block 1 keeps no key block, so rows
    128..255 see nothing; block (2, 0) is removed as well so the mask is not symmetric."""
    H, H_kv, det = MODES[mode]
    N = 350
    bm = np.ones((3, 3), np.uint8)
    bm[1, :] = 0
    bm[2, 0] = 0
    x = syn.make_inputs(1, H, N, d, "bf16", seed=4100 + d + (7 if causal else 0), causal=causal,
                        block_mask=bm, H_kv=H_kv)
    o, lse, dq, dk, dv = _run(cuda_lib, to_gpu(x), det)
    lse_ref = _check_against_oracle(x, o, lse, dq, dk, dv)
    assert np.all(np.isneginf(lse_ref[:, :, 128:256]))
    assert torch.all(o[:, :, 128:256] == 0)
    assert torch.all(torch.isneginf(lse[:, :, 128:256]))
    assert torch.all(dq[:, :, 128:256] == 0)
    for t in (dq, dk, dv):
        assert torch.isfinite(t.float()).all()


@pytest.mark.parametrize("mode", list(MODES))
@pytest.mark.parametrize("d", [64, 128])
def test_bwd_batch_entry_without_keys(cuda_lib, mode, d):
    """Key length 0 for batch entry 0 (every row of it sees nothing), a ragged length for entry
    1: entry 0 gets O = 0, lse = -inf and all-zero gradients; entry 1 matches the oracle."""
    H, H_kv, det = MODES[mode]
    N = 300
    x = syn.make_inputs(2, H, N, d, "bf16", seed=4200 + d, causal=True,
                        kv_len=np.array([0, 211], np.int32), H_kv=H_kv)
    o, lse, dq, dk, dv = _run(cuda_lib, to_gpu(x), det)
    _check_against_oracle(x, o, lse, dq, dk, dv)
    assert torch.all(o[0] == 0) and torch.all(torch.isneginf(lse[0]))
    for t in (dq, dk, dv):
        assert torch.all(t[0] == 0)
    assert torch.all(dk[1, :, 211:] == 0) and torch.all(dv[1, :, 211:] == 0)


def test_bwd_f32_fully_masked_rows(cuda_lib):
    """The fp32 backward: the same masked query block, every gradient within 1e-5 of the
    oracle relative to its largest magnitude, and the masked rows' dQ exactly 0."""
    N, d = 300, 48
    bm = np.ones((3, 3), np.uint8)
    bm[1, :] = 0
    x = syn.make_inputs(1, 2, N, d, "f32", seed=4300, causal=True, block_mask=bm)
    o, lse, dq, dk, dv = _run(cuda_lib, to_gpu(x), False)
    rq, rk, rv = oracle.attn_bwd(x["q"], x["k"], x["v"], x["do"], x["scale"], True, bm)
    for got, ref in ((dq, rq), (dk, rk), (dv, rv)):
        err = np.abs(f64(got) - ref).max() / np.abs(ref).max()
        assert err <= 1e-5
    assert torch.all(dq[:, :, 128:256] == 0)
