"""The d = 128 dK/dV kernel on CTA pairs (tcgen05 cta_group::2, M = 256 keys per pair), through
fa_bwd_deterministic_ex: parity with the FP64 oracle, and dK, dV bit-identical to the
single-CTA dK/dV kernel, which sums every element over the same terms in the same order.
Cases cover an even and an odd number of 128-key tiles (with an odd count the second CTA of the
last pair holds no key at all), causal, key padding, the block mask, grouped/multi-query heads,
a fully masked query block and a batch entry without keys."""
import numpy as np
import pytest
import torch

import oracle
import synthetic as syn
from gpu_util import compare_grad, f64, to_gpu

pytestmark = pytest.mark.gpu


def _bwd_both(fa, g):
    o, lse = fa.fwd(g["q"], g["k"], g["v"], g["scale"], g["causal"], g["block_mask"], g["kv_len"])
    args = (g["q"], g["k"], g["v"], o, lse, g["do"], g["scale"], g["causal"], g["block_mask"],
            g["kv_len"])
    pair = fa.bwd(*args, deterministic=True, dkdv_pair=True)
    single = fa.bwd(*args, deterministic=True, dkdv_pair=False)
    torch.cuda.synchronize()
    assert fa.device_status() == 0
    return pair, single


def _mask(kind, N):
    if kind == "band":
        return syn.block_mask_band_global(N)
    if kind == "hole":  # query block 1 keeps no key block
        nb = (N + 127) // 128
        bm = np.ones((nb, nb), np.uint8)
        bm[1, :] = 0
        return bm
    return None


CASES = [
    # B, H, H_kv, N, causal, kv_len, block mask
    (1, 2, 2, 1000, True, None, None),        # 8 key tiles: 4 full pairs
    (1, 2, 2, 900, False, None, None),
    (2, 1, 1, 640, True, [640, 333], None),   # 5 key tiles: the last pair's odd CTA is past N
    (1, 2, 2, 1100, True, None, "band"),
    (1, 4, 2, 700, True, None, None),         # grouped-query
    (2, 4, 1, 300, False, [300, 77], None),   # multi-query with padding, 3 key tiles
    (1, 1, 1, 129, True, None, None),
    (1, 1, 1, 1, True, None, None),
    (1, 2, 2, 350, False, None, "hole"),      # rows 128..255 see no key
    (2, 2, 2, 300, True, [0, 211], None),     # batch entry 0 has no key
]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_pair_dkdv_parity_and_bit_equality(cuda_lib, case):
    B, H, H_kv, N, causal, L, mk = CASES[case]
    x = syn.make_inputs(B, H, N, 128, "bf16", seed=5100 + case, causal=causal,
                        kv_len=None if L is None else np.array(L, np.int32),
                        block_mask=_mask(mk, N), H_kv=H_kv)
    (dq, dk, dv), (dq1, dk1, dv1) = _bwd_both(cuda_lib, to_gpu(x))
    rq, rk, rv = oracle.attn_bwd_gqa(x["q"], x["k"], x["v"], x["do"], x["scale"], causal,
                                     x["block_mask"], x["kv_len"])
    floor = max(float(np.abs(r).max()) for r in (rq, rk, rv))
    compare_grad(f64(dq), rq, "dQ", floor)
    compare_grad(f64(dk), rk, "dK", floor)
    compare_grad(f64(dv), rv, "dV", floor)
    assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
    assert torch.equal(dq, dq1)
    for t in (dk, dv):
        assert torch.isfinite(t.float()).all()


def test_pair_dkdv_long_causal(cuda_lib):
    """The long-context workload (B1 H16 N16384 d128 causal) in the bench's launch: the pair
    kernel's dK and dV equal the single-CTA kernel's bit for bit over all heads, and sampled key
    rows in every L2 group of heads match the oracle."""
    x = syn.workload_inputs("long_causal")
    (dq, dk, dv), (_, dk1, dv1) = _bwd_both(cuda_lib, to_gpu(x))
    assert torch.equal(dk, dk1) and torch.equal(dv, dv1)
    N, d = x["N"], x["d"]
    rng = np.random.default_rng(5199)
    keys = np.concatenate([h * N + np.unique(np.concatenate([[0, 127, 128, 255, 256, N - 1],
                                                             rng.choice(N, 6, replace=False)]))
                           for h in (0, 7, 9, 15)])
    rk, rv = oracle.attn_bwd_kv_rows(x["q"], x["k"], x["v"], x["do"], x["scale"], keys, True)
    compare_grad(f64(dk).reshape(-1, d)[keys], rk, "dK key rows")
    compare_grad(f64(dv).reshape(-1, d)[keys], rv, "dV key rows")
