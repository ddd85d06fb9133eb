"""Failure detection on the device without faulting it: a bounded mbarrier wait that nothing
satisfies gives up, records where, and the host reads FA_ERR_TIMEOUT; the context stays usable."""
import pytest
import torch

import synthetic as syn
from gpu_util import compare_o, f64, oracle_fwd, to_gpu

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    assert cuda_lib.device_status() == 0
    cuda_lib.diag_wait_timeout(1234)
    code = cuda_lib.device_status()
    assert code >> 16 == 1234
    assert cuda_lib.device_status() == 0           # reading clears it
    # the device still runs attention correctly afterwards
    x = syn.make_inputs(1, 2, 300, 64, "bf16", seed=8, causal=True, with_grad=False)
    g = to_gpu(x)
    o, lse = cuda_lib.fwd(g["q"], g["k"], g["v"], g["scale"], True)
    torch.cuda.synchronize()
    assert cuda_lib.device_status() == 0
    compare_o(f64(o), oracle_fwd(x)[0])
