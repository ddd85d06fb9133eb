"""The forward softmax's FMA-pipe 2^x: error bound of the algorithm (CPU model) and, on the GPU,
bit equality of the device code with that model and closeness to CUDA's exp2f."""
import numpy as np
import pytest
import torch

from exp2_model import exp2_fma_model

GRID = np.concatenate([np.linspace(-125.0, 8.0, 400001, dtype=np.float32),
                       np.array([0.0, -0.5, 0.5, -1.0, 1.0, 7.999, 8.0, -125.0], np.float32)])


def test_model_relative_error_bound():
    y = exp2_fma_model(GRID).astype(np.float64)
    ref = np.exp2(GRID.astype(np.float64))
    rel = np.abs(y - ref) / ref
    assert rel.max() < 1.1e-4
    assert exp2_fma_model(np.array([0.0], np.float32))[0] == 1.0


def test_model_underflow_is_tiny_and_nonnegative():
    x = np.array([-126.0, -200.0, -np.inf, -1e30], np.float32)
    y = exp2_fma_model(x)
    assert np.all(y >= 0) and np.all(y <= 2.0 ** -125)


@pytest.mark.gpu
def test_device_matches_model_and_exp2f(cuda_lib):
    x = torch.from_numpy(GRID).cuda()
    y_fma, y_mufu, y_ref = (t.cpu().numpy() for t in cuda_lib.diag_exp2(x))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y_fma.view(np.uint32), exp2_fma_model(GRID).view(np.uint32))
    rel = np.abs(y_fma.astype(np.float64) - y_ref) / y_ref
    assert rel.max() < 1.1e-4
    assert (np.abs(y_mufu.astype(np.float64) - y_ref) / y_ref).max() < 1e-5
