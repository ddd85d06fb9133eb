"""Bit-level CPU model of the forward softmax's FMA-pipe 2^x (test helper).

Each step is one IEEE float32 operation with round-to-nearest-even, as on the device:
fused multiply-adds are evaluated exactly in float64 and rounded once to float32.
"""
import numpy as np

ROUND = np.float32(12582912.0)     # 1.5 * 2^23
C1, C2, C3 = np.float32(0.6932829), np.float32(0.24221037), np.float32(0.05500858)


def _fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_fma_model(x: np.ndarray) -> np.ndarray:
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    j = (x + ROUND).astype(np.float32)
    n = (j - ROUND).astype(np.float32)
    f = _fma(n, np.float32(-1.0), x)
    p = _fma(np.full_like(f, C3), f, np.full_like(f, C2))
    p = _fma(p, f, np.full_like(f, C1))
    p = _fma(p, f, np.full_like(f, 1.0))
    bits = (p.view(np.uint32).astype(np.uint64) + (j.view(np.uint32).astype(np.uint64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)
