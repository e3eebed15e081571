"""tcgen05 GEMM (bf16) and fp32 SIMT GEMM against the oracle's Linear."""

import numpy as np
import pytest

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import dev, host, max_abs, rel_l2

pytestmark = pytest.mark.gpu

SHAPES = [
    (128, 112, 112), (300, 112, 112), (1000, 224, 448), (256, 448, 1792), (130, 16, 64),
    (257, 32, 24), (64, 64, 8), (129, 128, 112), (512, 896, 224), (384, 3584, 896),
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("with_bias,with_resid", [(False, False), (True, True)])
def test_linear_bf16(M, N, K, with_bias, with_resid):
    x = syn.normal(2, 0, (M, K), dtype="bf16")
    w = syn.normal(2, 1, (N, K), 0.05, dtype="bf16")
    b = syn.normal(2, 2, (N,), 0.1, dtype="bf16") if with_bias else None
    r = syn.normal(2, 3, (M, N), dtype="bf16") if with_resid else None
    y = hb.linear(dev(x), dev(w), None if b is None else dev(b), None if r is None else dev(r))
    assert hb.device_status() == 0
    ref = U.linear(x, w, np.zeros(N) if b is None else b)
    if r is not None:
        ref = ref + r
    # inputs exact in bf16; fp32 accumulation, one bf16 rounding of the output
    assert rel_l2(host(y), ref) < 4e-3
    assert max_abs(host(y), ref) <= 1e-2 * max(1.0, np.abs(ref).max())


@pytest.mark.parametrize("M,N,K", [(300, 112, 112), (1000, 224, 448), (97, 50, 33)])
def test_linear_f32(M, N, K):
    x = syn.normal(3, 0, (M, K), dtype="f32")
    w = syn.normal(3, 1, (N, K), 0.05, dtype="f32")
    b = syn.normal(3, 2, (N,), 0.1, dtype="f32")
    r = syn.normal(3, 3, (M, N), dtype="f32")
    y = hb.linear(dev(x, "f32"), dev(w, "f32"), dev(b, "f32"), dev(r, "f32"))
    ref = U.linear(x, w, b) + r
    assert max_abs(host(y), ref) < 1e-4
