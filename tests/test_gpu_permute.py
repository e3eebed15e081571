"""Unroll / Reroll kernels against the oracle's permutation: bit-exact."""

import numpy as np
import pytest
import torch

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import dev, host

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,G,C,levels", [
    (1, 8, 112, 3), (2, 32, 112, 3), (3, 64, 224, 2), (2, 32, 448, 1), (1, 16, 896, 0),
    (2, 128, 112, 3), (1, 24, 8, 3),
])
def test_unroll_reroll_bit_exact(dtype, B, G, C, levels):
    if dtype == "bf16" and C % 8:
        pytest.skip("bf16 rows must be 16-byte multiples")
    x = syn.normal(1, 0, (B, G * G, C), dtype=dtype)
    xt = dev(x, dtype)
    u = hb.unroll(xt, G, levels)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(u), U.unroll(x.astype(np.float64), G, levels))
    r = hb.reroll(u, G, levels)
    np.testing.assert_array_equal(host(r).reshape(B, G * G, C), x)
    assert hb.device_status() == 0


def test_unroll_full_2048_image_sampled():
    """Stage-0 grid of a 2048^2 image (512^2 tokens, 4096 mask units): sampled tokens."""
    B, G, C = 1, 512, 112
    x = torch.randn(B, G * G, C, device="cuda").to(torch.bfloat16)
    u = hb.unroll(x, G, 3)
    r = hb.reroll(u, G, 3)
    assert torch.equal(r.reshape(B, G * G, C), x)
    idx = U.unroll_index(G, 3).reshape(-1)
    rng = np.random.default_rng(0)
    sel = rng.choice(G * G, 4096, replace=False)
    got = u[0, torch.from_numpy(idx[sel]).cuda()]
    assert torch.equal(got, x[0, torch.from_numpy(sel).cuda()])
