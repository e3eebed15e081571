"""Patch embedding + pos_embed + Unroll through the C ABI against the fp64 oracle
("Phase 4: Hiera Backbone MLX Port", Architecture Summary: Conv2d(4 -> 112, 7x7,
stride 4, padding 3), a learned pos_embed added in raster order, then Unroll).

Element by element on every output:
- fp32: |got - ref| <= 1e-5 (fp32 accumulation of 196 products of magnitude <= 0.1);
- bf16: the kernel accumulates exact bf16 products in fp32 and rounds once, so
  |got - ref| <= 2^-8 |ref| + 1e-5 (one rounding to 8 significant bits plus the fp32 sum).
Sizes: 64^2 (one 16-pixel-wide grid), 224^2 (56-pixel grid: a ragged 128-pixel segment and
a ragged 4-row band), 512^2 (the backbone workload's grid, two images).
"""

import numpy as np
import pytest

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import dev, host

pytestmark = pytest.mark.gpu


def _reference(x, p, img):
    G = img // 4
    tok = U.patch_embed(x, p["patch_w"], p["patch_b"]) + np.asarray(p["pos_embed"], np.float64)[None]
    return U.unroll(tok, G, 3)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("img,B", [(64, 2), (224, 1), (512, 2)])
def test_patch_embed_matches_oracle(dtype, img, B):
    p = syn.backbone_params(41, img, dtype=dtype, affine="random")
    x = syn.image(41, B, img, dtype=dtype)
    packed = hb.patch_pack(dev(p["patch_w"], dtype), dev(p["patch_b"], dtype))
    got = host(hb.patch_embed(dev(x, dtype), packed, dev(p["pos_embed"], dtype)))
    assert hb.device_status() == 0
    ref = _reference(x, p, img)
    assert got.shape == ref.shape
    err = np.abs(got - ref)
    if dtype == "f32":
        assert err.max() <= 1e-5, err.max()
    else:
        bound = 2.0 ** -8 * np.abs(ref) + 1e-5
        worst = np.unravel_index(np.argmax(err - bound), err.shape)
        assert np.all(err <= bound), (worst, got[worst], ref[worst])


def test_patch_embed_bias_null_is_zero():
    """A NULL bias packs as zeros: same output as an explicit zero bias."""
    img, B = 64, 1
    p = syn.backbone_params(42, img, dtype="bf16", affine="random")
    x = dev(syn.image(42, B, img, dtype="bf16"), "bf16")
    w = dev(p["patch_w"], "bf16")
    pos = dev(p["pos_embed"], "bf16")
    a = host(hb.patch_embed(x, hb.patch_pack(w, None), pos))
    b = host(hb.patch_embed(x, hb.patch_pack(w, dev(np.zeros(112), "bf16")), pos))
    assert np.array_equal(a, b)
