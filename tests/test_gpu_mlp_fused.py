"""Fused HieraMLP kernel (norm2 + fc1 + GELU + fc2 + residual with the hidden activation
kept on chip) for the dims 112 and 224 ("Phase 4: Hiera Backbone MLX Port", Architecture
Summary: HieraMLP fc1 -> GELU -> fc2, hidden 4 dim).

- Against the fp64 oracle through the block forward (bf16 rel-L2 <= 1e-2, as every block).
- Against the two stand-alone GEMMs (the option switched off): the fused kernel issues the
  same tensor-core K steps per output element and shares the fold / GELU / rounding code,
  so both paths must store the same bf16 values, bit for bit, on a single ragged tile, on
  many persistent tiles per CTA, and through the whole backbone.
"""

import numpy as np
import pytest
import torch

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import TORCH_DT, block_weights_dev, dev, host, rel_l2

pytestmark = pytest.mark.gpu

# name: (B, tokens, d_in, d_out, heads, q_stride, window, mask_unit_attn)
CASES = {
    "d112_one_ragged_tile": (1, 64, 112, 112, 2, 1, 64, True),        # 64 rows < 128
    "d112_windowed": (2, 1024, 112, 112, 2, 1, 64, True),
    "d224_windowed_ragged": (3, 80, 224, 224, 4, 1, 16, True),         # 240 rows
    "d224_transition": (2, 1024, 112, 224, 4, 4, 64, True),
    "d112_many_tiles": (8, 16384, 112, 112, 2, 1, 64, True),         # 1024 tiles
    "d224_many_tiles": (8, 4096, 224, 224, 4, 1, 16, True),          # 256 tiles
}


def _forward(desc, packed, x, fused):
    with hb.fused_mlp(fused):
        y = hb.block_forward(desc, packed, x)
        assert hb.device_status() == 0
    return y


def _setup(name, seed):
    B, tokens, d_in, d_out, heads, qs, window, mua = CASES[name]
    p = syn.block_params(seed, d_in, d_out, d_in != d_out, dtype="bf16", affine="random")
    x = syn.activations(seed, (B, tokens, d_in), dtype="bf16")
    desc = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                        q_stride=qs, window_tokens=window, mask_unit_attn=mua,
                        dtype=torch.bfloat16)
    packed = hb.block_pack(desc, block_weights_dev(p, "bf16"))
    return desc, packed, p, x


@pytest.mark.parametrize("name", list(CASES))
def test_fused_mlp_matches_two_gemms_bitwise(name):
    desc, packed, p, x = _setup(name, 61)
    xd = dev(x, "bf16")
    y_fused = _forward(desc, packed, xd, True)
    y_split = _forward(desc, packed, xd, False)
    assert torch.equal(y_fused, y_split), int((y_fused != y_split).sum())


@pytest.mark.parametrize("name", ["d112_one_ragged_tile", "d112_windowed",
                                  "d224_windowed_ragged", "d224_transition"])
def test_fused_mlp_block_matches_oracle(name):
    desc, packed, p, x = _setup(name, 62)
    y = host(_forward(desc, packed, dev(x, "bf16"), True))
    B, tokens, d_in, d_out, heads, qs, window, mua = CASES[name]
    ref = U.block_forward(x, p, heads, qs, window, mua)
    assert rel_l2(y, ref) <= 1e-2, rel_l2(y, ref)


def test_fused_mlp_backbone_bitwise():
    img, B = 64, 2
    p = syn.backbone_params(63, img, dtype="bf16", affine="random")
    x = dev(syn.image(63, B, img, dtype="bf16"), "bf16")
    desc = hb.BackboneDesc(B=B, img=img)
    w = {"patch_w": dev(p["patch_w"]), "patch_b": dev(p["patch_b"]),
         "pos_embed": dev(p["pos_embed"]),
         "blocks": [{k: dev(v) for k, v in b.items()} for b in p["blocks"]]}
    packed = hb.backbone_pack(desc, w)
    outs = []
    for fused in (True, False):
        with hb.fused_mlp(fused):
            outs.append(hb.backbone_forward(desc, packed, x))
            assert hb.device_status() == 0
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_backbone_same_with_and_without_programmatic_launch():
    """Programmatic dependent launch only changes when kernels start their set-up; every
    kernel still waits for its predecessor, so the features are bit-identical."""
    img, B = 64, 2
    p = syn.backbone_params(64, img, dtype="bf16", affine="random")
    x = dev(syn.image(64, B, img, dtype="bf16"), "bf16")
    desc = hb.BackboneDesc(B=B, img=img)
    w = {"patch_w": dev(p["patch_w"]), "patch_b": dev(p["patch_b"]),
         "pos_embed": dev(p["pos_embed"]),
         "blocks": [{k: dev(v) for k, v in b.items()} for b in p["blocks"]]}
    packed = hb.backbone_pack(desc, w)
    outs = []
    for on in (True, False):
        with hb.pdl(on):
            outs.append(hb.backbone_forward(desc, packed, x))
            assert hb.device_status() == 0
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_option_api():
    assert hb.get_option(hb.OPT_FUSED_MLP) == 1
    assert hb.get_option(hb.OPT_PDL) == 1
    with pytest.raises(hb.HieraError):
        hb.set_option(hb.OPT_FUSED_MLP, 2)
    with pytest.raises(hb.HieraError):
        hb.set_option(7, 1)
    with hb.fused_mlp(False):
        assert hb.get_option(hb.OPT_FUSED_MLP) == 0
    assert hb.get_option(hb.OPT_FUSED_MLP) == 1
