"""The sixteen-epilogue-warp tcgen05 GEMMs for 224-column tiles (one CTA per 128 x 224
tile, or a CTA pair per 256 x 224 tile with tcgen05.mma.cta_group::2) against the
eight-warp kernel and the oracle's Linear ("Phase 4: Hiera Backbone MLX Port", Architecture
Summary: the block's qkv, proj, fc1 and fc2 Linear layers).

All three take every output element's dot product over K in the same 16-wide steps into fp32
accumulators and apply the same epilogue arithmetic, so their outputs are compared bit for
bit; the oracle comparison bounds the shared error (one bf16 rounding of an fp32 sum)."""

import numpy as np
import pytest
import torch

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import dev, host, max_abs, rel_l2

pytestmark = pytest.mark.gpu

# (M, N, K): N a multiple of 224 takes the sixteen-warp kernels. M = 300 leaves the second
# CTA of the pair form's last pair wholly past the last row; M = 1000 ends inside it.
SHAPES = [(256, 448, 1792), (1000, 224, 448), (300, 448, 448), (512, 896, 224),
          (384, 1792, 448), (8192, 448, 448)]


MODES = [hb.GEMM224_SIXTEEN_WARPS, hb.GEMM224_PAIR]


def _linear(x, w, b, r, mode):
    with hb.gemm224(mode):
        y = hb.linear(dev(x), dev(w), None if b is None else dev(b), None if r is None else dev(r))
        torch.cuda.synchronize()
    assert hb.device_status() == 0
    return host(y)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("M,N,K", SHAPES)
def test_wide_gemm_matches_eight_warp_kernel_bitwise_and_oracle(M, N, K, mode):
    x = syn.normal(81, 0, (M, K), dtype="bf16")
    w = syn.normal(81, 1, (N, K), 0.05, dtype="bf16")
    b = syn.normal(81, 2, (N,), 0.1, dtype="bf16")
    r = syn.normal(81, 3, (M, N), dtype="bf16")
    y2 = _linear(x, w, b, r, mode)
    y1 = _linear(x, w, b, r, hb.GEMM224_EIGHT_WARPS)
    assert np.array_equal(y1, y2), np.abs(y1 - y2).max()
    ref = U.linear(x, w, b) + r
    assert rel_l2(y2, ref) < 4e-3
    assert max_abs(y2, ref) <= 1e-2 * max(1.0, np.abs(ref).max())


def _block(desc, w, x, mode, fused_attn=True):
    packed = hb.block_pack(desc, w)
    with hb.gemm224(mode), hb.fused_attention(fused_attn):
        y = hb.block_forward(desc, packed, x)
        torch.cuda.synchronize()
    assert hb.device_status() == 0
    return y.float().cpu().numpy()


# stage-1 plain block (dim 224, qkv / proj / fused MLP), stage-2 global block (dim 448:
# qkv, proj, fc1 + GELU, fc2 with the norm partials they hand on), stage-3 block (dim 896)
BLOCKS = {
    "stage1": dict(B=2, tokens=1024, dim_in=224, dim_out=224, heads=4, q_stride=1,
                   window_tokens=16, mask_unit_attn=True),
    "stage2": dict(B=3, tokens=1024, dim_in=448, dim_out=448, heads=8, q_stride=1,
                   window_tokens=1, mask_unit_attn=False),
    "stage3": dict(B=2, tokens=256, dim_in=896, dim_out=896, heads=16, q_stride=1,
                   window_tokens=1, mask_unit_attn=False),
}


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("name", sorted(BLOCKS))
def test_wide_gemm_block_bitwise(name, mode):
    cfg = BLOCKS[name]
    desc = hb.BlockDesc(**cfg)
    p = syn.block_params(84, cfg["dim_in"], cfg["dim_out"], False, dtype="bf16")
    w = {k: torch.from_numpy(v).to("cuda", torch.bfloat16) for k, v in p.items()}
    x = torch.from_numpy(syn.activations(84, (cfg["B"], cfg["tokens"], cfg["dim_in"]))).to(
        "cuda", torch.bfloat16)
    a = _block(desc, w, x, mode)
    b = _block(desc, w, x, hb.GEMM224_EIGHT_WARPS)
    assert np.isfinite(a).all()
    assert np.array_equal(a, b), np.abs(a - b).max()


@pytest.mark.parametrize("mode", MODES)
def test_wide_gemm_backbone_bitwise(mode):
    img, B = 256, 2
    p = syn.backbone_params(85, img, dtype="bf16", affine="random")
    x = dev(syn.image(85, B, img, dtype="bf16"), "bf16")
    desc = hb.BackboneDesc(B=B, img=img)
    w = {"patch_w": dev(p["patch_w"]), "patch_b": dev(p["patch_b"]),
         "pos_embed": dev(p["pos_embed"]),
         "blocks": [{k: dev(v) for k, v in b.items()} for b in p["blocks"]]}
    packed = hb.backbone_pack(desc, w)
    outs = []
    for m in (mode, hb.GEMM224_EIGHT_WARPS):
        with hb.gemm224(m):
            outs.append(hb.backbone_forward(desc, packed, x))
            torch.cuda.synchronize()
            assert hb.device_status() == 0
    for a, b in zip(*outs):
        assert torch.isfinite(a.float()).all()
        assert torch.equal(a, b)
