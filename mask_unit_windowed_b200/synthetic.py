"""Seeded synthetic inputs and random-init weights for the Hiera block and backbone.

This module only draws numbers: it holds none of the block's arithmetic. Both the
CUDA path (through the binding) and the CPU oracle consume exactly the arrays made
here, so every parity comparison starts from identical values.

Recipe (the configurations the Hiera-B+ backbone is measured on):
  * activations ~ N(0, 1), images ~ U(-1, 1);
  * Linear weights ~ N(0, 0.02), biases 0, LayerNorm gamma = 1 and beta = 0
    (``affine="init"``);
  * parity tests use ``affine="random"`` instead, which draws non-trivial
    gamma ~ 1 + N(0, 0.1), beta ~ N(0, 0.1) and biases ~ N(0, 0.02) so that
    every affine term is exercised;
  * pos_embed ~ N(0, 0.02);
  * in bf16 mode every array is rounded to the nearest bf16 value (ties to even)
    and returned as float32 holding that exact bf16 value.

Each tensor has its own stream: numpy's PCG64 seeded with (seed, tensor id).
"""

from __future__ import annotations

import numpy as np

BF16 = "bf16"
F32 = "f32"

# Hiera-B+ stage table as the "Phase 4: Hiera Backbone MLX Port" plan lists it
# (Architecture Summary): blocks per stage, dim, heads; the mask-unit window is 8x8
# tokens at stage 0 and shrinks 4x per pooled stage.
STAGE_DEPTHS = (2, 3, 16, 3)
STAGE_DIMS = (112, 224, 448, 896)
STAGE_HEADS = (2, 4, 8, 16)
HEAD_DIM = 56
MLP_RATIO = 4
PATCH_KERNEL = 7
PATCH_STRIDE = 4
PATCH_PAD = 3
IN_CHANS = 4


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); float32 out."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.uint64)
    lsb = (bits >> np.uint64(16)) & np.uint64(1)
    rounded = (bits + np.uint64(0x7FFF) + lsb) & np.uint64(0xFFFF0000)
    return rounded.astype(np.uint32).view(np.float32).reshape(a.shape)


def _finish(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    if dtype == BF16:
        a = round_to_bf16(a)
    elif dtype != F32:
        raise ValueError(f"unknown dtype {dtype!r}")
    return np.ascontiguousarray(a)


def normal(seed: int, tensor_id: int, shape, std: float = 1.0, mean: float = 0.0,
           dtype: str = F32) -> np.ndarray:
    rng = np.random.default_rng([int(seed), int(tensor_id)])
    return _finish(mean + std * rng.standard_normal(shape, dtype=np.float64), dtype)


def uniform(seed: int, tensor_id: int, shape, lo: float = -1.0, hi: float = 1.0,
            dtype: str = F32) -> np.ndarray:
    rng = np.random.default_rng([int(seed), int(tensor_id)])
    return _finish(rng.uniform(lo, hi, size=shape), dtype)


def block_shapes(dim_in: int, dim_out: int, transition: bool) -> dict:
    """Weight shapes of one block, Linear weights stored [out, in]."""
    hidden = MLP_RATIO * dim_out
    shapes = {
        "norm1_w": (dim_in,), "norm1_b": (dim_in,),
        "qkv_w": (3 * dim_out, dim_in), "qkv_b": (3 * dim_out,),
        "attn_proj_w": (dim_out, dim_out), "attn_proj_b": (dim_out,),
        "norm2_w": (dim_out,), "norm2_b": (dim_out,),
        "fc1_w": (hidden, dim_out), "fc1_b": (hidden,),
        "fc2_w": (dim_out, hidden), "fc2_b": (dim_out,),
    }
    if transition:
        shapes["proj_w"] = (dim_out, dim_in)
        shapes["proj_b"] = (dim_out,)
    return shapes


_TENSOR_IDS = {name: i for i, name in enumerate([
    "norm1_w", "norm1_b", "qkv_w", "qkv_b", "proj_w", "proj_b", "attn_proj_w",
    "attn_proj_b", "norm2_w", "norm2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b"])}


def block_params(seed: int, dim_in: int, dim_out: int, transition: bool,
                 dtype: str = BF16, affine: str = "init", base_id: int = 0) -> dict:
    """Random-init weights of one block as float32 arrays (bf16-exact in bf16 mode)."""
    out = {}
    for name, shape in block_shapes(dim_in, dim_out, transition).items():
        tid = base_id + _TENSOR_IDS[name]
        is_ln_w = name in ("norm1_w", "norm2_w")
        is_ln_b = name in ("norm1_b", "norm2_b")
        if name.endswith("_w") and not is_ln_w:
            out[name] = normal(seed, tid, shape, 0.02, dtype=dtype)
        elif affine == "init":
            out[name] = _finish(np.ones(shape) if is_ln_w else np.zeros(shape), dtype)
        elif affine == "random":
            if is_ln_w:
                out[name] = normal(seed, tid, shape, 0.1, mean=1.0, dtype=dtype)
            elif is_ln_b:
                out[name] = normal(seed, tid, shape, 0.1, dtype=dtype)
            else:
                out[name] = normal(seed, tid, shape, 0.02, dtype=dtype)
        else:
            raise ValueError(f"unknown affine mode {affine!r}")
    return out


def backbone_block_table():
    """Per-block (dim_in, dim_out, heads, stage, transition) for Hiera-B+."""
    table = []
    prev_dim = STAGE_DIMS[0]
    for s, depth in enumerate(STAGE_DEPTHS):
        for i in range(depth):
            transition = s > 0 and i == 0
            dim_in = prev_dim if transition else STAGE_DIMS[s]
            table.append((dim_in, STAGE_DIMS[s], STAGE_HEADS[s], s, transition))
        prev_dim = STAGE_DIMS[s]
    return table


def backbone_params(seed: int, img: int, dtype: str = BF16, affine: str = "init") -> dict:
    """Patch-embed, pos_embed and 24 blocks of random-init weights."""
    g0 = img // PATCH_STRIDE
    p = {
        "patch_w": normal(seed, 1000, (STAGE_DIMS[0], PATCH_KERNEL, PATCH_KERNEL, IN_CHANS),
                          0.02, dtype=dtype),
        "patch_b": (normal(seed, 1001, (STAGE_DIMS[0],), 0.02, dtype=dtype) if affine == "random"
                    else _finish(np.zeros(STAGE_DIMS[0]), dtype)),
        "pos_embed": normal(seed, 1002, (g0 * g0, STAGE_DIMS[0]), 0.02, dtype=dtype),
        "blocks": [],
    }
    for i, (dim_in, dim_out, _heads, _s, transition) in enumerate(backbone_block_table()):
        p["blocks"].append(block_params(seed, dim_in, dim_out, transition, dtype=dtype,
                                        affine=affine, base_id=2000 + 32 * i))
    return p


def image(seed: int, batch: int, img: int, dtype: str = BF16) -> np.ndarray:
    """NHWC image [B, img, img, 4] ~ U(-1, 1)."""
    return uniform(seed, 7, (batch, img, img, IN_CHANS), dtype=dtype)


def activations(seed: int, shape, dtype: str = BF16) -> np.ndarray:
    """Block input x ~ N(0, 1)."""
    return normal(seed, 9, shape, 1.0, dtype=dtype)
