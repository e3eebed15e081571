"""The attention core (hiera_attention) against the fp64 oracle, element by element, on
inputs built to reach the edge cases of the softmax ("Phase 4: Hiera Backbone MLX Port",
Architecture Summary, MaskUnitAttention: scaled dot-product attention per mask-unit
window or over all tokens).

q, k and v are bf16 values drawn by the seeded generator; both sides see exactly those
values, so the only differences are the kernel's fp32 arithmetic and its bf16 softmax
weights. Error bound per output row (rel-L2 over the row's 56 channels of one head):
  * the weights enter the P V product truncated to bf16: each has a relative error below
    2^-7, and the denominator is the sum of the same truncated weights, so the row's error
    is at most 2^-7 * sum_j p_j |v_j - o| / |o| in the worst case and about 2^-9 on average;
  * the output is rounded to bf16 once (2^-9).
ROW_BOUND = 1e-2 covers a spread sum_j p_j |v_j - o| of up to ~|o| (measured on B200: at
most 4.2e-3 on any row of these cases); the whole-tensor rel-L2 must stay within
TENSOR_BOUND = 4e-3 (measured: at most 2.6e-3).
"""

import math

import numpy as np
import pytest
import torch

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

pytestmark = pytest.mark.gpu

ROW_BOUND = 1e-2
TENSOR_BOUND = 4e-3
HD = 56


def _padded(a56, ones_channel):
    """[..., T, 56] bf16-exact values -> CUDA bf16 [..., T, 64] in the library's layout."""
    shape = a56.shape[:-1] + (64,)
    a = np.zeros(shape, np.float32)
    a[..., :HD] = a56
    if ones_channel:
        a[..., HD] = 1.0
    return torch.from_numpy(a).to("cuda", torch.bfloat16)


def run(q, k, v):
    """q [B, nW, h, Tq, 56], k / v [B, nW, h, Tkv, 56] (bf16-exact float32). Returns the GPU
    and oracle outputs as [B, Tq, nW, h, 56] (token j*nW + w, head h)."""
    B, nW, heads, Tq, _ = q.shape
    o = hb.attention(_padded(q, False), _padded(k, False), _padded(v, True))
    assert hb.device_status() == 0
    got = o.double().cpu().numpy().reshape(B, Tq, nW, heads, HD)
    ref = U.attention_core(q, k, v, HD)                       # [B, nW, h, Tq, 56]
    return got, ref.transpose(0, 3, 1, 2, 4)


def check(got, ref, row_bound=ROW_BOUND, tensor_bound=TENSOR_BOUND):
    assert np.isfinite(got).all()
    err = np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    tensor = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    worst = np.unravel_index(np.argmax(err), err.shape)
    print(f"max row rel-L2 {err.max():.3e} at {worst}, tensor rel-L2 {tensor:.3e}")
    assert err.max() <= row_bound, (err.max(), worst)
    assert tensor <= tensor_bound, tensor


def bf16(a):
    return syn.round_to_bf16(np.asarray(a, np.float32))


def test_global_late_max_needs_the_running_max_rescale():
    """Branch: the 128-key-tile kernel's running-max raise with the O rescale in TMEM.
    Keys of tile t are scaled by 1 + 30 t, so every tile's row max exceeds the running max
    by about 15 in exp2 units (more than the 2^8 threshold) and the last tile's max exceeds
    the first tile's by several hundred: a kernel that kept the first tile's max would
    overflow 2^(s - m) to inf. 10 key tiles; 200 queries (the second query tile ragged)."""
    B, nW, heads, Tq, Tkv = 1, 1, 2, 200, 1280
    q = syn.normal(61, 1, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(61, 2, (B, nW, heads, Tkv, HD))
    scale = 1.0 + 30.0 * (np.arange(Tkv) // 128)
    k = bf16(k * scale[:, None])
    v = syn.normal(61, 3, (B, nW, heads, Tkv, HD), dtype="bf16")
    s = np.einsum("bwhqd,bwhkd->bwhqk", q, k) / math.sqrt(HD)
    first, last = s[..., :128].max(-1), s[..., -128:].max(-1)
    assert ((last - first) * math.log2(math.e) > 128).all()   # overflows without the rescale
    got, ref = run(q, k, v)
    check(got, ref)


def test_global_max_in_ragged_last_tile_peaked_rows():
    """Branch: ragged last key tile (1000 keys: 104 in the last tile) holding each row's max.
    Queries 0..103 each own one planted key in the last tile (k = 1.5 q, a score about 11
    where the others have standard deviation ~2: peaked rows, a few keys carry the
    weight); the other queries see near-uniform rows."""
    B, nW, heads, Tq, Tkv = 2, 1, 2, 256, 1000
    q = syn.normal(62, 1, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(62, 2, (B, nW, heads, Tkv, HD), std=2.0, dtype="bf16")
    k[..., 896:1000, :] = bf16(1.5 * q[..., 0:104, :])
    v = syn.normal(62, 3, (B, nW, heads, Tkv, HD), dtype="bf16")
    s = np.einsum("bwhqd,bwhkd->bwhqk", q, k) / math.sqrt(HD)
    assert (s[..., :104, :].argmax(-1) >= 896).all()
    got, ref = run(q, k, v)
    check(got, ref)


@pytest.mark.parametrize("std", [1.0, 4.0])
def test_global_pooled_queries(std):
    """The transition form at the attention level: 256 pooled queries against 1024 keys
    (Tq = Tkv / 4), near-uniform (std 1) and peaked (std 4) rows."""
    B, nW, heads, Tq, Tkv = 1, 1, 4, 256, 1024
    q = syn.normal(63, 1, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(63, 2, (B, nW, heads, Tkv, HD), std=std, dtype="bf16")
    v = syn.normal(63, 3, (B, nW, heads, Tkv, HD), dtype="bf16")
    got, ref = run(q, k, v)
    check(got, ref)


# (Tq, Tkv) of the windowed kernel: stage 0, the stage-1 transition, stage 1, the lagged
# block 5, and the other window sizes the kernel takes
WINDOWS = [(64, 64), (16, 64), (16, 16), (4, 16), (32, 32), (8, 32), (8, 8), (2, 8), (4, 4),
           (1, 4)]


@pytest.mark.parametrize("Tq,Tkv", WINDOWS)
def test_windowed_matches_oracle(Tq, Tkv):
    """Several (image, window, head) units per tensor-core tile: 2 images x 7 windows x 3
    heads = 42 units, not a multiple of the units per tile (the last tile is ragged)."""
    B, nW, heads = 2, 7, 3
    q = syn.normal(64, Tkv, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(65, Tkv, (B, nW, heads, Tkv, HD), dtype="bf16")
    v = syn.normal(66, Tkv, (B, nW, heads, Tkv, HD), dtype="bf16")
    got, ref = run(q, k, v)
    check(got, ref)


@pytest.mark.parametrize("Tq,Tkv", [(64, 64), (16, 64), (16, 16), (4, 16)])
def test_windowed_wide_range_max_in_second_half(Tq, Tkv):
    """Scores spanning hundreds of units with every row's max among the last half of its
    window's keys (those keys scaled by 40): the single-pass softmax must subtract the true
    row max or 2^(s - m) overflows."""
    B, nW, heads = 1, 9, 2
    q = syn.normal(67, Tkv, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(68, Tkv, (B, nW, heads, Tkv, HD))
    k[..., Tkv // 2:, :] *= 40.0
    k = bf16(k)
    v = syn.normal(69, Tkv, (B, nW, heads, Tkv, HD), dtype="bf16")
    s = np.einsum("bwhqd,bwhkd->bwhqk", q, k) / math.sqrt(HD)
    assert (s.argmax(-1) >= Tkv // 2).mean() > 0.95
    assert np.percentile((s.max(-1) - s.min(-1)) * math.log2(math.e), 10) > 64
    got, ref = run(q, k, v)
    check(got, ref)


def test_global_small_sizes_use_the_general_kernel():
    """Sizes outside the windowed kernel's table (48 keys; 100 queries against 300 keys)
    run the 128-key-tile kernel with masked keys and rows."""
    for (Tq, Tkv, seed) in ((48, 48, 70), (100, 300, 71), (12, 48, 72)):
        q = syn.normal(seed, 1, (2, 3, 2, Tq, HD), dtype="bf16")
        k = syn.normal(seed, 2, (2, 3, 2, Tkv, HD), dtype="bf16")
        v = syn.normal(seed, 3, (2, 3, 2, Tkv, HD), dtype="bf16")
        got, ref = run(q, k, v)
        check(got, ref)


def test_global_more_ctas_than_sms():
    """4 x 40 units x 2 query-tile pairs = 320 CTAs of the 128-key-tile kernel on 148 SMs
    (several waves, ragged query and key tiles). Each unit's keys carry their own scale (1x
    to 9x) and its last, ragged tile (44 of 300 keys) holds keys scaled 4x more, so a unit
    whose running max or rescale went wrong would be far off."""
    B, nW, heads, Tq, Tkv = 4, 1, 40, 300, 300
    q = syn.normal(73, 1, (B, nW, heads, Tq, HD), dtype="bf16")
    k = syn.normal(73, 2, (B, nW, heads, Tkv, HD))
    unit = np.arange(B * nW * heads).reshape(B, nW, heads)
    k = k * (1.0 + 2.0 * (unit % 5))[..., None, None]
    k[..., 256:, :] *= 4.0
    k = bf16(k)
    v = syn.normal(73, 3, (B, nW, heads, Tkv, HD), dtype="bf16")
    got, ref = run(q, k, v)
    check(got, ref)
