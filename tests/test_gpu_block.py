"""HieraBlock forward through the C ABI against the fp64 oracle.

Tolerances (stated for the block): fp32 mode max-abs <= 1e-4; bf16 mode (bf16 inputs and
weights, fp32 accumulation) rel-L2 <= 1e-2 over the whole output. Beside it, so that a
fault confined to one mask unit, one head, one image or the ragged last tile is not
diluted by the rest of the tensor:
  * every output row (token) within ROW_BOUND rel-L2;
  * the merged attention output (before proj, read from the workspace) of every
    (image, window, head) unit within UNIT_BOUND rel-L2 of the oracle's. That output
    carries the bf16 rounding of q, k and v (2^-9 each; a score error of about
    2^-8 |s| moves each softmax weight by that much relative) plus the bf16 softmax
    weights and the output rounding, with no residual to hide a wrong unit.
"""

import numpy as np
import pytest
import torch

from mask_unit_windowed_b200 import binding as hb
from mask_unit_windowed_b200 import synthetic as syn
from oracle import unrolled as U

from helpers import (TORCH_DT, block_weights_dev, dev, host, max_abs, rel_l2, row_rel_l2,
                     unit_rel_l2)

pytestmark = pytest.mark.gpu

F32_MAX_ABS = 1e-4
BF16_REL_L2 = 1e-2
ROW_BOUND = 1e-2     # measured on B200: at most 4.7e-3 on any output row of these cases
UNIT_BOUND = 1e-2    # measured: at most 5.0e-3 (7.0e-3 with the widened score range)


def run_case(B, tokens, d_in, d_out, heads, q_stride, window, mua, dtype, seed, affine,
             qk_scale=1.0, fused_attn=False):
    transition = d_in != d_out
    p = syn.block_params(seed, d_in, d_out, transition, dtype=dtype, affine=affine)
    if qk_scale != 1.0:   # wider score range: q and k rows of the qkv weight scaled
        w = p["qkv_w"].copy()
        w[:2 * d_out] = syn.round_to_bf16(w[:2 * d_out] * qk_scale) if dtype == "bf16" \
            else w[:2 * d_out] * qk_scale
        p["qkv_w"] = w
    x = syn.activations(seed, (B, tokens, d_in), dtype=dtype)
    desc = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                        q_stride=q_stride, window_tokens=window, mask_unit_attn=mua,
                        dtype=TORCH_DT[dtype])
    packed = hb.block_pack(desc, block_weights_dev(p, dtype))
    ws = torch.empty(hb.block_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    with hb.fused_attention(fused_attn):   # unfused: q, k, v, attention output in the workspace
        y = hb.block_forward(desc, packed, dev(x, dtype), workspace=ws)
    assert hb.device_status() == 0
    ref = U.block_forward(x, p, heads, q_stride, window, mua)
    return host(y), ref, desc, packed, p, x, ws


def check_units(desc, p, x, ws, bound=UNIT_BOUND):
    """Per (image, window, head) unit: the merged attention output in the workspace
    against the oracle's attention output before proj."""
    B, heads, qs = desc.B, desc.heads, desc.q_stride
    nW = desc.tokens // desc.window_tokens if desc.mask_unit_attn else 1
    Tq = desc.tokens // nW // qs
    off = hb.block_workspace_layout(desc)[3]
    n = B * Tq * nW * desc.dim_out
    o = host(ws[off:off + 2 * n].view(torch.bfloat16)).reshape(B, Tq * nW, desc.dim_out)
    xn = U.layer_norm(x, p["norm1_w"], p["norm1_b"])
    ref = U.attention_heads(xn, p["qkv_w"], p["qkv_b"], heads, qs, desc.window_tokens,
                            desc.mask_unit_attn)
    err = unit_rel_l2(o, ref, B, Tq, nW, heads)
    worst = np.unravel_index(np.argmax(err), err.shape)
    print(f"attention units: max rel-L2 {err.max():.3e} at (image, window, head) {worst}")
    assert err.max() <= bound, (err.max(), worst)


def check_rows(y, ref, bound=ROW_BOUND):
    err = row_rel_l2(y, ref)
    worst = np.unravel_index(np.argmax(err), err.shape)
    print(f"output rows: max rel-L2 {err.max():.3e} at {worst}, tensor {rel_l2(y, ref):.3e}")
    assert err.max() <= bound, (err.max(), worst)


CASES = {
    # name: (B, tokens, d_in, d_out, heads, q_stride, window, mask_unit_attn)
    "stage0_windowed": (2, 256, 112, 112, 2, 1, 64, True),
    "stage1_windowed": (2, 1024, 224, 224, 4, 1, 16, True),
    "stage1_transition": (2, 256, 112, 224, 4, 4, 64, True),
    "stage2_transition_lagged_mu": (2, 256, 224, 448, 8, 4, 16, True),
    "stage2_transition_global": (2, 1024, 224, 448, 8, 4, 16, False),
    "stage3_transition_small": (3, 64, 448, 896, 16, 4, 4, False),
    "global_ragged": (3, 1000, 448, 448, 8, 1, 1, False),
    "stage3_global": (2, 256, 896, 896, 16, 1, 1, False),
}


@pytest.mark.parametrize("name", list(CASES))
def test_block_bf16(name):
    y, ref, desc, _, p, x, ws = run_case(*CASES[name], dtype="bf16", seed=5, affine="random")
    assert y.shape == ref.shape
    assert np.isfinite(y).all()
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)
    check_units(desc, p, x, ws)


@pytest.mark.parametrize("name", ["stage0_windowed", "stage1_windowed", "stage1_transition",
                                  "stage2_transition_lagged_mu", "global_ragged",
                                  "stage2_transition_global"])
def test_block_bf16_wide_score_range(name):
    """q and k weights scaled by 3 (scores ~9x wider, softmax rows peaked) through the whole
    block, pooled transitions included. The bf16 rounding of q and k now moves scores by
    about 2^-8 |s|, so the attention units get twice the bound."""
    y, ref, desc, _, p, x, ws = run_case(*CASES[name], dtype="bf16", seed=12,
                                         affine="random", qk_scale=3.0)
    assert np.isfinite(y).all()
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)
    check_units(desc, p, x, ws, bound=2 * UNIT_BOUND)


@pytest.mark.parametrize("name", ["stage0_windowed", "stage1_transition", "global_ragged",
                                  "stage2_transition_lagged_mu", "stage3_transition_small"])
def test_block_f32(name):
    y, ref, *_ = run_case(*CASES[name], dtype="f32", seed=6, affine="random")
    print(f"max-abs {max_abs(y, ref):.3e}")
    assert max_abs(y, ref) <= F32_MAX_ABS, max_abs(y, ref)


def test_cfg1_stage0_block_f32():
    """Single stage-0 block, fp32, batch 1: 32x32 grid unrolled into 16 mask units of 64,
    dim 112, 2 heads, no q-pool, MLP 448; x ~ N(0,1), W ~ N(0,0.02), b=0, gamma=1, beta=0,
    seed 0."""
    y, ref, *_ = run_case(1, 1024, 112, 112, 2, 1, 64, True, dtype="f32", seed=0, affine="init")
    assert max_abs(y, ref) <= F32_MAX_ABS, max_abs(y, ref)


def test_cfg2_stage1_transition_bf16():
    """Stage-1 transition block, bf16, batch 4: 128x128 tokens at dim 112 -> 224, 4 heads,
    q_stride 4 (64 keys, 16 pooled queries per unit), MLP 896, seed 1."""
    y, ref, desc, _, p, x, ws = run_case(4, 16384, 112, 224, 4, 4, 64, True, dtype="bf16",
                                         seed=1, affine="init")
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)
    check_units(desc, p, x, ws)


def test_cfg3_stage2_global_bf16():
    """Stage-2 global block, bf16, batch 8: 1024 tokens, dim 448, 8 heads, MLP 1792, seed 2."""
    y, ref, desc, _, p, x, ws = run_case(8, 1024, 448, 448, 8, 1, 1, False, dtype="bf16",
                                         seed=2, affine="init")
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)
    check_units(desc, p, x, ws)


@pytest.mark.parametrize("shape", [
    # (B, tokens, d_in, d_out, heads, q_stride, window): 4 windows, rows copied out by lanes
    (2, 256, 112, 224, 4, 4, 64),
    # transition with 16 windows: k and v of the pooled tiles leave by 5-D TMA boxes
    (2, 1024, 112, 224, 4, 4, 64),
    # 64 windows, no pooling: q, k and v leave by 4-D TMA boxes of 32 windows
    (2, 1024, 224, 224, 4, 1, 16),
])
def test_qkv_scatter_layout_bf16(shape):
    """The qkv GEMM writes q (pooled in a transition), k, v head-major with zero padding:
    compare the workspace against the oracle's projections, for each way the rows leave."""
    B, tokens, d_in, d_out, heads, qs, window = shape
    transition = d_in != d_out
    p = syn.block_params(7, d_in, d_out, transition, dtype="bf16", affine="random")
    x = syn.activations(7, (B, tokens, d_in), dtype="bf16")
    desc = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                        q_stride=qs, window_tokens=window)
    packed = hb.block_pack(desc, block_weights_dev(p, "bf16"))
    ws = torch.empty(hb.block_workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    with hb.fused_attention(False):
        hb.block_forward(desc, packed, dev(x), workspace=ws)
    torch.cuda.synchronize()
    offs = hb.block_workspace_layout(desc)
    nW = tokens // window
    Tkv, Tq = window, window // qs
    xn = U.layer_norm(x, p["norm1_w"], p["norm1_b"])
    qkv = U.linear(xn, p["qkv_w"], p["qkv_b"]).reshape(B, Tkv, nW, 3, heads, 56)
    qkv = qkv.transpose(3, 0, 2, 4, 1, 5)               # [3, B, nW, h, T, 56]
    q = qkv[0].reshape(B, nW, heads, qs, Tq, 56).max(axis=3)

    def view(off, T):
        n = B * nW * heads * T * 64
        t = ws[off:off + 2 * n].view(torch.bfloat16).reshape(B, nW, heads, T, 64)
        return host(t)
    for i, (got, want) in enumerate(((view(offs[0], Tq), q), (view(offs[1], Tkv), qkv[1]),
                                     (view(offs[2], Tkv), qkv[2]))):
        if i == 2:   # v: the ones channel that carries the softmax denominator, then zeros
            assert np.all(got[..., 56] == 1) and np.all(got[..., 57:] == 0)
        else:
            assert np.all(got[..., 56:] == 0)
        assert rel_l2(got[..., :56], want) < 5e-3
        # every (image, window, head) block in place, not only the tensor as a whole
        err = np.sqrt(((got[..., :56] - want) ** 2).sum(axis=(-1, -2)) /
                      (want ** 2).sum(axis=(-1, -2)))
        assert err.max() < 1e-2, (i, float(err.max()))
    if transition:
        r = host(ws[offs[4]:offs[4] + 2 * B * (tokens // 4) * d_out].view(torch.bfloat16)
                 ).reshape(B, tokens // 4, d_out)
        r_ref = U.max_pool_tokens(U.linear(xn, p["proj_w"], p["proj_b"]), qs)
        assert rel_l2(r, r_ref) < 5e-3


def test_repeat_is_deterministic_bf16():
    args = CASES["stage1_transition"]
    y1, _, desc, packed, p, x, _ = run_case(*args, dtype="bf16", seed=8, affine="random")
    y2 = host(hb.block_forward(desc, packed, dev(x)))
    np.testing.assert_array_equal(y1, y2)


@pytest.mark.parametrize("name", list(CASES))
def test_block_batch_independent_bitwise(name):
    """Image 0 of a batch gives bit-identical output to the same image alone."""
    B, tokens, d_in, d_out, heads, qs, window, mua = CASES[name]
    p = syn.block_params(9, d_in, d_out, d_in != d_out, dtype="bf16", affine="random")
    x = syn.activations(9, (B, tokens, d_in), dtype="bf16")
    w = block_weights_dev(p, "bf16")
    dB = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                      q_stride=qs, window_tokens=window, mask_unit_attn=mua)
    d1 = hb.BlockDesc(B=1, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                      q_stride=qs, window_tokens=window, mask_unit_attn=mua)
    yB = hb.block_forward(dB, hb.block_pack(dB, w), dev(x))
    y1 = hb.block_forward(d1, hb.block_pack(d1, w), dev(x[:1]))
    diff = (yB[:1].float() - y1.float()).abs().max().item()
    assert torch.equal(yB[:1], y1), diff


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("name", ["global_ragged", "stage3_global", "stage1_transition",
                                  "stage0_windowed"])
def test_block_intermediates_deterministic(name, fused):
    """Race check: five forwards of the same block into workspaces pre-filled with
    different garbage give bit-identical q/k/v, attention output, residual, x1, MLP hidden
    (when the MLP is not fused: the fused kernel never writes it) and y."""
    B, tokens, d_in, d_out, heads, qs, window, mua = CASES[name]
    p = syn.block_params(10, d_in, d_out, d_in != d_out, dtype="bf16", affine="random")
    x = dev(syn.activations(10, (B, tokens, d_in), dtype="bf16"))
    desc = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads,
                        q_stride=qs, window_tokens=window, mask_unit_attn=mua)
    packed = hb.block_pack(desc, block_weights_dev(p, "bf16"))
    offs = hb.block_workspace_layout(desc)
    nW = tokens // window if mua else 1
    Tkv = tokens // nW
    Tq, Nq = Tkv // qs, tokens // qs
    sizes = [B * nW * heads * Tq * 64 * 2, B * nW * heads * Tkv * 64 * 2,
             B * nW * heads * Tkv * 64 * 2, B * Nq * d_out * 2, B * Nq * d_out * 2,
             B * Nq * d_out * 2, B * Nq * 4 * d_out * 2]
    if fused and d_out in (112, 224):
        sizes[6] = 0
    nbytes = hb.block_workspace_bytes(desc)
    ref = None
    for rep in range(5):
        ws = torch.full((nbytes,), (rep * 53 + 7) % 256, dtype=torch.uint8, device="cuda")
        with hb.fused_mlp(fused), hb.fused_attention(False):
            y = hb.block_forward(desc, packed, x, workspace=ws)
        torch.cuda.synchronize()
        parts = [ws[o:o + n].clone() for o, n in zip(offs, sizes) if o >= 0] + [y.clone()]
        if ref is None:
            ref = parts
        else:
            for i, (a, b) in enumerate(zip(parts, ref)):
                assert torch.equal(a, b), f"buffer {i} differs in repeat {rep}"
    assert hb.device_status() == 0


FUSED_ATTN_CASES = {
    # stage-0 shapes the fused attention half takes: dim 112, 2 heads, windows of 64
    "stage0_b2": (2, 256, 112, 112, 2, 1, 64, True),
    "stage0_32x32": (1, 1024, 112, 112, 2, 1, 64, True),
    "stage0_odd_tiles": (3, 384, 112, 112, 2, 1, 64, True),
}


@pytest.mark.parametrize("name", list(FUSED_ATTN_CASES))
def test_fused_attention_half_matches_oracle(name):
    """norm1 + qkv + windowed attention + proj + residual in one kernel (the block's
    intermediates never reach memory): whole-output and per-row bounds against the
    oracle, and within bf16 rounding of the separate kernels' result."""
    args = FUSED_ATTN_CASES[name]
    y, ref, desc, packed, p, x, _ = run_case(*args, dtype="bf16", seed=13, affine="random",
                                             fused_attn=True)
    assert np.isfinite(y).all()
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)
    with hb.fused_attention(False):
        y_sep = host(hb.block_forward(desc, packed, dev(x)))
    # the fused P V sums a window's keys in another order; the outputs agree to a few bf16
    # ulps of the attention branch
    assert rel_l2(y, y_sep) <= 2e-3, rel_l2(y, y_sep)


def test_fused_attention_half_wide_scores():
    y, ref, *_ = run_case(*FUSED_ATTN_CASES["stage0_32x32"], dtype="bf16", seed=14,
                          affine="random", qk_scale=3.0, fused_attn=True)
    assert rel_l2(y, ref) <= BF16_REL_L2, rel_l2(y, ref)
    check_rows(y, ref)


def test_fused_attention_half_deterministic_and_batch_independent():
    B, tokens, d_in, d_out, heads, qs, window, mua = FUSED_ATTN_CASES["stage0_odd_tiles"]
    p = syn.block_params(15, d_in, d_out, False, dtype="bf16", affine="random")
    x = syn.activations(15, (B, tokens, d_in), dtype="bf16")
    w = block_weights_dev(p, "bf16")
    dB = hb.BlockDesc(B=B, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads)
    d1 = hb.BlockDesc(B=1, tokens=tokens, dim_in=d_in, dim_out=d_out, heads=heads)
    pB, p1 = hb.block_pack(dB, w), hb.block_pack(d1, w)
    yB = hb.block_forward(dB, pB, dev(x))
    yB2 = hb.block_forward(dB, pB, dev(x))
    y1 = hb.block_forward(d1, p1, dev(x[2:3]))
    assert torch.equal(yB, yB2)
    assert torch.equal(yB[2:3], y1)
    assert hb.device_status() == 0
