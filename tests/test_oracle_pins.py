"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test checks the oracle against something other than itself: inverse
permutations, the stage shapes the "Phase 4: Hiera Backbone MLX Port" plan lists
(Sub-phase 4d shape tests; corridorkey-mlx README "Reference Fixtures" table),
brute-force per-query loops written in spatial coordinates, a second independent
formulation on NHWC grids, library routines (scipy's normal CDF) and closed forms.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.stats import norm

from mask_unit_windowed_b200 import synthetic as syn
from oracle import spatial as S
from oracle import unrolled as U

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- Unroll / Reroll
@pytest.mark.parametrize("G,levels", [(8, 3), (16, 3), (32, 2), (16, 1), (8, 0), (128, 3)])
def test_unroll_reroll_inverse(G, levels):
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2, G * G, 3))
    u = U.unroll_index(G, levels)
    assert sorted(u.reshape(-1).tolist()) == list(range(G * G))       # a permutation
    back = U.reroll(U.unroll(x, G, levels), G, levels)
    np.testing.assert_array_equal(back.reshape(2, G * G, 3), x)       # Reroll o Unroll = id
    xu = rng.standard_normal((2, G * G, 3))
    again = U.unroll(U.reroll(xu, G, levels).reshape(2, G * G, 3), G, levels)
    np.testing.assert_array_equal(again, xu)                          # Unroll o Reroll = id


@pytest.mark.parametrize("G,levels", [(16, 3), (32, 3), (32, 2)])
def test_mask_units_are_square_tiles(G, levels):
    """Window w = n mod nW holds exactly one (2^L x 2^L) spatial tile."""
    u = U.unroll_index(G, levels)
    side = 1 << levels
    nW = (G // side) ** 2
    pos = {int(u[y, x]): (y, x) for y in range(G) for x in range(G)}
    for w in range(nW):
        cells = {pos[n] for n in range(w, G * G, nW)}
        tiles = {(y // side, x // side) for (y, x) in cells}
        assert len(cells) == side * side and len(tiles) == 1


@pytest.mark.parametrize("G,levels", [(16, 3), (32, 2), (8, 1)])
def test_pool_chunks_are_2x2_cells_in_next_order(G, levels):
    """Tokens n + c N/4 (c = 0..3) form one 2x2 cell, and n is that cell's index in
    the next stage's unrolled order (so the pooled result needs no re-permutation)."""
    N = G * G
    u = U.unroll_index(G, levels)
    u_next = U.unroll_index(G // 2, levels - 1)
    pos = {int(u[y, x]): (y, x) for y in range(G) for x in range(G)}
    for n in range(N // 4):
        cell = [pos[n + c * (N // 4)] for c in range(4)]
        ys = {y // 2 for y, _ in cell}
        xs = {x // 2 for _, x in cell}
        assert len(ys) == 1 and len(xs) == 1
        assert len(set(cell)) == 4
        assert u_next[ys.pop(), xs.pop()] == n


def test_unroll_golden_small_grid():
    """A 4x4 grid with two levels: one mask unit, in-unit index with the finest 2x2
    offset outermost. Table written out by hand in tests/golden."""
    with open(os.path.join(GOLDEN, "unroll_4x4_levels2.json")) as f:
        gold = json.load(f)
    np.testing.assert_array_equal(U.unroll_index(4, 2), np.array(gold["u"]))


# ----------------------------------------------------------------------------- pooling / windows
def test_q_stride_one_is_identity():
    x = np.random.default_rng(1).standard_normal((2, 64, 5))
    np.testing.assert_array_equal(U.max_pool_tokens(x, 1), x)


def _tiny_block(seed, dim_in, dim_out, transition, affine="random"):
    p = syn.block_params(seed, dim_in, dim_out, transition, dtype="f32", affine=affine)
    # enlarge the weights so that attention is far from uniform
    for k in ("qkv_w", "attn_proj_w", "fc1_w", "fc2_w", "proj_w"):
        if k in p:
            p[k] = p[k] * 25.0
    return p


def test_one_window_of_all_tokens_is_global_attention():
    rng = np.random.default_rng(2)
    xn = rng.standard_normal((2, 64, 8))
    p = _tiny_block(3, 8, 8, False)
    a = U.mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"], p["attn_proj_b"],
                              2, 1, 64, True, head_dim=4)
    g = U.mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"], p["attn_proj_b"],
                              2, 1, 64, False, head_dim=4)
    np.testing.assert_array_equal(a, g)
    # and with q pooling
    a = U.mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"], p["attn_proj_b"],
                              2, 4, 64, True, head_dim=4)
    g = U.mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"], p["attn_proj_b"],
                              2, 4, 64, False, head_dim=4)
    np.testing.assert_array_equal(a, g)


# ----------------------------------------------------------------------------- brute force
def _bf_layer_norm(v, w, b, eps=1e-6):
    n = len(v)
    mean = sum(v) / n
    var = sum((t - mean) ** 2 for t in v) / n
    return [(t - mean) / math.sqrt(var + eps) * w[i] + b[i] for i, t in enumerate(v)]


def _bf_linear(v, W, b):
    return [sum(W[o][i] * v[i] for i in range(len(v))) + b[o] for o in range(len(W))]


def _bf_gelu(t):
    return 0.5 * t * (1.0 + math.erf(t / math.sqrt(2.0)))


def _bf_block(grid, p, heads, hd, tile, pool):
    """One block written as per-pixel, per-query loops in spatial coordinates.
    grid: dict (y, x) -> list of channels. tile: mask-unit side on the input grid or None."""
    G = int(round(math.sqrt(len(grid))))
    P = {k: np.asarray(v, np.float64).tolist() for k, v in p.items()}
    d_out = len(P["attn_proj_w"])
    xn = {c: _bf_layer_norm(v, P["norm1_w"], P["norm1_b"]) for c, v in grid.items()}
    qkv = {c: _bf_linear(v, P["qkv_w"], P["qkv_b"]) for c, v in xn.items()}
    Gq = G // pool
    resid = {}
    for yq in range(Gq):
        for xq in range(Gq):
            if pool == 2:
                cands = [_bf_linear(xn[(2 * yq + dy, 2 * xq + dx)], P["proj_w"], P["proj_b"])
                         for dy in range(2) for dx in range(2)]
                resid[(yq, xq)] = [max(c[i] for c in cands) for i in range(d_out)]
            else:
                resid[(yq, xq)] = list(grid[(yq, xq)])
    out = {}
    for yq in range(Gq):
        for xq in range(Gq):
            cells = [(yq * pool + dy, xq * pool + dx) for dy in range(pool) for dx in range(pool)]
            if tile is None:
                keys = list(grid.keys())
            else:
                ty, tx = (yq * pool) // tile, (xq * pool) // tile
                keys = [(y, x) for (y, x) in grid if y // tile == ty and x // tile == tx]
            merged = []
            for h in range(heads):
                q = [max(qkv[c][h * hd + e] for c in cells) for e in range(hd)]
                scores = []
                for kc in keys:
                    kv = qkv[kc]
                    scores.append(sum(q[e] * kv[d_out + h * hd + e] for e in range(hd)) / math.sqrt(hd))
                m = max(scores)
                ws = [math.exp(s - m) for s in scores]
                tot = sum(ws)
                o = [sum(ws[j] / tot * qkv[kc][2 * d_out + h * hd + e] for j, kc in enumerate(keys))
                     for e in range(hd)]
                merged.extend(o)
            a = _bf_linear(merged, P["attn_proj_w"], P["attn_proj_b"])
            x1 = [resid[(yq, xq)][i] + a[i] for i in range(d_out)]
            hdn = [_bf_gelu(t) for t in _bf_linear(_bf_layer_norm(x1, P["norm2_w"], P["norm2_b"]),
                                                    P["fc1_w"], P["fc1_b"])]
            m2 = _bf_linear(hdn, P["fc2_w"], P["fc2_b"])
            out[(yq, xq)] = [x1[i] + m2[i] for i in range(d_out)]
    return out


@pytest.mark.parametrize("case", [
    dict(G=8, levels=2, dim_in=8, dim_out=8, transition=False, mua=True),    # 4 windows of 16
    dict(G=8, levels=2, dim_in=6, dim_out=8, transition=True, mua=True),     # q pooled 16 -> 4
    dict(G=4, levels=1, dim_in=8, dim_out=8, transition=False, mua=False),   # global
    dict(G=8, levels=1, dim_in=6, dim_out=8, transition=True, mua=False),    # global + pooled
])
def test_block_matches_brute_force_spatial_loops(case):
    G, L = case["G"], case["levels"]
    heads, hd = 2, 4
    p = _tiny_block(11, case["dim_in"], case["dim_out"], case["transition"])
    rng = np.random.default_rng(12)
    raster = rng.standard_normal((1, G * G, case["dim_in"]))
    q_stride = 4 if case["transition"] else 1
    window_tokens = (1 << L) ** 2
    xu = U.unroll(raster, G, L)
    yu = U.block_forward(xu, p, heads, q_stride, window_tokens, case["mua"], head_dim=hd)
    L_out = L - 1 if case["transition"] else L
    y_grid = U.reroll(yu, G // (2 if case["transition"] else 1), L_out)[0]
    grid = {(y, x): raster[0, y * G + x].tolist() for y in range(G) for x in range(G)}
    bf = _bf_block(grid, p, heads, hd, (1 << L) if case["mua"] else None,
                   2 if case["transition"] else 1)
    for (y, x), v in bf.items():
        np.testing.assert_allclose(y_grid[y, x], v, rtol=1e-10, atol=1e-10)


def test_patch_embed_matches_brute_force_loops():
    rng = np.random.default_rng(5)
    img = rng.uniform(-1, 1, (1, 12, 12, 4))
    w = rng.standard_normal((5, 7, 7, 4))
    b = rng.standard_normal(5)
    out = U.patch_embed(img, w, b)                          # [1, 9, 5]
    for oy in range(3):
        for ox in range(3):
            for co in range(5):
                acc = b[co]
                for ky, kx, c in itertools.product(range(7), range(7), range(4)):
                    iy, ix = 4 * oy - 3 + ky, 4 * ox - 3 + kx
                    if 0 <= iy < 12 and 0 <= ix < 12:
                        acc += w[co, ky, kx, c] * img[0, iy, ix, c]
                assert abs(out[0, oy * 3 + ox, co] - acc) < 1e-12


def test_patch_embed_delta_kernel_samples_input():
    """A kernel that is 1 at the centre tap (3, 3) samples the input at (4y, 4x)."""
    rng = np.random.default_rng(6)
    img = rng.standard_normal((2, 16, 16, 4))
    w = np.zeros((4, 7, 7, 4))
    for c in range(4):
        w[c, 3, 3, c] = 1.0
    out = U.patch_embed(img, w, np.zeros(4)).reshape(2, 4, 4, 4)
    np.testing.assert_array_equal(out, img[:, ::4, ::4, :])


# ----------------------------------------------------------------------------- formulation S
@pytest.mark.parametrize("img", [64, 128])
def test_spatial_formulation_equals_unrolled(img):
    p = syn.backbone_params(21, img, dtype="f32", affine="random")
    x = syn.image(21, 2, img, dtype="f32")
    fu = U.backbone_forward(x, p)
    fs = S.spatial_backbone(x, p)
    for a, b in zip(fu, fs):
        assert a.shape == b.shape
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)


def test_spatial_formulation_equals_unrolled_lagged_mask_unit_flag():
    """Block 5 with mask-unit attention (16 keys, 4 pooled queries per unit)."""
    flags = [True] * 6 + [False] * 18
    p = syn.backbone_params(22, 64, dtype="f32", affine="random")
    x = syn.image(22, 1, 64, dtype="f32")
    fu = U.backbone_forward(x, p, mask_unit_attn_override=flags)
    fs = S.spatial_backbone(x, p, mask_unit_flags=flags)
    for a, b in zip(fu, fs):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-11)
    # and it differs from the default schedule (block 5 global)
    fd = U.backbone_forward(x, p)
    assert np.abs(fd[2] - fu[2]).max() > 1e-6


def test_stage_shapes_at_512():
    """128^2x112, 64^2x224, 32^2x448, 16^2x896 for a 512^2 input (the plan's shape tests
    and the README fixture table), four features."""
    with open(os.path.join(GOLDEN, "stage_shapes_512.json")) as f:
        gold = json.load(f)
    p = syn.backbone_params(3, 512, dtype="bf16")
    x = syn.image(3, 1, 512)
    feats = U.backbone_forward(x, p)
    assert len(feats) == len(gold["features"])
    for f, g in zip(feats, gold["features"]):
        assert list(f.shape) == [1] + g
        assert np.isfinite(f).all()
    assert U.patch_embed(x, p["patch_w"], p["patch_b"]).shape == (1, 128 * 128, 112)


def test_block_schedule_matches_plan_table():
    sched = U.block_schedule()
    assert len(sched) == 24
    assert [i for i, c in enumerate(sched) if c["q_stride"] > 1] == [2, 5, 21]
    assert U.stage_ends() == [1, 4, 20, 23]
    assert [c["dim_out"] for c in sched] == [112] * 2 + [224] * 3 + [448] * 16 + [896] * 3
    assert [c["heads"] for c in sched] == [2] * 2 + [4] * 3 + [8] * 16 + [16] * 3
    assert [c["mask_unit_attn"] for c in sched] == [True] * 5 + [False] * 19
    # the input generator's table agrees
    assert [(a, b, h) for a, b, h, _, _ in syn.backbone_block_table()] == \
        [(c["dim_in"], c["dim_out"], c["heads"]) for c in sched]


# ----------------------------------------------------------------------------- closed forms
def test_layer_norm_closed_form():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((50, 112)) * 3 + 2
    y = U.layer_norm(x, np.ones(112), np.zeros(112))
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    var = x.var(-1)
    np.testing.assert_allclose((y ** 2).mean(-1), var / (var + 1e-6), rtol=1e-12)
    # affine: y' = y * w + b
    w, b = rng.standard_normal(112), rng.standard_normal(112)
    np.testing.assert_allclose(U.layer_norm(x, w, b), y * w + b, rtol=1e-12, atol=1e-12)


def test_gelu_against_normal_cdf():
    x = np.linspace(-8, 8, 1001)
    # 1 + erf(x / sqrt 2) cancels in the far negative tail, so compare absolutely there
    np.testing.assert_allclose(U.gelu(x), x * norm.cdf(x), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(U.gelu(np.array([1.0])), [norm.cdf(1.0)], rtol=1e-14)
    assert U.gelu(np.array([0.0]))[0] == 0.0


def test_softmax_rows_sum_to_one_and_shift_invariant():
    s = np.random.default_rng(8).standard_normal((7, 33)) * 30
    p = U.softmax_rows(s)
    np.testing.assert_allclose(p.sum(-1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(U.softmax_rows(s + 100.0), p, rtol=1e-12)
    assert (p > 0).all()


def test_two_key_attention_closed_form():
    """One query, two keys, values e0 and e1: the output is (sigmoid(D/sqrt(hd)),
    1 - sigmoid(D/sqrt(hd))) with D the score difference; this fixes the scale and
    that the softmax runs over keys."""
    hd = 4
    # qkv weight builds q = x[0:4], k = x[4:8] for token 0 and 1, v = x[8:12]
    xn = np.zeros((1, 2, 12))
    xn[0, 0, 0:4] = [1.0, 0.5, 0.0, 0.0]       # query of token 0
    xn[0, 0, 4:8] = [2.0, 0.0, 0.0, 0.0]       # key of token 0
    xn[0, 1, 4:8] = [0.0, 1.0, 1.0, 0.0]       # key of token 1
    xn[0, 0, 8:12] = [1.0, 0.0, 0.0, 0.0]
    xn[0, 1, 8:12] = [0.0, 1.0, 0.0, 0.0]
    W = np.eye(12)
    o = U.mask_unit_attention(xn, W, np.zeros(12), np.eye(4), np.zeros(4), 1, 1, 2, False,
                              head_dim=hd)
    D = (1.0 * 2.0) - (0.5 * 1.0)
    a = 1.0 / (1.0 + math.exp(-D / math.sqrt(hd)))
    np.testing.assert_allclose(o[0, 0], [a, 1 - a, 0, 0], rtol=1e-14, atol=1e-15)


def test_all_zero_block_is_identity():
    p = syn.block_params(9, 112, 112, False, dtype="f32")
    p = {k: np.zeros_like(v) for k, v in p.items()}
    x = np.random.default_rng(9).standard_normal((2, 128, 112))
    y = U.block_forward(x, p, 2, 1, 64, True)
    np.testing.assert_array_equal(y, x)


def test_in_window_permutation_equivariance():
    """Permuting the tokens of one window (non-pooled block) permutes the output alike."""
    rng = np.random.default_rng(10)
    p = _tiny_block(13, 8, 8, False)
    N, nW = 64, 4
    x = rng.standard_normal((1, N, 8))
    y = U.block_forward(x, p, 2, 1, N // nW, True, head_dim=4)
    w = 1
    idx = np.arange(N)
    members = idx[w::nW]
    perm = idx.copy()
    perm[members] = members[rng.permutation(len(members))]
    y2 = U.block_forward(x[:, perm], p, 2, 1, N // nW, True, head_dim=4)
    np.testing.assert_allclose(y2, y[:, perm], rtol=1e-12, atol=1e-12)
    # and a token of another window is unaffected by that permutation
    np.testing.assert_allclose(y2[:, 0], y[:, 0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("case", [
    (2, 64, 8, 8, 2, 1, 16, True), (2, 64, 6, 8, 2, 4, 16, True), (1, 64, 8, 8, 2, 1, 64, False),
    (2, 64, 6, 8, 2, 4, 64, False)])
def test_block_rows_matches_full_block(case):
    """The per-row evaluation used for large sampled checks equals the full block."""
    B, N, d_in, d_out, heads, qs, window, mua = case
    p = _tiny_block(14, d_in, d_out, d_in != d_out)
    x = np.random.default_rng(15).standard_normal((B, N, d_in))
    full = U.block_forward(x, p, heads, qs, window, mua, head_dim=4)
    rows = [(b, n) for b in range(B) for n in range(0, N // qs, 3)]
    part = U.block_forward_rows(x, p, heads, qs, window, mua, rows, head_dim=4)
    for r, (b, n) in enumerate(rows):
        np.testing.assert_allclose(part[r], full[b, n], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("row_chunk", [1, 7, 64, 99])
def test_row_chunked_attention_equals_unchunked(row_chunk):
    """The row-chunked evaluation used for the 2048^2 global stages is the same definition:
    each query row's softmax involves only its own scores (ragged last chunk included)."""
    rng = np.random.default_rng(16)
    q = rng.standard_normal((2, 3, 1, 100, 8)) * 2
    k = rng.standard_normal((2, 3, 1, 130, 8)) * 2
    v = rng.standard_normal((2, 3, 1, 130, 8))
    full = U.attention_core(q, k, v, 8)
    part = U.attention_core(q, k, v, 8, row_chunk=row_chunk)
    np.testing.assert_allclose(part, full, rtol=1e-12, atol=1e-14)   # summation order only


def test_backbone_row_chunk_equals_plain():
    p = syn.backbone_params(17, 64, dtype="f32", affine="random")
    x = syn.image(17, 1, 64)
    for a, b in zip(U.backbone_forward(x, p), U.backbone_forward(x, p, row_chunk=3)):
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-13)


def test_attention_heads_is_mask_unit_attention_before_proj():
    """attention_heads (compared per unit against the GPU's attention output) composes with
    the proj Linear into MaskUnitAttention."""
    rng = np.random.default_rng(18)
    xn = rng.standard_normal((2, 64, 8))
    p = _tiny_block(19, 8, 8, False)
    o = U.attention_heads(xn, p["qkv_w"], p["qkv_b"], 2, 4, 16, True, head_dim=4)
    a = U.mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"], p["attn_proj_b"],
                              2, 4, 16, True, head_dim=4)
    np.testing.assert_allclose(U.linear(o, p["attn_proj_w"], p["attn_proj_b"]), a,
                               rtol=1e-13, atol=1e-14)
