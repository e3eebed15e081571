"""Formulation S of the oracle: the same Hiera network restated on NHWC grids.

TEST INFRASTRUCTURE ONLY (see the package docstring). float64 numpy throughout.

It never builds the unrolled token order. Instead, following the meaning the
"Phase 4: Hiera Backbone MLX Port" plan gives the pieces (Architecture Summary):
  * a mask unit is a square tile of the token grid: 8x8 tokens at stage 0
    (window=64), 4x4 at stage 1 (window=16);
  * a stage transition (blocks 2, 5, 21) reduces tokens 4x: here a 2x2 spatial
    max-pool, applied both to the projected residual and to the queries;
  * global attention (stages 2-3) attends over the whole grid;
  * features at the stage ends are the grids themselves (already NHWC).

Because attention is permutation-equivariant and LayerNorm / Linear / MLP act per
token, this must equal Reroll of formulation U at every stage end.
"""

from __future__ import annotations

import math

import numpy as np
from scipy.special import erf

EPS = 1e-6
HD = 56
DEPTHS = (2, 3, 16, 3)
DIMS = (112, 224, 448, 896)
HEADS = (2, 4, 8, 16)


def _ln(x, w, b, eps=EPS):
    x = np.asarray(x, dtype=np.float64)
    return (x - x.mean(-1, keepdims=True)) / np.sqrt(x.var(-1, keepdims=True) + eps) * w + b


def _lin(x, w, b):
    return np.einsum("...i,oi->...o", np.asarray(x, np.float64), np.asarray(w, np.float64)) + b


def _gelu(x):
    return x * 0.5 * (1.0 + erf(x / math.sqrt(2.0)))


def _pool2x2(g):
    """[B, H, W, C] -> [B, H/2, W/2, C], max over each 2x2 cell."""
    B, H, W, C = g.shape
    return g.reshape(B, H // 2, 2, W // 2, 2, C).max(axis=(2, 4))


def _attend(q, k, v):
    """q [n_q, h, hd], k/v [n_k, h, hd] -> [n_q, h, hd]."""
    hd = q.shape[-1]
    s = np.einsum("qhd,khd->hqk", q, k) / math.sqrt(hd)
    s = np.exp(s - s.max(-1, keepdims=True))
    s = s / s.sum(-1, keepdims=True)
    return np.einsum("hqk,khd->qhd", s, v)


def spatial_attention(xn, p, heads, pool, tile, hd=HD):
    """Attention on a grid. xn [B, G, G, d_in]; tile = mask-unit side on this (input)
    grid, or None for global; pool = 2 pools queries 2x2. Returns [B, G/pool, G/pool, d_out]."""
    B, G, _, _ = xn.shape
    d_out = p["attn_proj_w"].shape[0]
    qkv = _lin(xn, p["qkv_w"], p["qkv_b"])                  # [B, G, G, 3 d_out]
    q = qkv[..., :d_out]
    k = qkv[..., d_out:2 * d_out]
    v = qkv[..., 2 * d_out:]
    if pool == 2:
        q = _pool2x2(q)
    Gq = G // pool
    out = np.zeros((B, Gq, Gq, d_out))
    t_k = G if tile is None else tile
    t_q = t_k // pool
    for b in range(B):
        for ty in range(G // t_k):
            for tx in range(G // t_k):
                kk = k[b, ty * t_k:(ty + 1) * t_k, tx * t_k:(tx + 1) * t_k].reshape(-1, heads, hd)
                vv = v[b, ty * t_k:(ty + 1) * t_k, tx * t_k:(tx + 1) * t_k].reshape(-1, heads, hd)
                qq = q[b, ty * t_q:(ty + 1) * t_q, tx * t_q:(tx + 1) * t_q].reshape(-1, heads, hd)
                o = _attend(qq, kk, vv).reshape(t_q, t_q, d_out)
                out[b, ty * t_q:(ty + 1) * t_q, tx * t_q:(tx + 1) * t_q] = o
    return _lin(out, p["attn_proj_w"], p["attn_proj_b"])


def spatial_block(x, p, heads, pool, tile, hd=HD):
    """One block on an NHWC grid; pool = 2 at a stage transition."""
    xn = _ln(x, p["norm1_w"], p["norm1_b"])
    if pool == 2:
        x = _pool2x2(_lin(xn, p["proj_w"], p["proj_b"]))
    x = x + spatial_attention(xn, p, heads, pool, tile, hd)
    h = _ln(x, p["norm2_w"], p["norm2_b"])
    return x + _lin(_gelu(_lin(h, p["fc1_w"], p["fc1_b"])), p["fc2_w"], p["fc2_b"])


def spatial_patch_embed(img, w, b, stride=4, pad=3):
    """Direct convolution as a sum over the 49 kernel taps (no im2col)."""
    img = np.asarray(img, np.float64)
    B, H, W, _ = img.shape
    cout, kh, kw, _ = w.shape
    Ho = (H + 2 * pad - kh) // stride + 1
    Wo = (W + 2 * pad - kw) // stride + 1
    pimg = np.pad(img, ((0, 0), (pad, pad), (pad, pad), (0, 0)))
    out = np.zeros((B, Ho, Wo, cout)) + b
    for ky in range(kh):
        for kx in range(kw):
            tap = pimg[:, ky:ky + stride * (Ho - 1) + 1:stride, kx:kx + stride * (Wo - 1) + 1:stride]
            out += np.einsum("bhwc,oc->bhwo", tap, np.asarray(w[:, ky, kx, :], np.float64))
    return out


def spatial_backbone(img, params, mask_unit_flags=None):
    """Four NHWC features of Hiera-B+ computed on grids."""
    x = spatial_patch_embed(img, params["patch_w"], params["patch_b"])
    B, G, _, C = x.shape
    x = x + np.asarray(params["pos_embed"], np.float64).reshape(G, G, C)
    feats = []
    i = 0
    for s, depth in enumerate(DEPTHS):
        for j in range(depth):
            pool = 2 if (s > 0 and j == 0) else 1
            mu_flag = (s < 2) if mask_unit_flags is None else mask_unit_flags[i]
            # mask-unit side on this block's input grid: 8 at stage 0; the unit keeps its
            # spatial extent through a pooling block and shrinks 2x per pooled stage.
            tile = (8 >> max(s - 1, 0)) if pool == 2 else (8 >> s)
            x = spatial_block(x, params["blocks"][i], HEADS[s], pool, tile if mu_flag else None)
            i += 1
        feats.append(x)
    return feats
