"""Formulation U of the oracle: the Hiera block and backbone on unrolled tokens.

TEST INFRASTRUCTURE ONLY (see the package docstring). float64 numpy throughout.

Source: "Phase 4: Hiera Backbone MLX Port" (corridorkey-mrp-mlx plan),
section "Architecture Summary" (PatchEmbed, pos_embed, Unroll, the 24 HieraBlocks
in 4 stages, Reroll, stage transitions, MaskUnitAttention, MLP) and section
"Sub-phase 4a: Core backbone module" (unroll, reroll, undo_windowing,
MaskUnitAttention, HieraMLP, HieraBlock, HieraBackbone).

Readings taken where the plan is silent:
  * Unroll order: a stage-s grid of side G with L = 3 - s unroll levels and mask-unit
    grid side M = G / 2^L puts spatial (y, x), y = my*2^L + sum_k a_k 2^(k-1),
    x = mx*2^L + sum_k b_k 2^(k-1), at token
    u = (sum_{k=1..L} (2 a_k + b_k) 4^(L-k)) * M^2 + my*M + mx
    (the finest 2x2 offset is the outermost index; the plan only says the port of
    timm's Unroll is faithful).
  * Window w of token n is n mod nW and its in-window index is n div nW.
  * qkv output channel c splits as (which = c div d_out, head = (c mod d_out) div hd,
    e = c mod hd).
  * The q max-pool and the transition residual pool take the max over the
    q_stride outermost chunks of the token (or in-window) axis.
  * LayerNorm: population variance, eps 1e-6; GELU: exact erf form.
  * Transition residual: proj(norm1(x)) first, then the max-pool.
  * Patch embedding: 7x7 kernel, stride 4, padding 3, with bias, weights OHWI.
"""

from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
from scipy.special import erf
from threadpoolctl import threadpool_limits

LN_EPS = 1e-6
HEAD_DIM = 56
STAGE_DEPTHS = (2, 3, 16, 3)
STAGE_DIMS = (112, 224, 448, 896)
STAGE_HEADS = (2, 4, 8, 16)
MU_SIDE0 = 8          # mask unit = 8x8 tokens at stage 0 (window=64)
UNROLL_LEVELS = 3     # three 2x2 strides, one per stage transition
Q_STRIDE = 4          # 2x2 pooling at blocks 2, 5, 21


def _f64(a):
    return np.asarray(a, dtype=np.float64)


# --------------------------------------------------------------------------- Unroll / Reroll
def unroll_index(G: int, levels: int) -> np.ndarray:
    """u[y, x]: the unrolled token index of spatial (y, x) on a GxG grid.

    "Phase 4: Hiera Backbone MLX Port", Architecture Summary ("Unroll: Permutes tokens
    for mask-unit windowed attention") and Sub-phase 4a item 2; the bit order is the
    reading stated in the module docstring.
    """
    if G % (1 << levels):
        raise ValueError("grid side must be divisible by 2^levels")
    M = G >> levels
    y, x = np.meshgrid(np.arange(G), np.arange(G), indexing="ij")
    offset = np.zeros((G, G), dtype=np.int64)
    for k in range(1, levels + 1):
        a_k = (y >> (k - 1)) & 1
        b_k = (x >> (k - 1)) & 1
        offset += (2 * a_k + b_k) * 4 ** (levels - k)
    mu = (y >> levels) * M + (x >> levels)
    return offset * (M * M) + mu


def unroll(x_raster: np.ndarray, G: int, levels: int) -> np.ndarray:
    """[B, G*G, C] raster tokens -> [B, G*G, C] unrolled tokens."""
    u = unroll_index(G, levels).reshape(-1)
    out = np.empty_like(x_raster)
    out[:, u, :] = x_raster
    return out


def reroll(x_unrolled: np.ndarray, G: int, levels: int) -> np.ndarray:
    """[B, G*G, C] unrolled tokens -> NHWC [B, G, G, C] (Sub-phase 4a items 3-4)."""
    u = unroll_index(G, levels)
    return x_unrolled[:, u, :]


# --------------------------------------------------------------------------- token-wise ops
def layer_norm(x, w, b, eps=LN_EPS):
    """Population-variance LayerNorm over the last axis."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(w) + _f64(b)


def linear(x, w, b):
    """y = x W^T + b with W stored [out, in] (Checkpoint Details: Linear, no transpose)."""
    return _f64(x) @ _f64(w).T + _f64(b)


def gelu(x):
    """Exact GELU, x * Phi(x) with Phi the standard normal CDF written through erf."""
    x = _f64(x)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def mlp(x, fc1_w, fc1_b, fc2_w, fc2_b):
    """HieraMLP: fc1 (dim -> 4 dim) -> GELU -> fc2 (4 dim -> dim) (Architecture Summary, MLP)."""
    return linear(gelu(linear(x, fc1_w, fc1_b)), fc2_w, fc2_b)


def max_pool_tokens(x, stride):
    """Max over the `stride` outermost chunks of the token axis: [B, N, C] -> [B, N/stride, C]."""
    if stride == 1:
        return _f64(x)
    B, N, C = x.shape
    return _f64(x).reshape(B, stride, N // stride, C).max(axis=1)


def softmax_rows(s):
    """Row softmax in the max-subtracted form."""
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


# --------------------------------------------------------------------------- attention
def attention_core(q, k, v, head_dim=HEAD_DIM, row_chunk=None):
    """Scaled dot-product attention over the last two axes ("Architecture Summary",
    MaskUnitAttention: scaled dot-product attention with scale head_dim^-1/2):
    softmax_rows(q k^T / sqrt(head_dim)) v for q [..., Tq, hd], k and v [..., Tkv, hd].

    row_chunk, if given, evaluates that many query rows at a time. Each query row's
    softmax only involves its own scores, so this is the same definition; it bounds the
    host memory of long global attention (16384 queries x 65536 keys at 2048^2)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    scale = 1.0 / math.sqrt(head_dim)
    Tq = q.shape[-2]
    if row_chunk is None or Tq <= row_chunk:
        return softmax_rows((q @ k.swapaxes(-1, -2)) * scale) @ v
    out = np.empty(q.shape[:-1] + (v.shape[-1],))
    kt = k.swapaxes(-1, -2)

    def rows(r0):
        r1 = min(Tq, r0 + row_chunk)
        out[..., r0:r1, :] = softmax_rows((q[..., r0:r1, :] @ kt) * scale) @ v

    # the chunks are independent; numpy releases the GIL inside its kernels, so host
    # threads evaluate several at once, each with a single-threaded BLAS (each chunk's
    # arithmetic is unchanged)
    with threadpool_limits(1, user_api="blas"), \
            ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        list(ex.map(rows, range(0, Tq, row_chunk)))
    return out


def attention_heads(xn, qkv_w, qkv_b, heads, q_stride, window_tokens, mask_unit_attn,
                    head_dim=HEAD_DIM, row_chunk=None):
    """MaskUnitAttention up to the merged heads, before its output proj ("Architecture
    Summary", MaskUnitAttention).

    qkv = Linear(dim_in, 3 dim_out) split per window; at q_stride > 1 the queries are
    max-pooled over the q_stride axis; scaled dot-product attention inside each window;
    heads merged. window_tokens is the number of key tokens per mask-unit window at the
    block input; with mask_unit_attn False there is one window holding every token
    (global). Returns [B, N / q_stride, heads * head_dim], token j*nW + w, channel
    h*head_dim + e.
    """
    B, N, _ = xn.shape
    d_out = heads * head_dim
    nW = N // window_tokens if mask_unit_attn else 1
    T = N // nW
    qkv = linear(xn, qkv_w, qkv_b)                          # [B, N, 3 d_out]
    qkv = qkv.reshape(B, T, nW, 3, heads, head_dim)         # token n = j*nW + w
    qkv = qkv.transpose(3, 0, 4, 2, 1, 5)                   # [3, B, h, nW, T, hd]
    q, k, v = qkv[0], qkv[1], qkv[2]
    if q_stride > 1:
        q = q.reshape(B, heads, nW, q_stride, T // q_stride, head_dim).max(axis=3)
    o = attention_core(q, k, v, head_dim, row_chunk)       # [B, h, nW, Tq, hd]
    Tq = o.shape[3]
    return o.transpose(0, 3, 2, 1, 4).reshape(B, Tq * nW, d_out)   # token j*nW + w


def mask_unit_attention(xn, qkv_w, qkv_b, attn_proj_w, attn_proj_b, heads, q_stride,
                        window_tokens, mask_unit_attn, head_dim=HEAD_DIM, row_chunk=None):
    """MaskUnitAttention ("Architecture Summary", MaskUnitAttention): attention_heads
    followed by proj = Linear(dim_out, dim_out). Returns [B, N / q_stride, dim_out]."""
    d_out = attn_proj_w.shape[0]
    if d_out != heads * head_dim:
        raise ValueError("dim_out must equal heads * head_dim")
    o = attention_heads(xn, qkv_w, qkv_b, heads, q_stride, window_tokens, mask_unit_attn,
                        head_dim, row_chunk)
    return linear(o, attn_proj_w, attn_proj_b)


# --------------------------------------------------------------------------- block
def block_forward(x, p, heads, q_stride, window_tokens, mask_unit_attn, eps=LN_EPS,
                  head_dim=HEAD_DIM, row_chunk=None):
    """HieraBlock (Sub-phase 4a item 7): norm1 -> [proj + max-pool if transition]
    -> attn + residual -> norm2 -> MLP + residual.

    `p` holds numpy arrays keyed norm1_w, norm1_b, qkv_w, qkv_b, [proj_w, proj_b],
    attn_proj_w, attn_proj_b, norm2_w, norm2_b, fc1_w, fc1_b, fc2_w, fc2_b.
    row_chunk: see attention_core.
    """
    x = _f64(x)
    dim_in = x.shape[-1]
    dim_out = p["attn_proj_w"].shape[0]
    xn = layer_norm(x, p["norm1_w"], p["norm1_b"], eps)
    if dim_in != dim_out:
        x = max_pool_tokens(linear(xn, p["proj_w"], p["proj_b"]), q_stride)
    x = x + mask_unit_attention(xn, p["qkv_w"], p["qkv_b"], p["attn_proj_w"],
                                p["attn_proj_b"], heads, q_stride, window_tokens,
                                mask_unit_attn, head_dim, row_chunk)
    x = x + mlp(layer_norm(x, p["norm2_w"], p["norm2_b"], eps), p["fc1_w"], p["fc1_b"],
                p["fc2_w"], p["fc2_b"])
    return x


# --------------------------------------------------------------------------- backbone
def patch_embed(img_nhwc, w_ohwi, b, stride=4, pad=3):
    """HieraPatchEmbed: Conv2d(4 -> 112, 7x7, stride 4) flattened to [B, N, C] in raster
    order (Architecture Summary; the kernel weight is stored (112, 7, 7, 4) per
    Checkpoint Details). Written as an explicit im2col followed by one matmul."""
    img = _f64(img_nhwc)
    B, H, W, Cin = img.shape
    Cout, kh, kw, _ = w_ohwi.shape
    Ho = (H + 2 * pad - kh) // stride + 1
    Wo = (W + 2 * pad - kw) // stride + 1
    padded = np.zeros((B, H + 2 * pad, W + 2 * pad, Cin))
    padded[:, pad:pad + H, pad:pad + W, :] = img
    cols = np.empty((B, Ho, Wo, kh, kw, Cin))
    for ky in range(kh):
        for kx in range(kw):
            cols[:, :, :, ky, kx, :] = padded[:, ky:ky + stride * Ho:stride,
                                              kx:kx + stride * Wo:stride, :]
    out = cols.reshape(B, Ho * Wo, kh * kw * Cin) @ _f64(w_ohwi).reshape(Cout, -1).T
    return out + _f64(b)


def block_schedule():
    """Per-block (dim_in, dim_out, heads, q_stride, stage, mask_unit_attn) of Hiera-B+
    as the Architecture Summary lists the four stages (transitions at blocks 2, 5, 21;
    mask-unit attention in stages 0-1, global attention in stages 2-3)."""
    sched = []
    prev = STAGE_DIMS[0]
    for s, depth in enumerate(STAGE_DEPTHS):
        for i in range(depth):
            transition = s > 0 and i == 0
            sched.append(dict(dim_in=prev if transition else STAGE_DIMS[s],
                              dim_out=STAGE_DIMS[s], heads=STAGE_HEADS[s],
                              q_stride=Q_STRIDE if transition else 1, stage=s,
                              mask_unit_attn=s < 2))
        prev = STAGE_DIMS[s]
    return sched


def stage_ends():
    ends, acc = [], 0
    for d in STAGE_DEPTHS:
        acc += d
        ends.append(acc - 1)
    return ends


def backbone_forward(img_nhwc, params, mask_unit_attn_override=None, row_chunk=None):
    """HieraBackbone (Sub-phase 4a item 8): patch_embed + pos_embed + unroll + 24 blocks
    + reroll at the stage ends [1, 4, 20, 23]. Returns four NHWC features.

    mask_unit_attn_override, if given, is a list of 24 booleans replacing the
    per-block flag (used for the lagged-flag variant). row_chunk: see attention_core."""
    B, H, W, _ = img_nhwc.shape
    G = H // 4
    x = patch_embed(img_nhwc, params["patch_w"], params["patch_b"])
    x = x + _f64(params["pos_embed"])[None]
    x = unroll(x, G, UNROLL_LEVELS)
    mu_tokens = MU_SIDE0 * MU_SIDE0
    feats = []
    ends = stage_ends()
    for i, cfg in enumerate(block_schedule()):
        s = cfg["stage"]
        N = x.shape[1]
        flat_mu = mu_tokens // (4 ** s)          # q tokens per window after this block
        window_tokens = flat_mu * cfg["q_stride"]
        mua = cfg["mask_unit_attn"] if mask_unit_attn_override is None \
            else mask_unit_attn_override[i]
        if mua and N % window_tokens:
            raise ValueError("tokens not divisible into mask units")
        x = block_forward(x, params["blocks"][i], cfg["heads"], cfg["q_stride"],
                          window_tokens, mua, row_chunk=row_chunk)
        if i in ends:
            Gs = G >> s
            feats.append(reroll(x, Gs, UNROLL_LEVELS - s))
    return feats


def block_forward_rows(x, p, heads, q_stride, window_tokens, mask_unit_attn, rows,
                       eps=LN_EPS, head_dim=HEAD_DIM):
    """Output of block_forward for selected output tokens only (for sizes where the full
    attention matrix is too large for the host). `rows` is a list of (b, n_out) pairs with
    n_out indexing the block's output tokens. Same definition as block_forward, evaluated
    one query row at a time: keys and values of the query's window are projected for the
    whole window, the query is max-pooled over the q_stride outermost chunks of the
    window, softmax runs over that window's keys."""
    x = _f64(x)
    B, N, dim_in = x.shape
    d_out = p["attn_proj_w"].shape[0]
    nW = N // window_tokens if mask_unit_attn else 1
    T = N // nW
    Tq = T // q_stride
    out = np.empty((len(rows), d_out))
    cache = {}
    for r, (b, n_out) in enumerate(rows):
        w, jq = n_out % nW, n_out // nW
        key = (b, w)
        if key not in cache:
            toks = np.arange(T) * nW + w                       # window members, j = 0..T-1
            xn = layer_norm(x[b, toks], p["norm1_w"], p["norm1_b"], eps)
            qkv = linear(xn, p["qkv_w"], p["qkv_b"]).reshape(T, 3, heads, head_dim)
            resid = None
            if dim_in != d_out:
                resid = linear(xn, p["proj_w"], p["proj_b"])  # [T, d_out]
            cache = {key: (qkv, resid, toks)}
        qkv, resid, toks = cache[key]
        members = [c * Tq + jq for c in range(q_stride)]      # in-window indices pooled
        q = qkv[members, 0].max(axis=0)                       # [heads, hd]
        k, v = qkv[:, 1], qkv[:, 2]                            # [T, heads, hd]
        o = np.empty((heads, head_dim))
        for h in range(heads):
            s = (k[:, h] @ q[h]) / math.sqrt(head_dim)
            o[h] = softmax_rows(s[None])[0] @ v[:, h]
        a = linear(o.reshape(1, d_out), p["attn_proj_w"], p["attn_proj_b"])[0]
        if dim_in != d_out:
            res = resid[members].max(axis=0)
        else:
            res = x[b, toks[jq]]
        x1 = res + a
        h2 = layer_norm(x1[None], p["norm2_w"], p["norm2_b"], eps)
        out[r] = x1 + mlp(h2, p["fc1_w"], p["fc1_b"], p["fc2_w"], p["fc2_b"])[0]
    return out
