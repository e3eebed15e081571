"""The bench's per-launch work model (CPU): the FLOPs it divides by time must be the
algorithmic work of the Hiera-B+ backbone, counted independently here from the stage table
(head dim 56, not the padded 64), whichever way the MLP is launched."""

import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _expected(img, B):
    G0 = img // 4
    dims, depths, heads = (112, 224, 448, 896), (2, 3, 16, 3), (2, 4, 8, 16)
    gemm = attn = 0.0
    prev = dims[0]
    for s, depth in enumerate(depths):
        G = G0 >> s
        for j in range(depth):
            trans = s > 0 and j == 0
            d_in, d = (prev if trans else dims[s]), dims[s]
            n_in = (2 * G) ** 2 if trans else G * G          # tokens entering the block
            n_q = G * G                                      # tokens leaving it
            window = (64 >> (2 * s)) * (4 if trans else 1)   # mask-unit tokens at block input
            n_win = n_in // window if s < 2 else 1
            t_kv = n_in // n_win
            t_q = t_kv // (4 if trans else 1)
            gemm += 2 * n_in * d_in * (3 * d + (d if trans else 0))   # qkv (+ transition proj)
            gemm += 2 * n_q * d * d + 2 * 2 * n_q * d * 4 * d          # attn proj, fc1, fc2
            attn += 2 * 2 * heads[s] * n_win * t_q * t_kv * 56        # QK^T and PV
        prev = dims[s]
    patch = 2 * G0 * G0 * 112 * 196
    return B * gemm, B * attn, B * patch


@pytest.mark.parametrize("fused", [True, False])
def test_launch_flops_total_matches_the_architecture(fused):
    b = _bench()
    launches = b.launch_flops(512, 8, fused_mlp=fused, fused_attn=False)
    got = {}
    for cls, fl in launches:
        got[cls] = got.get(cls, 0.0) + fl
    gemm, attn, patch = _expected(512, 8)
    assert got["gemm"] == pytest.approx(gemm, rel=1e-12)
    assert got["attention"] == pytest.approx(attn, rel=1e-12)
    assert got["patch_embed"] == pytest.approx(patch, rel=1e-12)
    # with the stage-0 attention halves fused, the same total in fewer launches
    fl = b.launch_flops(512, 8, fused_mlp=fused, fused_attn=True)
    assert sum(f for _, f in fl) == pytest.approx(gemm + attn + patch, rel=1e-12)
    assert sum(1 for c, _ in fl if c == "attn_block") == 2
    assert len(fl) == len(launches) - 4
    # per image: 124.5 GF GEMM + 38.4 GF attention + 0.72 GF patch embedding
    assert gemm / 8 / 1e9 == pytest.approx(124.5, abs=0.05)
    assert attn / 8 / 1e9 == pytest.approx(38.4, abs=0.05)
    # launch counts: 24 qkv, 24 attention, 24 proj, MLP 24 x 2 (or 19 x 2 + 5 fused), 4 rerolls
    n_gemm = sum(1 for c, _ in launches if c == "gemm")
    assert n_gemm == (91 if fused else 96)
    assert sum(1 for c, _ in launches if c == "unroll_reroll") == 4


def test_reroll_bytes():
    b = _bench()
    # read + write, bf16, of the four NHWC features of a 512^2 batch of 8
    assert b.reroll_bytes(512, 8) == [2 * 2 * 8 * g * g * c for g, c in
                                      ((128, 112), (64, 224), (32, 448), (16, 896))]
