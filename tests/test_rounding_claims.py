"""Two bf16 rounding facts the tensor-core path relies on, checked in numpy (CPU).

1. Transition pooling ("Phase 4: Hiera Backbone MLX Port", MaskUnitAttention: q max-pooled
   over the q_stride axis; Stage transitions: residual proj + max-pool). The GEMM epilogue
   rounds the four pooling candidates to bf16 first and takes their max afterwards, on the
   packed values. That equals rounding the fp32 max, because round-to-nearest-even is
   monotonic: a <= b implies rne(a) <= rne(b).
2. Softmax weights cut to bf16 by truncation. The tcgen05 attention truncates P, and the
   denominator is the sum of the same bf16 weights (a ones row in V^T). For flat rows
   (many comparable weights) the mean truncation error then cancels in the normalised
   output, and the error matches round-to-nearest's. For peaked rows (a few weights
   dominate) it does not fully cancel, and the error is about twice round-to-nearest's.
   Both stay near 2e-3 rel-L2, far inside the block tolerance (rel-L2 1e-2).
"""

import numpy as np
import pytest


def bf16_rne(x):
    b = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32)


def bf16_trunc(x):
    return (np.asarray(x, np.float32).view(np.uint32) & np.uint32(0xFFFF0000)).view(np.float32)


def test_bf16_rne_helper_known_values():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7: even mantissa (1.0) wins; just above rounds up
    assert bf16_rne(np.float32(1.0 + 2.0 ** -8)) == np.float32(1.0)
    assert bf16_rne(np.float32(1.0 + 2.0 ** -8 + 2.0 ** -20)) == np.float32(1.0 + 2.0 ** -7)
    # 1 + 3 * 2^-8 is a tie between 1 + 2^-7 (odd) and 1 + 2^-6 (even): rounds up
    assert bf16_rne(np.float32(1.0 + 3 * 2.0 ** -8)) == np.float32(1.0 + 2.0 ** -6)
    assert bf16_trunc(np.float32(1.0 + 2.0 ** -7 + 2.0 ** -9)) == np.float32(1.0 + 2.0 ** -7)


@pytest.mark.parametrize("scale", [1e-3, 1.0, 300.0])
def test_max_of_rounded_candidates_is_rounded_max(scale):
    rng = np.random.default_rng(7)
    c = (rng.standard_normal((200000, 4)) * scale).astype(np.float32)
    # adversarial rows: candidates that straddle or sit on bf16 rounding ties
    base = bf16_rne(rng.standard_normal(2000).astype(np.float32) * scale)
    ulp = np.abs(base) * 2.0 ** -8
    ties = np.stack([base + ulp * f for f in (0.5, 0.49, 0.51, -0.5)], axis=1).astype(np.float32)
    c = np.concatenate([c, ties])
    pooled_then_rounded = bf16_rne(c.max(axis=1))
    rounded_then_pooled = bf16_rne(c).max(axis=1)
    assert np.array_equal(pooled_then_rounded.view(np.uint32) & 0x7FFFFFFF,
                          rounded_then_pooled.view(np.uint32) & 0x7FFFFFFF)
    assert np.array_equal(pooled_then_rounded, rounded_then_pooled)


@pytest.mark.parametrize("sigma", [0.3, 1.0, 3.0, 6.0])
def test_truncated_softmax_weights_stay_at_rounding_accuracy(sigma):
    rng = np.random.default_rng(11)
    rows, keys, d = 256, 1024, 56
    s = rng.normal(0.0, sigma, (rows, keys))
    v = bf16_rne(rng.normal(0.0, 1.0, (keys, d)).astype(np.float32)).astype(np.float64)
    p = np.exp2((s - s.max(axis=1, keepdims=True)) * np.log2(np.e)).astype(np.float32)
    exact = (p.astype(np.float64) @ v) / p.astype(np.float64).sum(axis=1, keepdims=True)

    def rel_err(round_fn):
        pb = round_fn(p).astype(np.float64)
        o = (pb @ v) / pb.sum(axis=1, keepdims=True)  # denominator from the same weights
        return np.linalg.norm(o - exact) / np.linalg.norm(exact)

    e_trunc, e_rne = rel_err(bf16_trunc), rel_err(bf16_rne)
    assert e_trunc <= 2.5e-3
    assert e_trunc <= 2.5 * e_rne
    if sigma <= 1.0:
        # flat rows: the matching denominator cancels the truncation bias (the error is
        # round-to-nearest's), while an unrounded denominator would keep it
        assert e_trunc <= 1.3 * e_rne
        pb = bf16_trunc(p).astype(np.float64)
        biased = (pb @ v) / p.astype(np.float64).sum(axis=1, keepdims=True)
        e_biased = np.linalg.norm(biased - exact) / np.linalg.norm(exact)
        assert e_biased > 1.5 * e_trunc
