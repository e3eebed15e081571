"""Shared helpers for the tests: device placement and error measures (no arithmetic of
the Hiera block lives here)."""

import numpy as np
import torch

TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}


def dev(a, dtype="bf16"):
    """numpy (already dtype-exact) -> contiguous CUDA tensor of the given dtype."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(
        device="cuda", dtype=TORCH_DT[dtype]).contiguous()


def host(t):
    return t.detach().to(torch.float64).cpu().numpy()


def rel_l2(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm((got - ref).ravel()) / max(np.linalg.norm(ref.ravel()), 1e-300))


def max_abs(got, ref):
    return float(np.max(np.abs(np.asarray(got, np.float64) - np.asarray(ref, np.float64))))


def block_weights_dev(p, dtype):
    return {k: dev(v, dtype) for k, v in p.items()}


def row_rel_l2(got, ref):
    """rel-L2 of every row (last axis) of got against ref."""
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)


def unit_rel_l2(o_got, o_ref, B, Tq, nW, heads, hd=56):
    """rel-L2 of every (image, window, head) unit of a merged attention output
    [B, Tq * nW, heads * hd] (token j * nW + w, channel h * hd + e): [B, nW, heads]."""
    g = np.asarray(o_got, np.float64).reshape(B, Tq, nW, heads, hd)
    r = np.asarray(o_ref, np.float64).reshape(B, Tq, nW, heads, hd)
    num = np.sqrt(((g - r) ** 2).sum(axis=(1, 4)))
    den = np.maximum(np.sqrt((r ** 2).sum(axis=(1, 4))), 1e-30)
    return num / den
