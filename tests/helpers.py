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
