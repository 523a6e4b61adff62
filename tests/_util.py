"""Helpers shared by the parity tests: move a seeded input draw to the GPU, compare with the
oracle, and measure the error the way the tolerance is stated (max over (batch, head) slices of
the relative L2 error)."""
from __future__ import annotations

import numpy as np

TOL = {"f32": 1e-4, "bf16": 1e-2}


def torch_inputs(inp, device):
    import torch
    xdt = torch.bfloat16 if inp.w.dtype == "bf16" else torch.float32

    def t(a, dtype=torch.float32):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device).to(dtype)

    return dict(x=t(inp.x, xdt), dt=t(inp.dt), A=t(inp.A), B=t(inp.B, xdt), C=t(inp.C, xdt),
                D=t(inp.D), init_state=t(inp.init))


def to_np(t):
    return t.detach().float().cpu().numpy()


def rel_l2(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def max_rel_per_pair(gpu_slices, ref_slices):
    """Max over the leading axis (one (batch, head) pair per entry) of the relative L2 error."""
    return max(rel_l2(np.asarray(g, np.float64), np.asarray(r, np.float64))
               for g, r in zip(gpu_slices, ref_slices))


def spread_pairs(batch, nheads, n, seed=0):
    """n (batch, head) pairs covering the corners and a random spread in between."""
    rng = np.random.default_rng(seed)
    pairs = {(0, 0), (batch - 1, nheads - 1), (0, nheads - 1), (batch - 1, 0)}
    while len(pairs) < min(n, batch * nheads):
        pairs.add((int(rng.integers(batch)), int(rng.integers(nheads))))
    return sorted(pairs)


def max_rel_slices(gpu, ref, reduce_axes):
    """Max relative L2 error over slices, vectorised: the norms are taken over `reduce_axes` of
    the two equally shaped arrays and the worst slice is returned (with its index)."""
    g = np.asarray(gpu, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    num = np.sqrt(np.sum((g - r) ** 2, axis=reduce_axes))
    den = np.maximum(np.sqrt(np.sum(r ** 2, axis=reduce_axes)), 1e-30)
    rel = num / den
    i = int(np.argmax(rel))
    return float(rel.flat[i]), np.unravel_index(i, rel.shape)

