"""Seeded synthetic inputs for the SSD layer scan (shared by the CUDA path's tests and the oracle).

This module only draws random numbers and rounds them to the storage type; it holds none of the
scan's arithmetic.  Draw order and distributions, all from one numpy PCG64 stream seeded with the
workload's seed:

    x  ~ N(0, 1)                                  (b, L, H, P)
    dt = clamp(softplus(N(0, 1) - 4), 1e-3, 0.1)  (b, L, H)      already positive: the kernels
                                                                   take dt after softplus/clamp
    A_h = -exp(U(0, ln 16))                       (H,)           so exp(dt*A) lies in (0, 1)
    B, C ~ N(0, 1) / sqrt(N)                      (b, L, G, N)
    D  ~ N(0, 1)                                  (H,)
    h0 ~ N(0, 0.1^2)                              (b, H, P, N)   only when the workload has one
                                                  ((nseq, H, P, N) for packed sequences)
    cu_seqlens: nseq - 1 distinct cut points drawn uniformly from 1 .. L-1, sorted, with 0 and
                L added (packed variable-length workloads only; drawn last)

Values are drawn in float32; x, B and C are then rounded to bfloat16 (round to nearest even) for
bf16 workloads, and every consumer reads the rounded values, so the oracle sees exactly what the
GPU sees.  The input-dependent B, C and dt follow the selection mechanism of Mamba
(mohakchugh.is-a.dev "Mamba-2", Mamba-1: Selective State Spaces); A_h < 0 is a per-head scalar
decay (chipfoundryservices.com "hybrid attention-SSM", scalar-times-identity transition).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from .configs import Workload


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); returns the 16-bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """float32 array holding exactly the bfloat16-rounded values of ``a``."""
    return bf16_bits_to_f32(bf16_bits(a))


@dataclass
class SSDInputs:
    """One draw of the layer's inputs.  Arrays are float32 holding the exact stored values."""
    w: Workload
    x: np.ndarray
    dt: np.ndarray
    A: np.ndarray
    B: np.ndarray
    C: np.ndarray
    D: np.ndarray
    init: Optional[np.ndarray]
    cu_seqlens: Optional[np.ndarray] = None   # int32 (nseq + 1,) for packed sequences


@dataclass
class BlockInputs:
    """The Mamba-2 block's raw projections around the scan (float32, exact stored values)."""
    z: np.ndarray          # gate, (b, L, H, P), rounded to bf16 for bf16 workloads
    dt_raw: np.ndarray     # dt projection before bias / softplus / clamp, (b, L, H)
    dt_bias: np.ndarray    # (H,)
    dt_limit: tuple        # clamp after the softplus


def make_block_inputs(w: Workload, seed: Optional[int] = None) -> BlockInputs:
    """z ~ N(0, 1); dt_raw ~ N(0, 1); dt_bias_h = -4 + U(-0.5, 0.5); clamp (1e-3, 0.1), so that
    softplus(dt_raw + dt_bias) matches the dt recipe above.  Drawn from its own PCG64 stream
    (seed + 500) so the scan inputs of the same workload are unchanged."""
    rng = np.random.Generator(np.random.PCG64((w.seed if seed is None else seed) + 500))
    b, L, H, P = w.batch, w.seqlen, w.nheads, w.headdim
    z = rng.standard_normal((b, L, H, P), dtype=np.float32)
    dt_raw = rng.standard_normal((b, L, H), dtype=np.float32)
    dt_bias = (-4.0 + rng.uniform(-0.5, 0.5, H)).astype(np.float32)
    if w.dtype == "bf16":
        z = round_bf16(z)
    return BlockInputs(z, dt_raw, dt_bias, (1e-3, 0.1))


@dataclass
class GradInputs:
    """Upstream gradients for the backward pass (float32, exact stored values)."""
    dy: np.ndarray         # like y, (b, L, H, P), rounded to bf16 for bf16 workloads
    dfinal: np.ndarray     # like the final state, (b, H, P, N)


def make_grad_inputs(w: Workload, seed: Optional[int] = None) -> GradInputs:
    """dy ~ N(0, 1) and dfinal ~ 0.1 N(0, 1), from their own PCG64 stream (seed + 700)."""
    rng = np.random.Generator(np.random.PCG64((w.seed if seed is None else seed) + 700))
    b, L, H, P, N = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate
    dy = rng.standard_normal((b, L, H, P), dtype=np.float32)
    dfinal = (0.1 * rng.standard_normal((b, H, P, N), dtype=np.float32)).astype(np.float32)
    if w.dtype == "bf16":
        dy = round_bf16(dy)
    return GradInputs(dy, dfinal)


def make_inputs(w: Workload, seed: Optional[int] = None) -> SSDInputs:
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    x = rng.standard_normal((b, L, H, P), dtype=np.float32)
    z = rng.standard_normal((b, L, H), dtype=np.float32).astype(np.float64) - 4.0
    dt = np.clip(np.log1p(np.exp(z)), 1e-3, 0.1).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, np.log(16.0), H))).astype(np.float32)
    inv = np.float32(1.0 / np.sqrt(N))
    B = rng.standard_normal((b, L, G, N), dtype=np.float32) * inv
    C = rng.standard_normal((b, L, G, N), dtype=np.float32) * inv
    D = rng.standard_normal(H, dtype=np.float32)
    init = None
    ns = w.nseq if w.nseq > 0 else b
    if w.init_state:
        init = rng.standard_normal((ns, H, P, N), dtype=np.float32) * np.float32(0.1)
    cu = None
    if w.nseq > 0:
        if b != 1 or w.nseq > L:
            raise ValueError("packed sequences need batch 1 and at most one sequence per token")
        cuts = np.sort(rng.choice(np.arange(1, L), size=w.nseq - 1, replace=False))
        cu = np.concatenate([[0], cuts, [L]]).astype(np.int32)
    if w.dtype == "bf16":
        x, B, C = round_bf16(x), round_bf16(B), round_bf16(C)
    elif w.dtype != "f32":
        raise ValueError(f"unknown dtype {w.dtype!r}")
    return SSDInputs(w, x, dt, A, B, C, D, init, cu)
