"""CPU float64 oracle for the SSD layer scan -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference legs may
import this package.  It wraps ``ssd_oracle.c`` (the token-by-token recurrence, see that file for
the definition and its sources) through ctypes and never touches the CUDA library.

Parity status: pinned.  ``tests/test_oracle_pins.py`` checks it against:

- the explicit semiseparable matrix form on tiny inputs;
- a hand-worked example;
- closed forms for N = P = 1;
- the low-rank property of off-diagonal blocks;
- invariances (dt = 0 padding, split/resume, linearity).

The block, varlen and decode variants are pinned by closed forms and by equalities with the
pinned scan.  The backward (``ssd_scan_bwd``) is pinned element by element against central
differences of the forward, and against a one-token closed form.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libssd_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fused multiply-add) if the library is missing or stale."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-std=c11", "-shared",
                    "-fPIC", _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.oracle_ssd_scan.restype = ctypes.c_int
        lib.oracle_ssd_scan.argtypes = [_I64] * 6 + [_D] * 6 + [_D, _D, _D, _D, _I64, _I64,
                                                                 ctypes.POINTER(_I64), _I64]
        lib.oracle_ssd_scan_bwd.restype = ctypes.c_int
        lib.oracle_ssd_scan_bwd.argtypes = [_I64] * 6 + [_D] * 16
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_num_threads.argtypes = []
        _lib = lib
    return _lib


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_D)


def ssd_scan(x, dt, A, B, C, D, init=None, every: int = 0,
             bh: Optional[Sequence[int]] = None):
    """Token-by-token SSD recurrence in float64.

    x (b, L, H, P), dt (b, L, H), A (H,), B/C (b, L, G, N), D (H,), init (b, H, P, N) or None.
    Returns (y (b, L, H, P), final_state (b, H, P, N), boundary) where boundary holds the state
    after every ``every``-th token, shape (b, H, L // every, P, N), or None when every == 0.
    With ``bh`` only the listed flattened b*H + h pairs are computed (others stay zero).
    """
    x, dt, A, B, C, D, init = map(_f64, (x, dt, A, B, C, D, init))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,) and D.shape == (H,)
    assert B.shape == (b, L, G, N) and C.shape == (b, L, G, N)
    assert init is None or init.shape == (b, H, P, N)
    y = np.zeros((b, L, H, P))
    final = np.zeros((b, H, P, N))
    nb = L // every if every > 0 else 0
    boundary = np.zeros((b, H, nb, P, N)) if every > 0 else None
    idx = None if bh is None else np.ascontiguousarray(bh, dtype=np.int64)
    rc = _load().oracle_ssd_scan(
        b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init),
        _ptr(y), _ptr(final), _ptr(boundary), every, nb,
        None if idx is None else idx.ctypes.data_as(ctypes.POINTER(_I64)),
        0 if idx is None else len(idx))
    if rc != 0:
        raise RuntimeError("oracle_ssd_scan rejected its arguments")
    return y, final, boundary


def ssd_scan_pairs(inp, pairs: Sequence[Tuple[int, int]], every: int = 0,
                   seqlen: Optional[int] = None):
    """Recurrence for selected (batch, head) pairs of a full-size input draw.

    The selected pairs are gathered (pure re-indexing, no arithmetic) into one batch whose
    "heads" are the pairs, each with its own group, so only those slices are widened to float64.
    Returns y (n, L, P), final (n, P, N) and the boundary states (n, nb, P, N) or None.
    """
    H = inp.A.shape[0]
    G = inp.B.shape[2]
    L = inp.x.shape[1] if seqlen is None else seqlen
    bs = np.array([p[0] for p in pairs], dtype=np.int64)
    hs = np.array([p[1] for p in pairs], dtype=np.int64)
    gs = hs // (H // G)
    x = np.stack([inp.x[b, :L, h] for b, h in pairs], 1)
    dt = np.stack([inp.dt[b, :L, h] for b, h in pairs], 1)
    Bv = np.stack([inp.B[b, :L, g] for b, g in zip(bs, gs)], 1)
    Cv = np.stack([inp.C[b, :L, g] for b, g in zip(bs, gs)], 1)
    init = None
    if inp.init is not None:
        init = np.stack([inp.init[b, h] for b, h in pairs], 0)[None]
    y, final, boundary = ssd_scan(x[None], dt[None], inp.A[hs], Bv[None], Cv[None], inp.D[hs],
                                  init, every=every)
    y = np.moveaxis(y[0], 1, 0)                      # (n, L, P)
    return y, final[0], (None if boundary is None else boundary[0])


def dt_prologue(dt, dt_bias=None, softplus: bool = False, dt_limit=None):
    """The dt the scan uses when the block's raw projection is passed: dt + dt_bias, then
    softplus(v) = log(1 + exp(v)) when asked, then clamped to dt_limit = (lo, hi) when given
    (mohakchugh.is-a.dev "Mamba-2", Architecture: Multi-Head SSM).  float64."""
    v = np.asarray(dt, dtype=np.float64)
    if dt_bias is not None:
        v = v + np.asarray(dt_bias, dtype=np.float64)
    if softplus:
        v = np.logaddexp(0.0, v)
    if dt_limit is not None:
        v = np.clip(v, dt_limit[0], dt_limit[1])
    return v


def ssd_scan_block(x, dt, A, B, C, D, init=None, z=None, dt_bias=None, softplus: bool = False,
                   dt_limit=None):
    """The scan with the Mamba-2 block's elementwise steps around it: the dt prologue above,
    then the recurrence, then the output gated by SiLU(z) = z / (1 + exp(-z)) (same page, the
    gated output of the block).  Returns (y, final_state)."""
    dt_eff = dt_prologue(dt, dt_bias, softplus, dt_limit)
    y, final, _ = ssd_scan(x, dt_eff, A, B, C, D, init)
    if z is not None:
        zf = np.asarray(z, dtype=np.float64)
        y = y * (zf / (1.0 + np.exp(-zf)))
    return y, final


def ssd_state_update_block(state, x, dt, A, B, C, D, z=None, dt_bias=None,
                           softplus: bool = False, dt_limit=None):
    """One decode step with the block's steps around it: the dt prologue, the recurrence over the
    token, the SiLU(z) gate.  x, z (b, H, P), dt (b, H).  Returns (y, new_state)."""
    dt_eff = dt_prologue(dt, dt_bias, softplus, dt_limit)
    y, new_state = ssd_state_update(state, x, dt_eff, A, B, C, D)
    if z is not None:
        zf = np.asarray(z, dtype=np.float64)
        y = y * (zf / (1.0 + np.exp(-zf)))
    return y, new_state


def ssd_scan_bwd(x, dt, A, B, C, D, dy, init=None, dfinal=None):
    """Gradients of L = sum_t <dy_t, y_t> + <dfinal, final_state> through the recurrence, by the
    adjoint recurrence (reverse-mode differentiation of the token loop, float64, in
    ``ssd_oracle.c``, ``oracle_ssd_scan_bwd``):

        g_t = dy_t (outer) C_t + a_{t+1} g_{t+1}           (g_{L-1} also gets dfinal)
        dx_t = D_h dy_t + dt_t g_t B_t                      dB_t += dt_t g_t^T x_t  (per group)
        dC_t += h_t^T dy_t  (per group)                     dD_h = sum_t <dy_t, x_t>
        dl_t = a_t <g_t, h_{t-1}>   (l_t = dt_t A_h)        ddt_t = <g_t B_t, x_t> + A_h dl_t
        dA_h = sum_t dt_t dl_t                              dinit = a_0 g_0

    The C loop gives each head's share of dB, dC, dA and dD; the group sums over heads and the
    batch sums are numpy sums here.

    x (b, L, H, P), dt (b, L, H), B/C (b, L, G, N), dy like x, init/dfinal (b, H, P, N) or None.
    Returns dict dx, ddt, dA, dB, dC, dD, dinit."""
    x, dt, A, B, C, D, dy, init, dfinal = map(_f64, (x, dt, A, B, C, D, dy, init, dfinal))
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    assert dt.shape == (b, L, H) and A.shape == (H,) and D.shape == (H,) and dy.shape == x.shape
    assert B.shape == (b, L, G, N) and C.shape == (b, L, G, N)
    assert init is None or init.shape == (b, H, P, N)
    assert dfinal is None or dfinal.shape == (b, H, P, N)
    dx = np.zeros_like(x)
    ddt = np.zeros_like(dt)
    dB_h = np.zeros((b, L, H, N))
    dC_h = np.zeros((b, L, H, N))
    dA_bh = np.zeros((b, H))
    dD_bh = np.zeros((b, H))
    dinit = np.zeros((b, H, P, N))
    rc = _load().oracle_ssd_scan_bwd(
        b, L, H, P, N, G, _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init),
        _ptr(dy), _ptr(dfinal), _ptr(dx), _ptr(ddt), _ptr(dB_h), _ptr(dC_h), _ptr(dA_bh),
        _ptr(dD_bh), _ptr(dinit))
    if rc != 0:
        raise RuntimeError("oracle_ssd_scan_bwd rejected its arguments")
    hpg = H // G
    return dict(dx=dx, ddt=ddt, dA=dA_bh.sum(0), dD=dD_bh.sum(0),
                dB=dB_h.reshape(b, L, G, hpg, N).sum(3), dC=dC_h.reshape(b, L, G, hpg, N).sum(3),
                dinit=dinit)


def ssd_scan_varlen(x, dt, A, B, C, D, cu_seqlens, init=None):
    """Packed variable-length sequences: sequence s (tokens cu_seqlens[s] .. cu_seqlens[s+1]-1
    of the single batch row) is its own recurrence, started from init[s] (or zeros), so this is
    the token-by-token oracle applied to each sequence separately.

    x (1, T, H, P) etc., cu_seqlens (nseq + 1,), init (nseq, H, P, N) or None.
    Returns (y (1, T, H, P), final (nseq, H, P, N)).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nseq = len(cu) - 1
    _, T, H, P = x.shape
    N = B.shape[3]
    y = np.zeros((1, T, H, P))
    final = np.zeros((nseq, H, P, N))
    for s in range(nseq):
        a, e = int(cu[s]), int(cu[s + 1])
        h0 = None if init is None else init[s:s + 1]
        if e == a:
            final[s] = 0.0 if h0 is None else h0[0]
            continue
        ys, fs, _ = ssd_scan(x[:, a:e], dt[:, a:e], A, B[:, a:e], C[:, a:e], D, h0)
        y[:, a:e] = ys
        final[s] = fs[0]
    return y, final


def ssd_state_update(state, x, dt, A, B, C, D):
    """One decode step: the recurrence over a single token, state (b, H, P, N) updated and returned.

    x (b, H, P), dt (b, H), B/C (b, G, N).  Returns (y (b, H, P), new_state).
    """
    x = np.asarray(x)
    y, final, _ = ssd_scan(x[:, None], np.asarray(dt)[:, None], A, np.asarray(B)[:, None],
                           np.asarray(C)[:, None], D, init=state)
    return y[:, 0], final
