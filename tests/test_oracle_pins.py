"""Pins for the CPU oracle: checks against what the pages and the mathematics fix, not against itself.

Each test states the passage or the mathematical fact it relies on.  Together they are chosen so
that a plausible slip in the oracle -- a dropped D term, the readout taken before the update,
a wrong decay sign, B and C swapped, p and n transposed, heads mapped to the wrong group, dt
missing from the input term -- fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(seed, b=2, L=29, H=4, G=2, P=3, N=5, init=True):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((b, L, H, P))
    dt = rng.uniform(0.01, 0.5, (b, L, H))
    A = -rng.uniform(0.1, 3.0, H)
    B = rng.standard_normal((b, L, G, N))
    C = rng.standard_normal((b, L, G, N))
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((b, H, P, N)) if init else None
    return x, dt, A, B, C, D, h0


def _matrix_form(x, dt, A, B, C, D, h0):
    """Brute force from the dual (matrix) form: y = M x + D x + C_t (prod a_j) h0, with
    M[t, i] = C_t . B_i * dt_i * prod_{j=i+1..t} a_j and a_j = exp(dt_j A_h)
    (eightmm.github.io "Mamba-2", Matrix Mixer View; mohakchugh.is-a.dev "Mamba-2", The Duality).
    Products are formed term by term, as written, not through a cumulative sum."""
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros_like(x)
    final = np.zeros((b, H, P, N))
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            a = np.exp(dt[bi, :, h] * A[h])
            M = np.zeros((L, L))
            for t in range(L):
                for i in range(t + 1):
                    M[t, i] = C[bi, t, g] @ B[bi, i, g] * dt[bi, i, h] * np.prod(a[i + 1:t + 1])
            y[bi, :, h] = M @ x[bi, :, h] + D[h] * x[bi, :, h]
            for i in range(L):
                final[bi, h] += np.prod(a[i + 1:]) * dt[bi, i, h] * np.outer(x[bi, i, h], B[bi, i, g])
            if h0 is not None:
                for t in range(L):
                    y[bi, t, h] += np.prod(a[:t + 1]) * (h0[bi, h] @ C[bi, t, g])
                final[bi, h] += np.prod(a) * h0[bi, h]
    return y, final


def _rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("init", [False, True])
def test_recurrence_equals_semiseparable_matrix(seed, init):
    case = _rand_case(seed, init=init)
    y, final, _ = oracle.ssd_scan(*case)
    y_ref, final_ref = _matrix_form(*case)
    assert _rel(y, y_ref) < 1e-12
    assert _rel(final, final_ref) < 1e-12


def test_group_mapping_contiguous():
    """Heads split into G contiguous groups (h // (H/G)); a case with G = H/2 and B, C that differ
    per group must match the matrix form, and not the one with an interleaved mapping."""
    x, dt, A, B, C, D, h0 = _rand_case(7, b=1, L=9, H=4, G=2, P=2, N=3)
    y, _, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    y_ref, _ = _matrix_form(x, dt, A, B, C, D, h0)
    assert _rel(y, y_ref) < 1e-12
    # swap groups of heads 1 and 2 (an interleaved h % G mapping would read these)
    Bs, Cs = B.copy(), C.copy()
    Bs[:, :, [0, 1]] = B[:, :, [1, 0]]
    Cs[:, :, [0, 1]] = C[:, :, [1, 0]]
    y_wrong, _ = _matrix_form(x, dt, A, Bs, Cs, D, h0)
    assert _rel(y[:, :, 1], y_wrong[:, :, 1]) > 1e-3


def test_hand_worked_example():
    d = json.load(open(os.path.join(GOLDEN, "worked_example_p2_n2.json")))
    A = np.array(d["A_over_ln2"]) * np.log(2.0)
    y, final, _ = oracle.ssd_scan(np.array(d["x"]), np.array(d["dt"]), A, np.array(d["B"]),
                                  np.array(d["C"]), np.array(d["D"]))
    np.testing.assert_allclose(y, np.array(d["y"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(final, np.array(d["final_state"]), rtol=0, atol=1e-12)


def _scalar(x, dt, A, B, C, D, h0=None):
    """N = P = 1, one head: 1-D sequences in, 1-D y out."""
    L = len(x)
    y, final, _ = oracle.ssd_scan(np.reshape(x, (1, L, 1, 1)), np.reshape(dt, (1, L, 1)),
                                  np.array([A]), np.reshape(B, (1, L, 1, 1)),
                                  np.reshape(C, (1, L, 1, 1)), np.array([D]),
                                  None if h0 is None else np.full((1, 1, 1, 1), h0))
    return y.reshape(L), final.reshape(())


def test_closed_form_constant_input_geometric_series():
    """dt, B, C, x constant (B = C = x = 1), h0 = 0: h_t = dt (1 - a^{t+1}) / (1 - a), a geometric
    series, so y_t = dt (1 - a^{t+1}) / (1 - a) + D."""
    L, dt, A, D = 50, 0.07, -1.3, 0.4
    a = np.exp(dt * A)
    y, _ = _scalar(np.ones(L), np.full(L, dt), A, np.ones(L), np.ones(L), D)
    t = np.arange(L)
    np.testing.assert_allclose(y, dt * (1 - a ** (t + 1)) / (1 - a) + D, rtol=1e-13)


def test_closed_form_no_decay_is_prefix_sum():
    """A = 0 makes every a_t = 1: the state is the running sum of dt B x, y_t = C_t sum_{i<=t}
    dt_i B_i x_i + D x_t."""
    rng = np.random.default_rng(3)
    L = 40
    x, dt, B, C = rng.standard_normal(L), rng.uniform(0, 1, L), rng.standard_normal(L), \
        rng.standard_normal(L)
    y, final = _scalar(x, dt, 0.0, B, C, 0.25)
    np.testing.assert_allclose(y, C * np.cumsum(dt * B * x) + 0.25 * x, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(final, np.sum(dt * B * x), rtol=1e-12)


def test_closed_form_free_decay_of_initial_state():
    """x = 0, h0 != 0: nothing enters, h_t = h0 exp(A sum_{j<=t} dt_j), y_t = C_t h_t."""
    rng = np.random.default_rng(4)
    L, A, h0 = 60, -2.0, 1.7
    dt, C = rng.uniform(0, 0.2, L), rng.standard_normal(L)
    y, final = _scalar(np.zeros(L), dt, A, rng.standard_normal(L), C, 0.9, h0=h0)
    decay = np.exp(A * np.cumsum(dt))
    np.testing.assert_allclose(y, C * h0 * decay, rtol=1e-12)
    np.testing.assert_allclose(final, h0 * decay[-1], rtol=1e-12)


def test_zero_dt_token_leaves_state_unchanged():
    """dt = 0 gives a = exp(0) = 1 and no input: the state passes through untouched, and y at that
    token is C_t h_{t-1} + D x_t."""
    rng = np.random.default_rng(5)
    L = 12
    x, dt, B, C = (rng.standard_normal(L), rng.uniform(0.01, 0.3, L), rng.standard_normal(L),
                   rng.standard_normal(L))
    dt[6] = 0.0
    _, h5 = _scalar(x[:6], dt[:6], -1.1, B[:6], C[:6], 0.3)
    _, h6 = _scalar(x[:7], dt[:7], -1.1, B[:7], C[:7], 0.3)
    y, _ = _scalar(x[:7], dt[:7], -1.1, B[:7], C[:7], 0.3)
    assert h6 == h5
    np.testing.assert_allclose(y[6], C[6] * h5 + 0.3 * x[6], rtol=1e-14)


def test_off_diagonal_blocks_have_rank_at_most_N():
    """Every lower-triangular submatrix M[k:, :k] of the SSD matrix has rank <= N, the state size
    (mohakchugh.is-a.dev "Mamba-2", The Duality; eightmm.github.io, Structured Semiseparable
    Matrices).  M is read off the oracle column by column (x = unit vectors, D = 0, h0 = 0); its
    singular values past the N-th vanish while the N-th does not."""
    rng = np.random.default_rng(6)
    L, N = 24, 3
    dt = rng.uniform(0.05, 0.4, (1, L, 1))
    A = np.array([-0.8])
    B = rng.standard_normal((1, L, 1, N))
    C = rng.standard_normal((1, L, 1, N))
    M = np.zeros((L, L))
    for i in range(L):
        e = np.zeros((1, L, 1, 1))
        e[0, i, 0, 0] = 1.0
        y, _, _ = oracle.ssd_scan(e, dt, A, B, C, np.zeros(1))
        M[:, i] = y[0, :, 0, 0]
    assert np.all(np.triu(M, 1) == 0.0)                 # causal
    for k in (6, 12, 18):
        s = np.linalg.svd(M[k:, :k], compute_uv=False)
        assert s[N] / s[0] < 1e-10
        assert s[N - 1] / s[0] > 1e-6


def test_split_resume_equals_single_call():
    """The state is the whole memory of the past (ql.gl, Recurrent state): running the first part,
    then the rest from its final state, equals one call."""
    x, dt, A, B, C, D, h0 = _rand_case(8, L=31)
    y, final, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    y1, f1, _ = oracle.ssd_scan(x[:, :13], dt[:, :13], A, B[:, :13], C[:, :13], D, h0)
    y2, f2, _ = oracle.ssd_scan(x[:, 13:], dt[:, 13:], A, B[:, 13:], C[:, 13:], D, f1)
    np.testing.assert_allclose(np.concatenate([y1, y2], 1), y, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(f2, final, rtol=1e-13, atol=1e-13)


def test_linear_in_input_and_initial_state():
    x, dt, A, B, C, D, h0 = _rand_case(9)
    x2, _, _, _, _, _, h2 = _rand_case(10)
    ya, fa, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    yb, fb, _ = oracle.ssd_scan(x2, dt, A, B, C, D, h2)
    yc, fc, _ = oracle.ssd_scan(2 * x - 3 * x2, dt, A, B, C, D, 2 * h0 - 3 * h2)
    np.testing.assert_allclose(yc, 2 * ya - 3 * yb, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(fc, 2 * fa - 3 * fb, rtol=1e-12, atol=1e-12)


def test_causal():
    x, dt, A, B, C, D, h0 = _rand_case(11)
    y, _, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    x2, B2 = x.copy(), B.copy()
    x2[:, 20:] += 1.0
    B2[:, 20:] *= -2.0
    y2, _, _ = oracle.ssd_scan(x2, dt, A, B2, C, D, h0)
    np.testing.assert_array_equal(y2[:, :20], y[:, :20])


def test_boundary_states_match_prefix_finals():
    x, dt, A, B, C, D, h0 = _rand_case(12, L=30)
    _, _, bnd = oracle.ssd_scan(x, dt, A, B, C, D, h0, every=8)
    assert bnd.shape == (2, 4, 3, 3, 5)
    for k in range(3):
        _, f, _ = oracle.ssd_scan(x[:, :8 * (k + 1)], dt[:, :8 * (k + 1)], A, B[:, :8 * (k + 1)],
                                  C[:, :8 * (k + 1)], D, h0)
        np.testing.assert_array_equal(bnd[:, :, k], f)


def test_decode_steps_equal_scan():
    """Running the recurrence one token per call (the O(1)-per-token decode of crackai.dev
    "Transformers are SSMs", Why It Matters) equals the scan over the same sequence."""
    x, dt, A, B, C, D, h0 = _rand_case(13, L=10)
    y, final, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    st = h0.copy()
    for t in range(10):
        yt, st = oracle.ssd_state_update(st, x[:, t], dt[:, t], A, B[:, t], C[:, t], D)
        np.testing.assert_allclose(yt, y[:, t], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(st, final, rtol=1e-13, atol=1e-13)


def test_selected_pairs_match_full_scan():
    w = configs.SSD_F32_SMALL.with_(batch=2, seqlen=40, nheads=4, ngroups=2, headdim=4, dstate=8,
                                    init_state=True)
    inp = inputs.make_inputs(w)
    y, final, bnd = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init, every=16)
    pairs = [(1, 3), (0, 0), (1, 1)]
    ys, fs, bs = oracle.ssd_scan_pairs(inp, pairs, every=16)
    for j, (b, h) in enumerate(pairs):
        np.testing.assert_array_equal(ys[j], y[b, :, h])
        np.testing.assert_array_equal(fs[j], final[b, h])
        np.testing.assert_array_equal(bs[j], bnd[b, h])


def test_bf16_rounding_matches_torch():
    import torch
    rng = np.random.default_rng(14)
    a = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ours = inputs.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_input_recipe_ranges():
    inp = inputs.make_inputs(configs.SSD_370M.with_(seqlen=256))
    assert inp.dt.min() >= 1e-3 and inp.dt.max() <= 0.1
    assert np.all(inp.A < 0) and np.all(inp.A >= -16.0) and np.all(inp.A <= -1.0)
    np.testing.assert_array_equal(inputs.round_bf16(inp.x), inp.x)
    assert abs(inp.B.std() * np.sqrt(128) - 1.0) < 0.05


# ------------------------------------------------------------------ packed variable-length input
def _packed_matrix_form(x, dt, A, B, C, D, cu, h0):
    """Brute force for packed sequences from the matrix form: one T x T mixing matrix per head
    that is block diagonal over the sequences (M[t, i] = 0 when t and i lie in different
    sequences), each block the semiseparable matrix of _matrix_form, and each sequence's initial
    state decayed from its own first token."""
    _, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    nseq = len(cu) - 1
    seq = np.zeros(T, dtype=int)
    for s in range(nseq):
        seq[cu[s]:cu[s + 1]] = s
    y = np.zeros_like(x)
    final = np.zeros((nseq, H, P, N))
    for h in range(H):
        g = h // (H // G)
        a = np.exp(dt[0, :, h] * A[h])
        M = np.zeros((T, T))
        for t in range(T):
            for i in range(t + 1):
                if seq[i] == seq[t]:
                    M[t, i] = C[0, t, g] @ B[0, i, g] * dt[0, i, h] * np.prod(a[i + 1:t + 1])
        y[0, :, h] = M @ x[0, :, h] + D[h] * x[0, :, h]
        for s in range(nseq):
            lo, hi = cu[s], cu[s + 1]
            for i in range(lo, hi):
                final[s, h] += np.prod(a[i + 1:hi]) * dt[0, i, h] * np.outer(x[0, i, h], B[0, i, g])
            if h0 is not None:
                for t in range(lo, hi):
                    y[0, t, h] += np.prod(a[lo:t + 1]) * (h0[s, h] @ C[0, t, g])
                final[s, h] += np.prod(a[lo:hi]) * h0[s, h]
    return y, final


def _packed_case(seed, T=37, H=4, G=2, P=3, N=5):
    x, dt, A, B, C, D, _ = _rand_case(seed, b=1, L=T, H=H, G=G, P=P, N=N, init=False)
    cu = np.array([0, 6, 6, 7, 22, T], dtype=np.int32)   # an empty and a one-token sequence
    rng = np.random.default_rng(seed + 7)
    h0 = 0.3 * rng.standard_normal((len(cu) - 1, H, P, N))
    return x, dt, A, B, C, D, cu, h0


@pytest.mark.parametrize("seed", [3, 4])
def test_packed_sequences_equal_block_diagonal_matrix(seed):
    x, dt, A, B, C, D, cu, h0 = _packed_case(seed)
    y, final = oracle.ssd_scan_varlen(x, dt, A, B, C, D, cu, h0)
    y_ref, f_ref = _packed_matrix_form(x, dt, A, B, C, D, cu, h0)
    assert _rel(y, y_ref) < 1e-12
    assert _rel(final, f_ref) < 1e-12
    assert np.array_equal(final[1], h0[1])   # the empty sequence hands its initial state back


def test_packed_single_sequence_is_the_plain_scan():
    x, dt, A, B, C, D, _, h0 = _packed_case(5)
    cu = np.array([0, x.shape[1]], dtype=np.int32)
    y, final = oracle.ssd_scan_varlen(x, dt, A, B, C, D, cu, h0[:1])
    y_ref, f_ref, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0[:1])
    assert np.array_equal(y, y_ref) and np.array_equal(final, f_ref)


def test_packed_sequences_do_not_see_each_other():
    x, dt, A, B, C, D, cu, h0 = _packed_case(6)
    y, final = oracle.ssd_scan_varlen(x, dt, A, B, C, D, cu, h0)
    x2, B2 = x.copy(), B.copy()
    x2[0, cu[3]:cu[4]] *= -3.0          # change only the fourth sequence's inputs
    B2[0, cu[3]:cu[4]] += 1.0
    y2, final2 = oracle.ssd_scan_varlen(x2, dt, A, B2, C, D, cu, h0)
    outside = np.ones(x.shape[1], dtype=bool)
    outside[cu[3]:cu[4]] = False
    assert np.array_equal(y[0, outside], y2[0, outside])
    assert np.array_equal(np.delete(final, 3, 0), np.delete(final2, 3, 0))
    assert not np.allclose(y[0, ~outside], y2[0, ~outside])


def test_packed_input_recipe():
    w = configs.SSD_VARLEN.with_(seqlen=300, nheads=2, seed=77)
    inp = inputs.make_inputs(w)
    cu = inp.cu_seqlens
    assert cu.dtype == np.int32 and len(cu) == w.nseq + 1
    assert cu[0] == 0 and cu[-1] == w.seqlen and np.all(np.diff(cu) > 0)
    assert inp.init.shape == (w.nseq, w.nheads, w.headdim, w.dstate)


# ------------------------------------------------------------------ fused block steps
def test_gate_closed_forms():
    """SiLU(0) = 0 and SiLU(z) = z (1 - 1/(1+e^z)) -> z for large z: a zero gate silences the
    output, a large gate scales it by z, and the state never sees the gate."""
    x, dt, A, B, C, D, h0 = _rand_case(8)
    y, f, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    y0, f0 = oracle.ssd_scan_block(x, dt, A, B, C, D, h0, z=np.zeros_like(x))
    assert np.all(y0 == 0.0) and np.array_equal(f0, f)
    y50, _ = oracle.ssd_scan_block(x, dt, A, B, C, D, h0, z=np.full_like(x, 50.0))
    assert _rel(y50, 50.0 * y) < 1e-14
    ym, _ = oracle.ssd_scan_block(x, dt, A, B, C, D, h0, z=np.full_like(x, -50.0))
    assert np.max(np.abs(ym)) <= 50.0 * np.exp(-50.0) * np.max(np.abs(y)) * 1.01


def test_softplus_prologue_closed_form():
    """softplus(log(e^v - 1)) = v: a raw dt of log(expm1(v)) reproduces the scan at dt = v."""
    x, dt, A, B, C, D, h0 = _rand_case(9)
    raw = np.log(np.expm1(dt))
    y, f, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    y2, f2 = oracle.ssd_scan_block(x, raw, A, B, C, D, h0, softplus=True)
    assert _rel(y2, y) < 1e-12 and _rel(f2, f) < 1e-12
    bias = np.linspace(-0.3, 0.4, A.shape[0])
    y3, f3 = oracle.ssd_scan_block(x, raw - bias, A, B, C, D, h0, dt_bias=bias, softplus=True)
    assert _rel(y3, y) < 1e-12 and _rel(f3, f) < 1e-12


def test_clamp_prologue_equals_clipped_dt():
    x, dt, A, B, C, D, h0 = _rand_case(10)
    lo, hi = 0.05, 0.3
    y, f, _ = oracle.ssd_scan(x, np.clip(dt, lo, hi), A, B, C, D, h0)
    y2, f2 = oracle.ssd_scan_block(x, dt, A, B, C, D, h0, dt_limit=(lo, hi))
    assert np.array_equal(y2, y) and np.array_equal(f2, f)
    assert np.any(dt < lo) and np.any(dt > hi)   # the clamp is exercised on both sides


def test_block_input_recipe():
    w = configs.SSD_370M.with_(seqlen=512, nheads=8)
    blk = inputs.make_block_inputs(w)
    dt = oracle.dt_prologue(blk.dt_raw, blk.dt_bias, True, blk.dt_limit)
    assert dt.min() >= 1e-3 and dt.max() <= 0.1
    base = inputs.make_inputs(w)          # the scan inputs are not disturbed by the extra draw
    again = inputs.make_inputs(w)
    assert np.array_equal(base.x, again.x)
    assert blk.z.shape == base.x.shape and np.array_equal(inputs.round_bf16(blk.z), blk.z)


def test_block_decode_steps_equal_block_scan():
    """The gated decode step with the dt prologue, repeated over a sequence, is the gated scan
    with the same prologue (both are the recurrence with the same per-token dt and gate)."""
    x, dt, A, B, C, D, h0 = _rand_case(11, b=2, L=12)
    rng = np.random.default_rng(12)
    z = rng.standard_normal(x.shape)
    raw = rng.standard_normal(dt.shape)
    bias = -rng.uniform(0.5, 1.5, A.shape[0])
    y_ref, f_ref = oracle.ssd_scan_block(x, raw, A, B, C, D, h0, z=z, dt_bias=bias,
                                         softplus=True, dt_limit=(0.05, 0.4))
    state = h0.copy()
    for t in range(x.shape[1]):
        y_t, state = oracle.ssd_state_update_block(state, x[:, t], raw[:, t], A, B[:, t],
                                                   C[:, t], D, z=z[:, t], dt_bias=bias,
                                                   softplus=True, dt_limit=(0.05, 0.4))
        assert _rel(y_t, y_ref[:, t]) < 1e-12
    assert _rel(state, f_ref) < 1e-12


# ------------------------------------------------------------------ backward
def _loss(x, dt, A, B, C, D, h0, dy, dfin):
    y, f, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
    return float(np.sum(dy * y) + np.sum(dfin * f))


@pytest.mark.parametrize("seed", [21, 22])
def test_backward_equals_finite_differences(seed):
    """Every gradient of the adjoint oracle against central differences of the (pinned) forward
    oracle, element by element, on a tiny input with two groups and an initial state."""
    x, dt, A, B, C, D, h0 = _rand_case(seed, b=1, L=7, H=4, G=2, P=2, N=3)
    rng = np.random.default_rng(seed + 1)
    dy = rng.standard_normal(x.shape)
    dfin = rng.standard_normal(h0.shape)
    g = oracle.ssd_scan_bwd(x, dt, A, B, C, D, dy, h0, dfin)
    args = dict(x=x, dt=dt, A=A, B=B, C=C, D=D, init=h0)
    key = dict(x="dx", dt="ddt", A="dA", B="dB", C="dC", D="dD", init="dinit")
    eps = 1e-6
    for name, arr in args.items():
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            saved = arr[idx]
            arr[idx] = saved + eps
            lp = _loss(*(args[k] for k in ("x", "dt", "A", "B", "C", "D", "init")), dy, dfin)
            arr[idx] = saved - eps
            lm = _loss(*(args[k] for k in ("x", "dt", "A", "B", "C", "D", "init")), dy, dfin)
            arr[idx] = saved
            num[idx] = (lp - lm) / (2 * eps)
        assert _rel(g[key[name]], num) < 1e-7, name


def test_backward_closed_form_scalar():
    """N = P = 1, one token: y = (a h0 + dt x B) C + D x, so every gradient is a product."""
    x, dt, A, B, C, D, h0 = 0.7, 0.3, -1.2, 0.5, -0.8, 0.4, 0.9
    a = np.exp(dt * A)
    g = oracle.ssd_scan_bwd(np.full((1, 1, 1, 1), x), np.full((1, 1, 1), dt), np.array([A]),
                            np.full((1, 1, 1, 1), B), np.full((1, 1, 1, 1), C), np.array([D]),
                            np.ones((1, 1, 1, 1)), np.full((1, 1, 1, 1), h0))
    assert np.isclose(g["dx"].item(), D + dt * B * C)
    assert np.isclose(g["dB"].item(), dt * x * C)
    assert np.isclose(g["dC"].item(), a * h0 + dt * x * B)
    assert np.isclose(g["ddt"].item(), x * B * C + A * a * h0 * C)
    assert np.isclose(g["dA"].item(), dt * a * h0 * C)
    assert np.isclose(g["dD"].item(), x)
    assert np.isclose(g["dinit"].item(), a * C)
