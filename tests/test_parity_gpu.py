"""GPU parity: the CUDA path through the C ABI against the float64 oracle, element by element.

Tolerance (max over (batch, head) slices of the relative L2 error, for y and for the final
state): 1e-4 for float32 inputs, 1e-2 for bf16 inputs with float32 accumulation.

Every case compares every output: the small cases and the full-size workloads alike (the latter
in the same launch configuration the benchmark times, with the oracle run over blocks of batch
rows to bound host memory).  Guard bands of sentinel values around y, the final state and the
workspace catch writes out of bounds.
"""
import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_per_pair, max_rel_slices, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _guarded_empty(torch, shape, dtype, device, guard=4096, fill=1234.5):
    """A tensor view with `guard` sentinel elements on both sides."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * guard,), fill, dtype=dtype, device=device)
    return buf, buf[guard:guard + n].view(*shape)


def _check_guard(buf, n, guard=4096, fill=1234.5):
    import torch
    want = torch.tensor(fill, dtype=buf.dtype).item()
    assert bool((buf[:guard] == want).all()), "write before the output"
    assert bool((buf[guard + n:] == want).all()), "write past the output"


def run_fwd(torch, t, w, chunk, device, guards=True):
    b, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups
    shape = ssd.make_shape(b, L, H, P, N, G, ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32)
    ws_n = ssd.workspace_size(shape, chunk)
    ws_buf = torch.full((ws_n + 65536,), 0xA5, dtype=torch.uint8, device=device)
    ws = ws_buf[:ws_n]
    ybuf, y = _guarded_empty(torch, (b, L, H, P), t["x"].dtype, device)
    fbuf, final = _guarded_empty(torch, (b, H, P, N), torch.float32, device)
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk,
                       init_state=t["init_state"], y=y, final_state=final, workspace=ws)
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK
    if guards:
        _check_guard(ybuf, y.numel())
        _check_guard(fbuf, final.numel())
        assert bool((ws_buf[ws_n:] == 0xA5).all()), "write past the workspace"
    return y, final


def _rows(inp, b0, b1):
    """The inputs of batch rows [b0, b1) (re-indexing only)."""
    init = None if inp.init is None else inp.init[b0:b1]
    return (inp.x[b0:b1], inp.dt[b0:b1], inp.A, inp.B[b0:b1], inp.C[b0:b1], inp.D, init)


def check_against_oracle(inp, y, final, rows_per_block=None):
    """Every output of y (b, L, H, P) and of the final state against the oracle, as the max over
    (batch, head) slices of the relative L2 error.  The oracle runs on blocks of batch rows."""
    w = inp.w
    tol = TOL[w.dtype]
    rb = rows_per_block or max(1, w.batch)
    ey = ef = 0.0
    for b0 in range(0, w.batch, rb):
        b1 = min(w.batch, b0 + rb)
        y_ref, f_ref, _ = oracle.ssd_scan(*_rows(inp, b0, b1))
        yn, fn = to_np(y[b0:b1]), to_np(final[b0:b1])
        assert np.isfinite(yn).all()
        ey = max(ey, max_rel_slices(yn, y_ref, (1, 3))[0])
        ef = max(ef, max_rel_slices(fn, f_ref, (2, 3))[0])
    assert ey <= tol, f"y relative L2 error {ey:.3e} > {tol}"
    assert ef <= tol, f"final state relative L2 error {ef:.3e} > {tol}"
    return ey, ef


# ------------------------------------------------------------------ small, every output checked
SMALL = [
    # (name, workload, chunk): f32 -> CUDA-core path; bf16 Q in {128, 256} -> tensor cores
    ("f32_cfg0", configs.SSD_F32_SMALL, 64),
    ("f32_ragged_g2_init", configs.SSD_F32_SMALL.with_(batch=2, seqlen=333, nheads=4, ngroups=2,
                                                       init_state=True), 32),
    ("f32_q16_n32_p16", configs.SSD_F32_SMALL.with_(seqlen=77, headdim=16, dstate=32), 16),
    ("bf16_simt_q64", configs.SSD_370M.with_(seqlen=300, nheads=4), 64),
    ("bf16_tc_q256", configs.SSD_370M.with_(seqlen=512, nheads=8), 256),
    ("bf16_tc_q128", configs.SSD_370M.with_(seqlen=512, nheads=8), 128),
    ("bf16_tc_ragged", configs.SSD_370M.with_(batch=3, seqlen=700, nheads=10), 256),
    ("bf16_tc_short", configs.SSD_370M.with_(batch=2, seqlen=100, nheads=9), 256),
    ("bf16_tc_one_token", configs.SSD_370M.with_(batch=2, seqlen=1, nheads=3), 256),
    ("bf16_tc_groups_init", configs.SSD_LONG.with_(seqlen=1000, nheads=16, ngroups=4), 256),
    ("bf16_tc_groups_q128", configs.SSD_LONG.with_(seqlen=640, nheads=24, ngroups=8), 128),
    ("bf16_tc_many_heads", configs.SSD_2P7B.with_(batch=1, seqlen=384), 256),
    # runs long enough that the last share of each second-tile run goes to the third group of
    # CTAs (80 heads in one group: 1360 items, runs of 18-19, tails of 1; 4 groups of 10 heads:
    # 720 items, runs of 9-10, tails of 1), with a 100-token last chunk whose second tiles are
    # skipped, also inside tails, and tails that start inside a segment
    ("bf16_tc_tails_many_heads", configs.SSD_2P7B.with_(batch=1, seqlen=4196), 256),
    ("bf16_tc_tails_groups", configs.SSD_LONG.with_(batch=2, seqlen=2148, nheads=40,
                                                     ngroups=4), 256),
]


@pytest.mark.parametrize("name,w,chunk", SMALL, ids=[s[0] for s in SMALL])
def test_small_full_parity(cuda_device, name, w, chunk):
    import torch
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, final = run_fwd(torch, t, w, chunk, cuda_device)
    check_against_oracle(inp, y, final)


# The tensor-core cases again with a nonzero initial state and a fresh draw.
TC_SMALL = [s for s in SMALL if s[0].startswith("bf16_tc")]


@pytest.mark.parametrize("name,w,chunk", TC_SMALL, ids=[s[0] for s in TC_SMALL])
def test_small_parity_with_initial_state(cuda_device, name, w, chunk):
    import torch
    inp = inputs.make_inputs(w.with_(init_state=True, seed=w.seed + 17))
    t = torch_inputs(inp, cuda_device)
    y, final = run_fwd(torch, t, inp.w, chunk, cuda_device)
    check_against_oracle(inp, y, final)


# ------------------------------------------------------------------ full-size workloads
FULL = [("ssd_370m", configs.SSD_370M, None),
        ("ssd_2p7b", configs.SSD_2P7B, 1),
        ("ssd_2p7b_init", configs.SSD_2P7B.with_(init_state=True), 1),
        ("ssd_long", configs.SSD_LONG, 1)]


@pytest.mark.parametrize("name,w,rows", FULL, ids=[f[0] for f in FULL])
def test_full_size_parity_every_output(cuda_device, name, w, rows):
    """Every (batch, head) slice of y and of the final state at the workload's full size, in
    the benchmark's launch configuration."""
    import torch
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, final = run_fwd(torch, t, w, w.chunk, cuda_device, guards=False)
    check_against_oracle(inp, y, final, rows_per_block=rows)


def test_f32_config_parity_every_output(cuda_device):
    import torch
    w = configs.SSD_F32_SMALL
    inp = inputs.make_inputs(w)
    y, final = run_fwd(torch, torch_inputs(inp, cuda_device), w, w.chunk, cuda_device)
    ey, ef = check_against_oracle(inp, y, final)
    assert ey < 1e-5  # float32 path stays well inside its bound


# ------------------------------------------------------------------ invariances
@pytest.mark.parametrize("dtype,chunks", [("f32", (16, 32, 64, 128, 256)),
                                          ("bf16", (64, 128, 256))])
def test_chunk_size_invariance(cuda_device, dtype, chunks):
    """The chunked result equals the recurrence for every chunk size (ql.gl, The Core of SSD:
    chunking preserves the sequential state computation)."""
    import torch
    w = configs.SSD_370M.with_(seqlen=777, nheads=8, dtype=dtype, init_state=True)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    outs = [run_fwd(torch, t, w, q, cuda_device, guards=False) for q in chunks]
    for y, f in outs:
        check_against_oracle(inp, y, f)
    y0, f0 = map(to_np, outs[0])
    for y, f in outs[1:]:
        assert np.linalg.norm(to_np(y) - y0) / np.linalg.norm(y0) <= 2 * TOL[dtype]


@pytest.mark.parametrize("dtype,chunk", [("f32", 64), ("bf16", 256), ("bf16", 128)])
def test_split_resume_equals_single_call(cuda_device, dtype, chunk):
    """final_state of the first part as init_state of the second equals one call."""
    import torch
    w = configs.SSD_370M.with_(seqlen=900, nheads=8, dtype=dtype, init_state=True)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, f = run_fwd(torch, t, w, chunk, cuda_device, guards=False)
    cut = 333
    t1 = {k: (v[:, :cut].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in t.items()}
    y1, f1 = run_fwd(torch, t1, w.with_(seqlen=cut), chunk, cuda_device, guards=False)
    t2 = {k: (v[:, cut:].contiguous() if k in ("x", "dt", "B", "C") else v) for k, v in t.items()}
    t2["init_state"] = f1
    y2, f2 = run_fwd(torch, t2, w.with_(seqlen=900 - cut), chunk, cuda_device, guards=False)
    ycat = np.concatenate([to_np(y1), to_np(y2)], 1)
    tol = TOL[dtype]
    assert np.linalg.norm(ycat - to_np(y)) / np.linalg.norm(to_np(y)) <= tol
    assert np.linalg.norm(to_np(f2) - to_np(f)) / np.linalg.norm(to_np(f)) <= tol
    check_against_oracle(inp, torch.from_numpy(ycat), f2)


@pytest.mark.parametrize("dtype,chunk", [("f32", 64), ("bf16", 256)])
def test_zero_dt_padding_changes_nothing(cuda_device, dtype, chunk):
    """Appending tokens with dt = 0 (decay 1, no input) leaves y of the real tokens and the final
    state unchanged; a partial last chunk is exactly such padding."""
    import torch
    w = configs.SSD_370M.with_(seqlen=500, nheads=8, dtype=dtype, init_state=True)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, f = run_fwd(torch, t, w, chunk, cuda_device, guards=False)
    pad = 12
    tp = dict(t)
    for k in ("x", "B", "C"):
        tp[k] = torch.cat([t[k], torch.randn_like(t[k][:, :pad])], 1).contiguous()
    tp["dt"] = torch.cat([t["dt"], torch.zeros_like(t["dt"][:, :pad])], 1).contiguous()
    yp, fp = run_fwd(torch, tp, w.with_(seqlen=500 + pad), chunk, cuda_device, guards=False)
    tol = TOL[dtype]
    assert np.linalg.norm(to_np(yp)[:, :500] - to_np(y)) / np.linalg.norm(to_np(y)) <= tol / 10
    assert np.linalg.norm(to_np(fp) - to_np(f)) / np.linalg.norm(to_np(f)) <= tol / 10


def test_linear_in_input_and_initial_state(cuda_device):
    import torch
    w = configs.SSD_F32_SMALL.with_(seqlen=300, nheads=4, init_state=True)
    inp = inputs.make_inputs(w)
    inp2 = inputs.make_inputs(w, seed=77)
    t = torch_inputs(inp, cuda_device)
    t2 = torch_inputs(inp2, cuda_device)
    ya, fa = run_fwd(torch, t, w, 64, cuda_device, guards=False)
    tb = dict(t, x=t2["x"], init_state=t2["init_state"])
    yb, fb = run_fwd(torch, tb, w, 64, cuda_device, guards=False)
    tc = dict(t, x=(2 * t["x"] - 3 * t2["x"]).contiguous(),
              init_state=(2 * t["init_state"] - 3 * t2["init_state"]).contiguous())
    yc, fc = run_fwd(torch, tc, w, 64, cuda_device, guards=False)
    lhs, rhs = to_np(yc), 2 * to_np(ya) - 3 * to_np(yb)
    assert np.linalg.norm(lhs - rhs) / np.linalg.norm(rhs) < 1e-5
    assert np.linalg.norm(to_np(fc) - (2 * to_np(fa) - 3 * to_np(fb))) / np.linalg.norm(to_np(fc)) < 1e-5


def test_empty_sequence_returns_initial_state(cuda_device):
    import torch
    w = configs.SSD_F32_SMALL.with_(seqlen=0, init_state=True)
    h0 = torch.randn(1, 2, 64, 64, device=cuda_device)
    x = torch.empty(1, 0, 2, 64, device=cuda_device)
    dt = torch.empty(1, 0, 2, device=cuda_device)
    BC = torch.empty(1, 0, 1, 64, device=cuda_device)
    A = torch.full((2,), -1.0, device=cuda_device)
    y, f = ssd.chunk_scan_fwd(x, dt, A, BC, BC, A, 64, init_state=h0,
                              workspace=torch.empty(256, dtype=torch.uint8, device=cuda_device))
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.equal(f, h0)
    y, f = ssd.chunk_scan_fwd(x, dt, A, BC, BC, A, 64,
                              workspace=torch.empty(256, dtype=torch.uint8, device=cuda_device))
    torch.cuda.synchronize()
    assert torch.count_nonzero(f) == 0


def test_final_state_may_alias_initial_state(cuda_device):
    import torch
    w = configs.SSD_370M.with_(seqlen=400, nheads=8, init_state=True)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    _, f_ref = run_fwd(torch, t, w, 256, cuda_device, guards=False)
    h = t["init_state"].clone()
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256, init_state=h,
                       final_state=h)
    torch.cuda.synchronize()
    assert torch.allclose(h, f_ref, rtol=0, atol=0)


# ------------------------------------------------------------------ decode
def _decode_steps(torch, t, w, device, steps):
    """Run `steps` single-token updates from the initial state; returns y (b, steps, H, P) and the
    state.  Inputs are re-laid out time-major so each step reads contiguous slices."""
    xs = t["x"][:, :steps].transpose(0, 1).contiguous()
    dts = t["dt"][:, :steps].transpose(0, 1).contiguous()
    Bs = t["B"][:, :steps].transpose(0, 1).contiguous()
    Cs = t["C"][:, :steps].transpose(0, 1).contiguous()
    state = t["init_state"].clone()
    ys = torch.empty_like(xs)
    for s in range(steps):
        ssd.state_update(state, xs[s], dts[s], t["A"], Bs[s], Cs[s], t["D"], y=ys[s])
    torch.cuda.synchronize()
    return ys.transpose(0, 1), state


@pytest.mark.parametrize("dtype,dstate", [("bf16", 128), ("f32", 64), ("bf16", 256),
                                          ("f32", 32)])
def test_decode_small_vs_oracle(cuda_device, dtype, dstate):
    import torch
    w = configs.SSD_DECODE.with_(batch=3, seqlen=40, nheads=6, ngroups=2, dstate=dstate,
                                 dtype=dtype)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, state = _decode_steps(torch, t, w, cuda_device, w.seqlen)
    check_against_oracle(inp, y, state)


def test_decode_full_size_vs_oracle_and_chunked(cuda_device):
    """1000 single-token updates at (batch 128, 80 heads, 64 x 128 fp32 state): every output and
    the final state against the oracle, and every output against the chunked scan of the same
    sequence."""
    import torch
    w = configs.SSD_DECODE
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, state = _decode_steps(torch, t, w, cuda_device, w.seqlen)
    check_against_oracle(inp, y, state, rows_per_block=16)
    yc, fc = run_fwd(torch, t, w, w.chunk, cuda_device, guards=False)
    err = 0.0
    for b0 in range(0, w.batch, 16):
        err = max(err, max_rel_slices(to_np(y[b0:b0 + 16]), to_np(yc[b0:b0 + 16]), (1, 3))[0])
    assert err <= TOL["bf16"]
    ef = max_rel_slices(to_np(state), to_np(fc), (2, 3))[0]
    assert ef <= TOL["bf16"]
