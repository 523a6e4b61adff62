"""GPU parity of the fused block steps (ssd_chunk_scan_fwd_ex) against the float64 oracle.

The dt the scan uses is softplus(dt_raw + dt_bias) clamped to (1e-3, 0.1) -- the same
distribution as the plain workloads' dt -- and the output is gated by SiLU(z).  Both are fused:
the prologue runs before the cumsum, the gate in the chunk-scan epilogue, on the tensor-core and
on the CUDA-core paths.  Tolerances as for the plain scan (max over (batch, head) slices of the
relative L2 error of y and of the final state).
"""
import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_per_pair, max_rel_slices, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _run(torch, inp, blk, chunk, device, gate=True, prologue=True):
    t = torch_inputs(inp, device)
    xdt = t["x"].dtype
    z = torch.from_numpy(blk.z).to(device).to(xdt) if gate else None
    if prologue:
        dt = torch.from_numpy(blk.dt_raw).to(device)
        bias = torch.from_numpy(blk.dt_bias).to(device)
        y, final = ssd.chunk_scan_fwd(t["x"], dt, t["A"], t["B"], t["C"], t["D"], chunk,
                                      init_state=t["init_state"], z=z, dt_bias=bias,
                                      dt_softplus=True, dt_limit=blk.dt_limit)
    else:
        y, final = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk,
                                      init_state=t["init_state"], z=z)
    torch.cuda.synchronize()
    return y, final


def _reference(inp, blk, gate=True, prologue=True):
    if prologue:
        return oracle.ssd_scan_block(inp.x, blk.dt_raw, inp.A, inp.B, inp.C, inp.D, inp.init,
                                     z=blk.z if gate else None, dt_bias=blk.dt_bias,
                                     softplus=True, dt_limit=blk.dt_limit)
    return oracle.ssd_scan_block(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init,
                                 z=blk.z if gate else None)


def _compare(w, y, final, y_ref, f_ref):
    yn, fn = to_np(y), to_np(final)
    pairs = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    ey = max_rel_per_pair([yn[b, :, h] for b, h in pairs], [y_ref[b, :, h] for b, h in pairs])
    ef = max_rel_per_pair([fn[b, h] for b, h in pairs], [f_ref[b, h] for b, h in pairs])
    assert np.isfinite(yn).all()
    assert ey <= TOL[w.dtype], f"y relative L2 error {ey:.3e}"
    assert ef <= TOL[w.dtype], f"final state relative L2 error {ef:.3e}"


CASES = [
    # (name, workload, chunk, gate, prologue)
    ("tc_q256_both", configs.SSD_370M.with_(batch=2, seqlen=700, nheads=10, init_state=True), 256,
     True, True),
    ("tc_q128_gate", configs.SSD_370M.with_(batch=1, seqlen=600, nheads=8, ngroups=2), 128,
     True, False),
    ("tc_q256_prologue", configs.SSD_370M.with_(batch=1, seqlen=300, nheads=6), 256, False,
     True),
    # runs long enough for the chunk scan's third group of CTAs (4 groups of 10 heads: the last
    # 128/1024 of each second-tile run), a 100-token last chunk (its second tiles skipped, also
    # by the warp that stages the gate rows), segments that end inside runs
    ("tc_q256_both_tails_groups", configs.SSD_LONG.with_(batch=2, seqlen=2148, nheads=40,
                                                          ngroups=4), 256, True, True),
    ("f32_simt_both", configs.SSD_F32_SMALL.with_(batch=2, seqlen=333, nheads=4, ngroups=2,
                                                  init_state=True), 64, True, True),
    ("bf16_simt_both", configs.SSD_370M.with_(batch=1, seqlen=300, nheads=4), 64, True, True),
]


@pytest.mark.parametrize("name,w,chunk,gate,prologue", CASES, ids=[c[0] for c in CASES])
def test_fused_block_parity(cuda_device, name, w, chunk, gate, prologue):
    import torch
    inp = inputs.make_inputs(w)
    blk = inputs.make_block_inputs(w)
    y, final = _run(torch, inp, blk, chunk, cuda_device, gate, prologue)
    y_ref, f_ref = _reference(inp, blk, gate, prologue)
    _compare(w, y, final, y_ref, f_ref)


def test_fused_block_full_size_every_output(cuda_device):
    """The 2.7B-layer shape in the benchmark's launch configuration, gated and with the dt
    prologue: every (batch, head) slice of y and of the final state against the oracle's gated
    scan, one batch row at a time."""
    import torch
    w = configs.SSD_2P7B
    inp = inputs.make_inputs(w)
    blk = inputs.make_block_inputs(w)
    y, final = _run(torch, inp, blk, w.chunk, cuda_device)
    ey = ef = 0.0
    for b in range(w.batch):
        y_ref, f_ref = oracle.ssd_scan_block(
            inp.x[b:b + 1], blk.dt_raw[b:b + 1], inp.A, inp.B[b:b + 1], inp.C[b:b + 1], inp.D,
            None, z=blk.z[b:b + 1], dt_bias=blk.dt_bias, softplus=True, dt_limit=blk.dt_limit)
        yn = to_np(y[b:b + 1])
        assert np.isfinite(yn).all()
        ey = max(ey, max_rel_slices(yn, y_ref, (1, 3))[0])
        ef = max(ef, max_rel_slices(to_np(final[b:b + 1]), f_ref, (2, 3))[0])
    assert ey <= TOL["bf16"], f"y relative L2 error {ey:.3e}"
    assert ef <= TOL["bf16"], f"final state relative L2 error {ef:.3e}"


def test_plain_options_equal_plain_scan(cuda_device):
    """A zeroed options struct is the plain scan, bit for bit."""
    import ctypes
    import torch
    w = configs.SSD_370M.with_(batch=1, seqlen=512, nheads=8)
    t = torch_inputs(inputs.make_inputs(w), cuda_device)
    y0, f0 = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256)
    shape = ssd.make_shape(1, 512, 8, 64, 128, 1, ssd.SSD_BF16)
    opts = ssd.FwdOptions(None, None, 0, 0.0, 0.0)
    ws = ssd.new_workspace(shape, 256, cuda_device)
    y1 = torch.empty_like(y0)
    f1 = torch.empty_like(f0)
    rc = ssd.lib().ssd_chunk_scan_fwd_ex(
        ctypes.byref(shape), t["x"].data_ptr(), t["dt"].data_ptr(), t["A"].data_ptr(),
        t["B"].data_ptr(), t["C"].data_ptr(), t["D"].data_ptr(), 256, None, y1.data_ptr(),
        f1.data_ptr(), ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream,
        ctypes.byref(opts))
    assert rc == ssd.SSD_OK, ssd.last_error()
    torch.cuda.synchronize()
    assert torch.equal(y0, y1) and torch.equal(f0, f1)


def test_decode_with_block_options(cuda_device):
    """Gated decode steps with the dt prologue against the oracle, over 6 steps."""
    import torch
    rng = np.random.default_rng(77)
    b, H, P, N, G = 8, 8, 64, 128, 2
    state0 = (0.1 * rng.standard_normal((b, H, P, N))).astype(np.float32)
    A = (-np.exp(rng.uniform(0.0, np.log(16.0), H))).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    bias = (-4.0 + rng.uniform(-0.5, 0.5, H)).astype(np.float32)
    dev = cuda_device
    st = torch.from_numpy(state0).to(dev)
    ref_state = state0.astype(np.float64)
    errs = []
    for step in range(6):
        x = inputs.round_bf16(rng.standard_normal((b, H, P)).astype(np.float32))
        z = inputs.round_bf16(rng.standard_normal((b, H, P)).astype(np.float32))
        raw = rng.standard_normal((b, H)).astype(np.float32)
        Bv = inputs.round_bf16((rng.standard_normal((b, G, N)) / np.sqrt(N)).astype(np.float32))
        Cv = inputs.round_bf16((rng.standard_normal((b, G, N)) / np.sqrt(N)).astype(np.float32))
        tt = lambda a, d=torch.float32: torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(d)
        y = ssd.state_update(st, tt(x, torch.bfloat16), tt(raw), tt(A), tt(Bv, torch.bfloat16),
                             tt(Cv, torch.bfloat16), tt(D), z=tt(z, torch.bfloat16),
                             dt_bias=tt(bias), dt_softplus=True, dt_limit=(1e-3, 0.1))
        y_ref, ref_state = oracle.ssd_state_update_block(ref_state, x, raw, A, Bv, Cv, D, z=z,
                                                         dt_bias=bias, softplus=True,
                                                         dt_limit=(1e-3, 0.1))
        torch.cuda.synchronize()
        yn = to_np(y)
        errs.append(max_rel_per_pair([yn[i, h] for i in range(b) for h in range(H)],
                                     [y_ref[i, h] for i in range(b) for h in range(H)]))
    sn = to_np(st)
    es = max_rel_per_pair([sn[i, h] for i in range(b) for h in range(H)],
                          [ref_state[i, h] for i in range(b) for h in range(H)])
    assert max(errs) <= TOL["bf16"] and es <= 1e-5
