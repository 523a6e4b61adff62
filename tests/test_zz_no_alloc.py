"""The no-allocation entry point, ssd_chunk_scan_fwd_static, against ssd_chunk_scan_fwd.

Callers that may not allocate device memory where they run the scan -- a locked allocator
inside a framework's planning or capture phase, a runtime that owns all device memory, a host
with a fixed memory budget -- call ssd_chunk_scan_fwd_static.  It runs the same kernels but uses
a scratch array built into the library instead of a caller-provided workspace.  These tests
call it through the C ABI twice in a row (the second call must not be disturbed by what the
first left in the shared array), read the array's status word after each call, and require each
result to equal the workspace entry point's bit for bit (the same kernels on the same inputs)
and to match the float64 oracle within the bf16 parity tolerance; they also check that problems
larger than the array are refused.

The file is named so that pytest collects it last: if it fails, a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_slices, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _static_entry():
    f = ssd.lib().ssd_chunk_scan_fwd_static
    f.restype = ctypes.c_int
    f.argtypes = ([ctypes.POINTER(ssd.Shape)] + [ctypes.c_void_p] * 6 + [ctypes.c_int]
                  + [ctypes.c_void_p] * 4)
    return f


def _status_entry():
    f = ssd.lib().ssd_chunk_scan_fwd_static_status
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p]
    return f


def _shape(w):
    return ssd.make_shape(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                          ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32)


def _call_static(torch, t, w, chunk):
    y = torch.empty_like(t["x"])
    final = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                        device=t["x"].device)
    init = t["init_state"]
    stream = torch.cuda.current_stream().cuda_stream
    rc = _static_entry()(ctypes.byref(_shape(w)), t["x"].data_ptr(), t["dt"].data_ptr(),
                         t["A"].data_ptr(), t["B"].data_ptr(), t["C"].data_ptr(),
                         t["D"].data_ptr(), chunk, None if init is None else init.data_ptr(),
                         y.data_ptr(), final.data_ptr(), stream)
    assert rc == ssd.SSD_OK, ssd.last_error()
    st = _status_entry()(stream)
    assert st == ssd.SSD_OK, ssd.last_error()
    return y, final


def test_static_scratch_matches_workspace_entry_point_on_two_calls(cuda_device):
    import torch
    cases = [
        (configs.SSD_370M, 256),   # batch 2 x 2048 x 24 heads: ~19.3 MB of scratch
        (configs.SSD_370M.with_(seqlen=1500, nheads=16, init_state=True, seed=4242), 256),
    ]
    prepared = []
    for w, chunk in cases:
        inp = inputs.make_inputs(w)
        t = torch_inputs(inp, cuda_device)
        y_ref, f_ref = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], chunk,
                                          init_state=t["init_state"])
        prepared.append((inp, chunk, t, y_ref, f_ref))
    torch.cuda.synchronize()
    outs = [_call_static(torch, t, inp.w, chunk) for inp, chunk, t, _, _ in prepared]
    torch.cuda.synchronize()
    for (inp, chunk, t, y_ref, f_ref), (y, f) in zip(prepared, outs):
        assert torch.equal(y, y_ref), "y differs from ssd_chunk_scan_fwd's"
        assert torch.equal(f, f_ref), "final state differs from ssd_chunk_scan_fwd's"
        yo, fo, _ = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init)
        yn = to_np(y)
        assert np.isfinite(yn).all()
        ey = max_rel_slices(yn, yo, (1, 3))[0]
        ef = max_rel_slices(to_np(f), fo, (2, 3))[0]
        assert ey <= TOL[inp.w.dtype], f"y relative L2 error against the oracle {ey:.3e}"
        assert ef <= TOL[inp.w.dtype], f"final state relative L2 error {ef:.3e}"


def test_static_scratch_refuses_problems_larger_than_the_array(cuda_device):
    w = configs.SSD_2P7B   # ~257 MB of scratch needed
    assert ssd.workspace_size(_shape(w), w.chunk) > 32 << 20
    p = ctypes.c_void_p(1 << 20)
    rc = _static_entry()(ctypes.byref(_shape(w)), p, p, p, p, p, p, w.chunk, None, p, None, None)
    assert rc == ssd.SSD_ERR_UNSUPPORTED
    assert "ssd_chunk_scan_fwd_static" in ssd.last_error()


def test_static_scratch_status_is_cleared_by_the_next_call(cuda_device):
    """A call whose chunk scan is made to time out (the test control of include/ssd_testing.h:
    one CTA's producer leaves its first stage unissued) leaves the scratch array's status word at
    SSD_ERR_TIMEOUT; the next call clears it and matches the oracle."""
    import torch
    arm = ssd.lib().ssd_testing_skip_stage
    arm.restype = ctypes.c_int
    arm.argtypes = [ctypes.c_int, ctypes.c_int]
    w = configs.SSD_370M.with_(batch=1, seqlen=1024, nheads=8, init_state=True, seed=608)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    torch.cuda.synchronize()
    assert arm(2, 1) == ssd.SSD_OK, ssd.last_error()   # the chunk scan, CTA 1
    stream = torch.cuda.current_stream().cuda_stream
    y = torch.empty_like(t["x"])
    final = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), dtype=torch.float32,
                        device=t["x"].device)
    rc = _static_entry()(ctypes.byref(_shape(w)), t["x"].data_ptr(), t["dt"].data_ptr(),
                         t["A"].data_ptr(), t["B"].data_ptr(), t["C"].data_ptr(),
                         t["D"].data_ptr(), w.chunk, t["init_state"].data_ptr(), y.data_ptr(),
                         final.data_ptr(), stream)
    assert rc == ssd.SSD_OK, ssd.last_error()
    assert _status_entry()(stream) == ssd.SSD_ERR_TIMEOUT
    y, final = _call_static(torch, t, w, w.chunk)   # asserts SSD_OK from the status word
    torch.cuda.synchronize()
    yo, fo, _ = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init)
    assert max_rel_slices(to_np(y), yo, (1, 3))[0] <= TOL["bf16"]
    assert max_rel_slices(to_np(final), fo, (2, 3))[0] <= TOL["bf16"]
