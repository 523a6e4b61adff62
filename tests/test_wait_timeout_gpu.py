"""The bounded in-kernel waits give up, report SSD_ERR_TIMEOUT and leave the context usable.

Every wait of the tensor-core kernels on a shared-memory barrier ends after about 2 s: the waiting
thread records the timeout, the CTA lets its own in-flight tensor-core work and copies finish,
frees its tensor memory and returns, and the call's workspace status word reports the timeout.
A correct run never comes near the bound, so the failure is made on the host's request
(include/ssd_testing.h): one CTA's TMA producer leaves its first operand stage unissued, so the
consumers wait on a barrier that nothing will complete -- no fault, no trap, nothing out of
bounds.  The tests then check that the call reports the timeout and that the next ordinary call
on the same workspace matches the oracle.
"""
import ctypes
import time

import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_slices, to_np, torch_inputs

pytestmark = pytest.mark.gpu

SSD_TESTING_CHUNK_STATE, SSD_TESTING_CHUNK_SCAN = 1, 2


def _arm(kernel, cta):
    f = ssd.lib().ssd_testing_skip_stage
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_int]
    assert f(kernel, cta) == ssd.SSD_OK, ssd.last_error()


@pytest.mark.parametrize("kernel,cta", [(SSD_TESTING_CHUNK_SCAN, 0), (SSD_TESTING_CHUNK_SCAN, 3),
                                        (SSD_TESTING_CHUNK_STATE, 0), (SSD_TESTING_CHUNK_STATE, 2)],
                         ids=["scan_cta0", "scan_cta3", "state_cta0", "state_cta2"])
def test_wait_runs_out_reports_timeout_then_recovers(cuda_device, kernel, cta):
    import torch
    w = configs.SSD_370M.with_(batch=1, seqlen=1024, nheads=8, init_state=True, seed=606)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    shape = ssd.make_shape(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                           ssd.SSD_BF16)
    ws = ssd.new_workspace(shape, w.chunk, cuda_device)
    _arm(kernel, cta)
    t0 = time.perf_counter()
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], w.chunk,
                       init_state=t["init_state"], workspace=ws)
    assert ssd.workspace_status(ws) == ssd.SSD_ERR_TIMEOUT
    assert "bound" in ssd.last_error()
    assert time.perf_counter() - t0 < 30.0
    # the context still works and the same workspace starts clean
    y, final = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], w.chunk,
                                  init_state=t["init_state"], workspace=ws)
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK
    y_ref, f_ref, _ = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init)
    assert max_rel_slices(to_np(y), y_ref, (1, 3))[0] <= TOL["bf16"]
    assert max_rel_slices(to_np(final), f_ref, (2, 3))[0] <= TOL["bf16"]


def test_injection_is_used_once(cuda_device):
    """An armed injection affects one launch; a CTA number past the grid injects nothing."""
    import torch
    w = configs.SSD_370M.with_(batch=1, seqlen=256, nheads=4, seed=607)
    t = torch_inputs(inputs.make_inputs(w), cuda_device)
    shape = ssd.make_shape(1, 256, 4, 64, 128, 1, ssd.SSD_BF16)
    ws = ssd.new_workspace(shape, 256, cuda_device)
    _arm(SSD_TESTING_CHUNK_SCAN, 1 << 20)
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256, workspace=ws)
    assert ssd.workspace_status(ws) == ssd.SSD_OK
    ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256, workspace=ws)
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK
