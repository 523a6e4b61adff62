"""A scan captured into a CUDA graph (ssd.CapturedScan) against the launched call.

The graph holds the same kernels on the same buffers, so each replay must give the launched
call's result bit for bit, also after the inputs are refilled in place, and match the oracle.
"""
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_slices, to_np, torch_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("gated", [False, True], ids=["plain", "gated"])
def test_replay_equals_launched_call_after_refill(cuda_device, gated):
    import torch
    w1 = configs.SSD_370M.with_(batch=2, seqlen=700, nheads=8, init_state=True, seed=71)
    i1, i2 = inputs.make_inputs(w1), inputs.make_inputs(w1.with_(seed=72))
    t, t2 = torch_inputs(i1, cuda_device), torch_inputs(i2, cuda_device)
    kw = {}
    if gated:
        kw = dict(z=torch.randn(t["x"].shape, device=cuda_device).to(t["x"].dtype))
    cap = ssd.CapturedScan(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                           init_state=t["init_state"], **kw)

    def replay_and_compare():
        y, final = (v.clone() for v in cap.replay())
        y_ref, f_ref = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                          init_state=t["init_state"], **kw)
        torch.cuda.synchronize()
        assert ssd.workspace_status(cap.workspace) == ssd.SSD_OK
        assert torch.equal(y, y_ref) and torch.equal(final, f_ref)
        return y, final

    replay_and_compare()
    for k in ("x", "dt", "A", "B", "C", "D", "init_state"):   # refill the captured inputs
        t[k].copy_(t2[k])
    y, final = replay_and_compare()
    if not gated:
        yo, fo, _ = oracle.ssd_scan(i2.x, i2.dt, i2.A, i2.B, i2.C, i2.D, i2.init)
        assert max_rel_slices(to_np(y), yo, (1, 3))[0] <= TOL["bf16"]
        assert max_rel_slices(to_np(final), fo, (2, 3))[0] <= TOL["bf16"]
