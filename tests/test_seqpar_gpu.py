"""GPU parity of the sequence-parallel scan (ssd_seqpar_local / ssd_seqpar_finish).

The ranks are emulated on one GPU: each contiguous segment of the sequence runs its local phase,
the per-segment outputs are stacked in rank order (what the all-gather delivers), then each
segment runs its finish phase.  The concatenated y and the last segment's final state must match
the float64 oracle on the whole sequence (bf16 tolerance, max over (batch, head) slices); with
one segment the result equals ssd_chunk_scan_fwd bit for bit.  The exchange itself
(ssd.exchange_states over torch.distributed) is tested with gloo ranks in
test_multirank_cpu.py; this run has one GPU.
"""
import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_per_pair, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _emulated(torch, t, cuts, chunk):
    segs = [(cuts[r], cuts[r + 1]) for r in range(len(cuts) - 1)]
    cut = lambda v, a, e: v[:, a:e].contiguous()
    local = [ssd.seqpar_local(cut(t["x"], a, e), cut(t["dt"], a, e), t["A"], cut(t["B"], a, e),
                              chunk) for a, e in segs]
    h_all = torch.stack([h for h, _, _ in local])
    l_all = torch.stack([l for _, l, _ in local])
    ys, finals = [], []
    for r, (a, e) in enumerate(segs):
        y, f = ssd.seqpar_finish(cut(t["x"], a, e), cut(t["B"], a, e), cut(t["C"], a, e), t["D"],
                                 local[r][2], h_all, l_all, r, chunk,
                                 init_state=t["init_state"])
        ys.append(y)
        finals.append(f)
    torch.cuda.synchronize()
    return torch.cat(ys, 1), finals[-1], local


CASES = [
    # (name, workload, segment boundaries, chunk)
    ("two_even", configs.SSD_370M.with_(batch=2, seqlen=1024, nheads=8, init_state=True),
     [0, 512, 1024], 256),
    ("four_ragged", configs.SSD_370M.with_(batch=1, seqlen=1500, nheads=8, ngroups=2,
                                          init_state=True), [0, 300, 301, 1000, 1500], 256),
    ("empty_segment_q128", configs.SSD_370M.with_(batch=2, seqlen=900, nheads=6), [0, 400, 400,
                                                                                   900], 128),
]


@pytest.mark.parametrize("name,w,cuts,chunk", CASES, ids=[c[0] for c in CASES])
def test_emulated_ranks_match_whole_sequence(cuda_device, name, w, cuts, chunk):
    import torch
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    y, final, _ = _emulated(torch, t, cuts, chunk)
    y_ref, f_ref, _ = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, inp.init)
    yn, fn = to_np(y), to_np(final)
    pairs = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    ey = max_rel_per_pair([yn[b, :, h] for b, h in pairs], [y_ref[b, :, h] for b, h in pairs])
    ef = max_rel_per_pair([fn[b, h] for b, h in pairs], [f_ref[b, h] for b, h in pairs])
    assert np.isfinite(yn).all()
    assert ey <= TOL["bf16"], f"y relative L2 error {ey:.3e}"
    assert ef <= TOL["bf16"], f"final state relative L2 error {ef:.3e}"


def test_local_phase_outputs(cuda_device):
    """h_loc is the segment's final state from zero, log_decay the sum of dt A over it."""
    import torch
    w = configs.SSD_370M.with_(batch=1, seqlen=700, nheads=4)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    h_loc, log_decay, _ = ssd.seqpar_local(t["x"], t["dt"], t["A"], t["B"], 256)
    torch.cuda.synchronize()
    _, f_ref, _ = oracle.ssd_scan(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, None)
    ld_ref = (inp.dt.astype(np.float64) * inp.A).sum(axis=1)
    assert max_rel_per_pair([to_np(h_loc)[0, h] for h in range(4)],
                            [f_ref[0, h] for h in range(4)]) <= TOL["bf16"]
    assert np.allclose(to_np(log_decay), ld_ref, rtol=1e-5, atol=1e-4)


def test_one_rank_equals_plain_scan(cuda_device):
    """With one rank the two phases run the plain scan's kernels (chunk states, then state
    passing, then the chunk scan), so they equal it bit for bit."""
    import torch
    w = configs.SSD_370M.with_(batch=2, seqlen=800, nheads=8, init_state=True)
    t = torch_inputs(inputs.make_inputs(w), cuda_device)
    y, final, _ = _emulated(torch, t, [0, 800], 256)
    y0, f0 = ssd.chunk_scan_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], 256,
                                init_state=t["init_state"])
    torch.cuda.synchronize()
    assert torch.equal(y, y0) and torch.equal(final, f0)
