"""GPU parity of the packed variable-length scan (ssd_chunk_scan_varlen_fwd) through the C ABI.

Packed sequences share one batch row; each carries its own state, so the reference for sequence
s is the float64 oracle run on that sequence alone from its own initial state.  The tolerance is
the bf16 bound, max over (sequence, head) slices of the relative L2 error of y and of the final
states.  The cases cover an empty sequence, one-token sequences, sequences of exactly one chunk
and one chunk plus a token, several groups, both tensor-core chunk sizes, the full-size packed
workload (every slice), and cu_seqlens that the device rejects.
"""
import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_per_pair, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _packed(w, cu):
    """Input draw of workload w (batch 1, seqlen = cu[-1]) with explicit sequence boundaries."""
    inp = inputs.make_inputs(w.with_(batch=1, seqlen=int(cu[-1]), nseq=0, init_state=False))
    rng = np.random.default_rng(w.seed + 11)
    init = (0.1 * rng.standard_normal((len(cu) - 1, w.nheads, w.headdim, w.dstate))
            ).astype(np.float32)
    return inp, np.asarray(cu, dtype=np.int32), init


def _run(torch, inp, cu, init, chunk, device):
    t = torch_inputs(inp, device)
    cu_t = torch.from_numpy(cu).to(device)
    init_t = None if init is None else torch.from_numpy(init).to(device)
    w = inp.w
    shape = ssd.make_shape(1, int(cu[-1]), w.nheads, w.headdim, w.dstate, w.ngroups, ssd.SSD_BF16)
    ws = torch.empty(ssd.varlen_workspace_size(shape, len(cu) - 1, chunk), dtype=torch.uint8,
                     device=device)
    y, final = ssd.chunk_scan_varlen_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], cu_t,
                                         chunk, init_states=init_t, workspace=ws)
    torch.cuda.synchronize()
    assert ssd.workspace_status(ws) == ssd.SSD_OK, ssd.last_error()
    return t, y, final


def _check_all(inp, cu, init, y, final):
    y_ref, f_ref = oracle.ssd_scan_varlen(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, cu, init)
    yn, fn = to_np(y), to_np(final)
    H = inp.w.nheads
    nonempty = [s for s in range(len(cu) - 1) if cu[s + 1] > cu[s]]
    ey = max_rel_per_pair([yn[0, cu[s]:cu[s + 1], h] for s in nonempty for h in range(H)],
                          [y_ref[0, cu[s]:cu[s + 1], h] for s in nonempty for h in range(H)])
    ef = max_rel_per_pair([fn[s, h] for s in range(len(cu) - 1) for h in range(H)],
                          [f_ref[s, h] for s in range(len(cu) - 1) for h in range(H)])
    assert np.isfinite(yn).all()
    assert ey <= TOL["bf16"], f"y relative L2 error {ey:.3e}"
    assert ef <= TOL["bf16"], f"final state relative L2 error {ef:.3e}"


CASES = [
    # (name, workload, cu_seqlens, chunk)
    ("edges_q256", configs.SSD_370M.with_(nheads=8, ngroups=2),
     [0, 1, 257, 257, 513, 770, 1000], 256),
    ("edges_q128", configs.SSD_370M.with_(nheads=8, ngroups=2),
     [0, 1, 129, 129, 257, 386, 600], 128),
    ("many_short", configs.SSD_370M.with_(nheads=4, seed=2024),
     [0, 3, 40, 41, 42, 100, 300, 301, 555], 256),
    ("groups_8", configs.SSD_LONG.with_(nheads=16, ngroups=8),
     [0, 700, 1400, 1401, 2000], 256),
]


@pytest.mark.parametrize("name,w,cu,chunk", CASES, ids=[c[0] for c in CASES])
def test_packed_parity_every_output(cuda_device, name, w, cu, chunk):
    import torch
    inp, cu, init = _packed(w, cu)
    _, y, final = _run(torch, inp, cu, init, chunk, cuda_device)
    _check_all(inp, cu, init, y, final)


def test_packed_without_initial_states(cuda_device):
    import torch
    inp, cu, _ = _packed(configs.SSD_370M.with_(nheads=8, seed=31), [0, 300, 301, 900])
    _, y, final = _run(torch, inp, cu, None, 256, cuda_device)
    _check_all(inp, cu, None, y, final)


def test_packed_equals_separate_calls(cuda_device):
    """Each sequence's chunks are cut exactly as a standalone call cuts them, so the packed result
    equals ssd_chunk_scan_fwd on every sequence alone, bit for bit."""
    import torch
    inp, cu, init = _packed(configs.SSD_370M.with_(nheads=8, ngroups=2, seed=99),
                            [0, 513, 514, 1300, 1800])
    t, y, final = _run(torch, inp, cu, init, 256, cuda_device)
    for s in range(len(cu) - 1):
        a, e = int(cu[s]), int(cu[s + 1])
        init_s = torch.from_numpy(init[s:s + 1].copy()).to(cuda_device)
        y_s, f_s = ssd.chunk_scan_fwd(*(t[k][:, a:e].contiguous() for k in ("x", "dt")), t["A"],
                                      t["B"][:, a:e].contiguous(), t["C"][:, a:e].contiguous(),
                                      t["D"], 256, init_state=init_s)
        torch.cuda.synchronize()
        assert torch.equal(y[:, a:e], y_s), f"sequence {s}: y differs"
        assert torch.equal(final[s], f_s[0]), f"sequence {s}: final state differs"


def test_full_size_packed_workload_every_output(cuda_device):
    """The full packed workload (16384 tokens as 12 sequences, 80 heads): every (sequence, head)
    slice of y and of the final states against the oracle run on each sequence alone."""
    import torch
    w = configs.SSD_VARLEN
    inp = inputs.make_inputs(w)
    cu = inp.cu_seqlens
    _, y, final = _run(torch, inp, cu, inp.init, w.chunk, cuda_device)
    _check_all(inp, cu, inp.init, y, final)


def test_inconsistent_cu_seqlens_reported(cuda_device):
    import torch
    inp, _, _ = _packed(configs.SSD_370M.with_(nheads=4), [0, 400])
    bad = np.array([0, 300, 200, 400], dtype=np.int32)   # decreasing
    t = torch_inputs(inp, cuda_device)
    shape = ssd.make_shape(1, 400, 4, 64, 128, 1, ssd.SSD_BF16)
    ws = torch.empty(ssd.varlen_workspace_size(shape, 3, 256), dtype=torch.uint8,
                     device=cuda_device)
    ssd.chunk_scan_varlen_fwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"],
                              torch.from_numpy(bad).to(cuda_device), 256, workspace=ws)
    assert ssd.workspace_status(ws) == ssd.SSD_ERR_INVALID_ARG
    assert "cu_seqlens" in ssd.last_error()
