"""GPU parity of the backward pass (ssd_chunk_scan_bwd) against the float64 adjoint oracle.

Every gradient is compared with oracle.ssd_scan_bwd on the same seeded inputs and upstream
gradients (dy rounded to bf16 like y, dfinal float32).  The bar is the bf16 bound of the forward,
max over slices of the relative L2 error: per (batch, head) for dx, ddt and dinit, per
(batch, group) for dB and dC, over the head vector for dA and dD (those are sums over the batch
and the sequence).  The cases span several chunks with a ragged tail, both tensor-core chunk
sizes, several groups, with and without an initial state and dfinal, one token, and the
2.7B-layer shape with every slice of every gradient.
"""
import numpy as np
import pytest

import oracle
from mamba_ssd_layer_scan_b200 import configs, inputs, ssd

from _util import TOL, max_rel_per_pair, rel_l2, to_np, torch_inputs

pytestmark = pytest.mark.gpu


def _run(torch, inp, gin, chunk, device, with_init=True, with_dfinal=True):
    t = torch_inputs(inp, device)
    dy = torch.from_numpy(gin.dy).to(device).to(t["x"].dtype)
    dfinal = torch.from_numpy(gin.dfinal).to(device) if with_dfinal else None
    init = t["init_state"] if with_init else None
    g = ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], dy, chunk,
                           init_state=init, dfinal=dfinal)
    torch.cuda.synchronize()
    return {k: (None if v is None else to_np(v)) for k, v in g.items()}


def _check(w, g, ref, names=("dx", "ddt", "dB", "dC", "dA", "dD", "dinit")):
    b, H, G = w.batch, w.nheads, w.ngroups
    errs = {}
    for k in names:
        if k in ("dx", "ddt"):
            errs[k] = max_rel_per_pair([g[k][i, :, h] for i in range(b) for h in range(H)],
                                       [ref[k][i, :, h] for i in range(b) for h in range(H)])
        elif k in ("dB", "dC"):
            errs[k] = max_rel_per_pair([g[k][i, :, j] for i in range(b) for j in range(G)],
                                       [ref[k][i, :, j] for i in range(b) for j in range(G)])
        elif k == "dinit":
            errs[k] = max_rel_per_pair([g[k][i, h] for i in range(b) for h in range(H)],
                                       [ref[k][i, h] for i in range(b) for h in range(H)])
        else:
            errs[k] = rel_l2(g[k], ref[k])
        assert np.isfinite(g[k]).all(), k
    bad = {k: e for k, e in errs.items() if not e <= TOL["bf16"]}
    assert not bad, f"relative L2 errors above {TOL['bf16']}: {bad} (all: {errs})"


CASES = [
    # (name, workload, chunk, with init_state, with dfinal)
    ("q256_ragged_init", configs.SSD_370M.with_(batch=2, seqlen=600, nheads=8, ngroups=2,
                                                 init_state=True), 256, True, True),
    ("q128_ragged", configs.SSD_370M.with_(batch=1, seqlen=333, nheads=6, seed=77), 128, False,
     True),
    ("q256_no_dfinal", configs.SSD_370M.with_(batch=1, seqlen=512, nheads=4, init_state=True,
                                               seed=78), 256, True, False),
    ("q256_groups4", configs.SSD_370M.with_(batch=1, seqlen=700, nheads=8, ngroups=4,
                                             init_state=True, seed=79), 256, True, True),
    ("one_token", configs.SSD_370M.with_(batch=2, seqlen=1, nheads=4, init_state=True, seed=80),
     256, True, True),
    # three heads per group: the dB / dC chunk outputs take one head per CTA
    ("q256_three_heads_per_group", configs.SSD_370M.with_(batch=2, seqlen=300, nheads=6,
                                                          ngroups=2, init_state=True, seed=81),
     256, True, True),
]


@pytest.mark.parametrize("name,w,chunk,with_init,with_dfinal", CASES, ids=[c[0] for c in CASES])
def test_backward_parity_every_gradient(cuda_device, name, w, chunk, with_init, with_dfinal):
    import torch
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g = _run(torch, inp, gin, chunk, cuda_device, with_init, with_dfinal)
    ref = oracle.ssd_scan_bwd(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, gin.dy,
                              init=inp.init if with_init else None,
                              dfinal=gin.dfinal if with_dfinal else None)
    _check(w, g, ref)


def test_backward_full_size_every_gradient(cuda_device):
    """The 2.7B-layer shape (batch 4, 4096 tokens, 80 heads, one group) in one call, with an
    initial state and dfinal: all seven gradients, every slice, against the adjoint oracle."""
    import torch
    w = configs.SSD_2P7B.with_(init_state=True)
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g = _run(torch, inp, gin, w.chunk, cuda_device)
    ref = oracle.ssd_scan_bwd(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, gin.dy, init=inp.init,
                              dfinal=gin.dfinal)
    _check(w, g, ref)


def test_backward_is_deterministic(cuda_device):
    """Two calls on the same inputs give bit-identical gradients (no order-dependent sums)."""
    import torch
    w = configs.SSD_370M.with_(batch=3, seqlen=700, nheads=8, ngroups=2, init_state=True,
                               seed=84)
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g1 = _run(torch, inp, gin, 256, cuda_device)
    g2 = _run(torch, inp, gin, 256, cuda_device)
    for k in g1:
        assert np.array_equal(g1[k], g2[k]), k


def test_backward_dD_and_linearity_in_D(cuda_device):
    """dD_h is sum <dy, x> over the batch and the sequence, and D enters the gradients only
    through dx = D dy + (a term independent of D): properties that hold at any size."""
    import torch
    w = configs.SSD_370M.with_(batch=1, seqlen=1024, nheads=8, seed=81)
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g1 = _run(torch, inp, gin, 256, cuda_device, False, True)
    inp.D = inp.D + 0.5
    g2 = _run(torch, inp, gin, 256, cuda_device, False, True)
    dD = np.einsum("blhp,blhp->h", gin.dy.astype(np.float64), inp.x.astype(np.float64))
    assert rel_l2(g1["dD"], dD) <= 1e-5
    diff = (g2["dx"] - g1["dx"]) - 0.5 * gin.dy
    assert np.abs(diff).max() <= 1e-5 * max(1.0, np.abs(g1["dx"]).max())
    for k in ("ddt", "dB", "dC", "dA", "dinit"):
        assert np.array_equal(g1[k], g2[k]), k


def test_backward_unsupported_shape_rejected(cuda_device):
    import torch
    w = configs.SSD_F32_SMALL.with_(batch=1, seqlen=64, nheads=2)
    inp = inputs.make_inputs(w)
    t = torch_inputs(inp, cuda_device)
    with pytest.raises(ssd.SSDError):
        ssd.chunk_scan_bwd(t["x"], t["dt"], t["A"], t["B"], t["C"], t["D"], t["x"].clone(), 64)


def test_backward_empty_sequence(cuda_device):
    """No token: the final state is the initial state, so dinit = dfinal exactly and every other
    gradient is empty or zero."""
    import torch
    w = configs.SSD_370M.with_(batch=2, seqlen=0, nheads=4, init_state=True, seed=82)
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g = _run(torch, inp, gin, 256, cuda_device)
    assert np.array_equal(g["dinit"], gin.dfinal)
    assert not g["dA"].any() and not g["dD"].any()
    for k in ("dx", "ddt", "dB", "dC"):
        assert g[k].size == 0, k
    g = _run(torch, inp, gin, 256, cuda_device, with_dfinal=False)
    assert not g["dinit"].any()


def test_backward_empty_batch(cuda_device):
    import torch
    w = configs.SSD_370M.with_(batch=0, seqlen=300, nheads=4, seed=83)
    inp = inputs.make_inputs(w)
    gin = inputs.make_grad_inputs(w)
    g = _run(torch, inp, gin, 256, cuda_device, with_init=False)
    assert not g["dA"].any() and not g["dD"].any()
    assert g["dx"].size == 0 and g["dinit"].size == 0
