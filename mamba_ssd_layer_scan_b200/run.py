"""Run the scan or the decode update on one of the named synthetic workloads and print device
times per iteration (CUDA events).

    python -m mamba_ssd_layer_scan_b200.run --workload ssd_2p7b --iters 3
    python -m mamba_ssd_layer_scan_b200.run --workload ssd_decode --op decode --iters 3

Workload names: ssd_f32_small, ssd_370m, ssd_2p7b, ssd_long, ssd_decode (see configs.py).  Inputs
come from inputs.make_inputs (seeded), so a run is reproducible; this is also the command the
ncu summaries under profiles/ were captured with.
"""
from __future__ import annotations

import argparse
import json

import numpy as np

from . import configs, inputs, ssd

NAMES = {"ssd_f32_small": configs.SSD_F32_SMALL, "ssd_370m": configs.SSD_370M,
         "ssd_2p7b": configs.SSD_2P7B, "ssd_long": configs.SSD_LONG,
         "ssd_decode": configs.SSD_DECODE}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", default="ssd_2p7b", choices=sorted(NAMES))
    ap.add_argument("--op", default="scan", choices=["scan", "decode"])
    ap.add_argument("--iters", type=int, default=3)
    ap.add_argument("--chunk", type=int, default=None)
    args = ap.parse_args()
    import torch
    w = NAMES[args.workload]
    dev = torch.device("cuda", 0)
    xdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    if args.op == "decode":
        w = w.with_(seqlen=1)
    inp = inputs.make_inputs(w)

    def t(a, dtype=torch.float32):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(dtype)

    x, dt, A, B, C, D, h0 = (t(inp.x, xdt), t(inp.dt), t(inp.A), t(inp.B, xdt), t(inp.C, xdt),
                             t(inp.D), t(inp.init))
    times = []
    if args.op == "scan":
        chunk = args.chunk or w.chunk
        shape = ssd.make_shape(w.batch, w.seqlen, w.nheads, w.headdim, w.dstate, w.ngroups,
                               ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32)
        ws = ssd.new_workspace(shape, chunk, dev)
        y = torch.empty_like(x)
        final = torch.empty((w.batch, w.nheads, w.headdim, w.dstate), device=dev)
        for _ in range(args.iters):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ssd.chunk_scan_fwd(x, dt, A, B, C, D, chunk, init_state=h0, y=y, final_state=final,
                               workspace=ws)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        status = ssd.workspace_status(ws)
    else:
        state = h0.clone() if h0 is not None else torch.zeros(
            (w.batch, w.nheads, w.headdim, w.dstate), device=dev)
        y = torch.empty_like(x[:, 0])
        for _ in range(args.iters):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            ssd.state_update(state, x[:, 0].contiguous(), dt[:, 0].contiguous(), A,
                             B[:, 0].contiguous(), C[:, 0].contiguous(), D, y=y)
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
        status = 0
    print(json.dumps({"workload": w.name, "op": args.op, "ms": times, "status": status}))
    return 0 if status == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
