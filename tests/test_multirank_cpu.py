"""Multi-rank host logic on CPU (gloo, world size 2): the benchmark's max-over-ranks timing and
whole-job throughput, and the reference arm under torchrun (rank 0 alone prints one line).

The scan and the decode update shard over (batch, head) with no exchange between ranks, so a
multi-GPU run is one independent replica per GPU; what is shared across ranks is only the timing.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mx = bench.max_over_ranks(10.0 + 5.0 * rank)        # rank 1 is the slow one
        out.put((rank, mx, bench.scaled_throughput(1000.0, world, mx)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_throughput_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, mx, thr in res:
        assert mx == 15.0                                  # every rank sees the slowest time
        assert thr == pytest.approx(world * 1000.0 / 15.0)


def test_single_process_max_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.scaled_throughput(10.0, 1, 2.0) == 5.0


def test_reference_arm_under_torchrun_prints_once():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["n_gpus"] == 2
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


# ------------------------------------------------------------------ sequence parallelism
def _seqpar_worker(rank, world, port, out):
    """Each rank owns one contiguous segment of a sequence: its local state from zero and its
    log-decay (oracle), the exchange through the library's own exchange_states over gloo, the
    combine, then the oracle on the segment from the combined state."""
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from mamba_ssd_layer_scan_b200 import ssd
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(123)          # every rank draws the same whole sequence
        b, L, H, P, N, G = 2, 90, 3, 4, 5, 1
        x = rng.standard_normal((b, L, H, P))
        dt = rng.uniform(0.01, 0.3, (b, L, H))
        A = -rng.uniform(0.2, 2.0, H)
        B = rng.standard_normal((b, L, G, N))
        C = rng.standard_normal((b, L, G, N))
        D = rng.standard_normal(H)
        h0 = rng.standard_normal((b, H, P, N))
        cut = [0, 37, L]                          # uneven segments
        a, e = cut[rank], cut[rank + 1]
        seg = lambda t: t[:, a:e]
        _, h_loc, _ = oracle.ssd_scan(seg(x), seg(dt), A, seg(B), seg(C), D, None)
        log_decay = (seg(dt) * A).sum(axis=1)     # sum over the segment's tokens of dt A_h
        h_all, l_all = ssd.exchange_states(torch.from_numpy(h_loc), torch.from_numpy(log_decay))
        h_in = h0.copy()
        for q in range(rank):                     # the combine, in rank order
            h_in = np.exp(l_all[q].numpy())[:, :, None, None] * h_in + h_all[q].numpy()
        y, fin, _ = oracle.ssd_scan(seg(x), seg(dt), A, seg(B), seg(C), D, h_in)
        y_full, f_full, _ = oracle.ssd_scan(x, dt, A, B, C, D, h0)
        err_y = float(np.max(np.abs(y - y_full[:, a:e])) / np.max(np.abs(y_full)))
        err_f = float(np.max(np.abs(fin - f_full)) / np.max(np.abs(f_full))) if rank == world - 1 else 0.0
        out.put((rank, err_y, err_f, tuple(h_all.shape)))
    finally:
        dist.destroy_process_group()


def test_sequence_parallel_exchange_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_seqpar_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err_y, err_f, shape in res:
        assert shape == (world, 2, 3, 4, 5)
        assert err_y < 1e-12 and err_f < 1e-12
