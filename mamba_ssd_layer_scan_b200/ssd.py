"""Thin Python binding over the C ABI in ``include/ssd.h`` (argument marshalling only).

Every computation runs in ``libssd_b200.so``'s CUDA kernels; torch is used for device memory,
streams and dtypes.  There is no fallback: if the shared library is missing or was built
without the CUDA kernels, loading it raises.

    y, final = chunk_scan_fwd(x, dt, A, B, C, D, chunk_size=256, init_state=None)
    y, finals = chunk_scan_varlen_fwd(x, dt, A, B, C, D, cu_seqlens)   # packed sequences
    y = state_update(state, x, dt, A, B, C, D)          # state updated in place
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssd_b200.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "ssd.h")

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(5)
SSD_F32, SSD_BF16 = 0, 1


class SSDError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"ssd status {status}: {message}")
        self.status = status


class Shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("dstate", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("dtype", ctypes.c_int32)]


class FwdOptions(ctypes.Structure):
    _fields_ = [("z", ctypes.c_void_p), ("dt_bias", ctypes.c_void_p),
                ("dt_softplus", ctypes.c_int32), ("dt_min", ctypes.c_float),
                ("dt_max", ctypes.c_float)]


_lib = None
_vp = ctypes.c_void_p


def declared_functions():
    """Names of the functions ``include/ssd.h`` declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))


def lib():
    """Load the shared library (raises if it is missing: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m mamba_ssd_layer_scan_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.ssd_chunk_scan_workspace_size.restype = ctypes.c_size_t
    L.ssd_chunk_scan_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    L.ssd_chunk_scan_fwd.restype = ctypes.c_int
    L.ssd_chunk_scan_fwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                     ctypes.c_int, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]
    L.ssd_chunk_scan_fwd_staged.restype = ctypes.c_int
    L.ssd_chunk_scan_fwd_staged.argtypes = L.ssd_chunk_scan_fwd.argtypes + [
        ctypes.POINTER(ctypes.c_void_p)]
    L.ssd_chunk_scan_fwd_ex_workspace_size.restype = ctypes.c_size_t
    L.ssd_chunk_scan_fwd_ex_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int,
                                                       ctypes.POINTER(FwdOptions)]
    L.ssd_chunk_scan_fwd_ex.restype = ctypes.c_int
    L.ssd_chunk_scan_fwd_ex.argtypes = L.ssd_chunk_scan_fwd.argtypes + [
        ctypes.POINTER(FwdOptions)]
    L.ssd_seqpar_workspace_size.restype = ctypes.c_size_t
    L.ssd_seqpar_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    L.ssd_seqpar_local.restype = ctypes.c_int
    L.ssd_seqpar_local.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, ctypes.c_int, _vp,
                                   _vp, _vp, ctypes.c_size_t, _vp]
    L.ssd_seqpar_finish.restype = ctypes.c_int
    L.ssd_seqpar_finish.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, ctypes.c_int, _vp,
                                    _vp, ctypes.c_int, ctypes.c_int, _vp, _vp, _vp, _vp,
                                    ctypes.c_size_t, _vp]
    L.ssd_chunk_scan_varlen_workspace_size.restype = ctypes.c_size_t
    L.ssd_chunk_scan_varlen_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int,
                                                       ctypes.c_int]
    L.ssd_chunk_scan_varlen_fwd.restype = ctypes.c_int
    L.ssd_chunk_scan_varlen_fwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                            ctypes.c_int, _vp, ctypes.c_int, _vp, _vp, _vp, _vp,
                                            ctypes.c_size_t, _vp]
    L.ssd_chunk_scan_bwd_workspace_size.restype = ctypes.c_size_t
    L.ssd_chunk_scan_bwd_workspace_size.argtypes = [ctypes.POINTER(Shape), ctypes.c_int]
    L.ssd_chunk_scan_bwd.restype = ctypes.c_int
    L.ssd_chunk_scan_bwd.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp,
                                     ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _vp, _vp, ctypes.c_size_t, _vp]
    L.ssd_state_update.restype = ctypes.c_int
    L.ssd_state_update.argtypes = [ctypes.POINTER(Shape), _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                   _vp, _vp]
    L.ssd_state_update_ex.restype = ctypes.c_int
    L.ssd_state_update_ex.argtypes = L.ssd_state_update.argtypes + [ctypes.POINTER(FwdOptions)]
    L.ssd_workspace_status.restype = ctypes.c_int
    L.ssd_workspace_status.argtypes = [_vp, ctypes.c_size_t, _vp]
    L.ssd_last_error.restype = ctypes.c_char_p
    L.ssd_last_error.argtypes = []
    L.ssd_version.restype = ctypes.c_char_p
    L.ssd_version.argtypes = []
    _lib = L
    return L


def last_error() -> str:
    return lib().ssd_last_error().decode()


def _check(status: int):
    if status != SSD_OK:
        raise SSDError(status, last_error())


def make_shape(batch, seqlen, nheads, headdim, dstate, ngroups, dtype) -> Shape:
    return Shape(batch, seqlen, nheads, headdim, dstate, ngroups, dtype)


def workspace_size(shape: Shape, chunk_size: int) -> int:
    n = lib().ssd_chunk_scan_workspace_size(ctypes.byref(shape), chunk_size)
    if n == 0:
        raise SSDError(SSD_ERR_INVALID_ARG, last_error())
    return n


# ---------------------------------------------------------------- torch marshalling
def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"x must be float32 or bfloat16, got {t.dtype}")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _require(t, name, dtype=None, device=None):
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} must be on {device}, got {t.device}")


def new_workspace(shape: Shape, chunk_size: int, device):
    """A device buffer of ssd_chunk_scan_workspace_size bytes (256-byte aligned by torch)."""
    torch = _torch()
    return torch.empty(workspace_size(shape, chunk_size), dtype=torch.uint8, device=device)


def chunk_scan_fwd(x, dt, A, B, C, D, chunk_size: int = 256, init_state=None,
                   return_final_state: bool = True, y=None, final_state=None, workspace=None,
                   stream=None, stage_events=None, z=None, dt_bias=None,
                   dt_softplus: bool = False, dt_limit=None):
    """Chunked SSD scan.  x (b, L, H, P), dt (b, L, H) f32, A/D (H,) f32, B/C (b, L, G, N),
    init_state (b, H, P, N) f32 or None.  Returns (y, final_state or None).

    stage_events: optional list of 5 recorded-once torch.cuda.Event objects, recorded on the
    stream around the four kernels (see ssd_chunk_scan_fwd_staged).
    z, dt_bias, dt_softplus, dt_limit=(lo, hi): the fused block steps of
    ssd_chunk_scan_fwd_ex (gated output y * silu(z); dt <- clamp(softplus(dt + dt_bias)))."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    code = _dtype_code(x)
    for t, n in ((x, "x"), (B, "B"), (C, "C")):
        _require(t, n, x.dtype, dev)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D")):
        _require(t, n, torch.float32, dev)
    if init_state is not None:
        _require(init_state, "init_state", torch.float32, dev)
    shape = make_shape(b, L, H, P, N, G, code)
    opts = None
    if z is not None or dt_bias is not None or dt_softplus or dt_limit is not None:
        if stage_events is not None:
            raise ValueError("stage_events and the fused block options cannot be combined")
        if z is not None:
            _require(z, "z", x.dtype, dev)
        if dt_bias is not None:
            _require(dt_bias, "dt_bias", torch.float32, dev)
        lo, hi = dt_limit if dt_limit is not None else (0.0, 0.0)
        opts = FwdOptions(_ptr(z), _ptr(dt_bias), 1 if dt_softplus else 0, lo, hi)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    if workspace is None:
        if opts is None:
            workspace = new_workspace(shape, chunk_size, dev)
        else:
            n = lib().ssd_chunk_scan_fwd_ex_workspace_size(ctypes.byref(shape), chunk_size,
                                                          ctypes.byref(opts))
            if n == 0:
                raise SSDError(SSD_ERR_INVALID_ARG, last_error())
            workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    args = (ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
            chunk_size, _ptr(init_state), _ptr(y), _ptr(final_state), _ptr(workspace),
            workspace.numel(), _stream_handle(stream))
    if opts is not None:
        _check(lib().ssd_chunk_scan_fwd_ex(*args, ctypes.byref(opts)))
    elif stage_events is None:
        _check(lib().ssd_chunk_scan_fwd(*args))
    else:
        handles = (ctypes.c_void_p * 5)(*[ev.cuda_event for ev in stage_events])
        _check(lib().ssd_chunk_scan_fwd_staged(*args, handles))
    return y, final_state


class CapturedScan:
    """One chunk_scan_fwd call captured into a CUDA graph, replayed as a whole.

    For steps short enough that launching the scan's kernels is a visible share of the step (at
    2 x 2048 tokens x 24 heads the replay takes about 42 us against 48 us for the launched call;
    at 4 x 4096 x 80 the two are equal).  The graph holds the call's kernels with their
    programmatic dependent launches, bound to the tensors given here: refill x, dt, A, B, C, D
    (and init_state) in place between replays; the outputs land in ``y`` and ``final_state``
    each time.  Keyword arguments are those of chunk_scan_fwd (the fused block options
    included; stage_events excluded)."""

    def __init__(self, x, dt, A, B, C, D, chunk_size: int = 256, init_state=None, **kw):
        torch = _torch()
        if "stage_events" in kw or "stream" in kw:
            raise ValueError("CapturedScan takes no stage_events or stream")
        dev = x.device
        b, L, H, P = x.shape
        N = B.shape[3]
        self.y = kw.pop("y", None)
        if self.y is None:
            self.y = torch.empty_like(x)
        self.final_state = kw.pop("final_state", None)
        if self.final_state is None and kw.pop("return_final_state", True):
            self.final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
        self.workspace = kw.pop("workspace", None)
        args = (x, dt, A, B, C, D, chunk_size)

        def call(stream):
            chunk_scan_fwd(*args, init_state=init_state, y=self.y,
                           final_state=self.final_state,
                           return_final_state=self.final_state is not None,
                           workspace=self.workspace, stream=stream, **kw)

        if self.workspace is None:   # allocated once, outside the capture
            self.workspace = _workspace_for(x, B, chunk_size, kw)
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            call(side)   # first launch outside the capture (module load, kernel attributes)
        side.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=side):
            call(side)
        torch.cuda.current_stream(dev).wait_stream(side)

    def replay(self):
        """Run the captured call on the current stream; returns (y, final_state)."""
        self.graph.replay()
        return self.y, self.final_state


def _workspace_for(x, B, chunk_size, kw):
    """The workspace chunk_scan_fwd would allocate for this call."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    shape = make_shape(b, L, H, P, N, G, _dtype_code(x))
    z, dt_bias = kw.get("z"), kw.get("dt_bias")
    if z is None and dt_bias is None and not kw.get("dt_softplus") and kw.get("dt_limit") is None:
        return new_workspace(shape, chunk_size, x.device)
    lo, hi = kw.get("dt_limit") or (0.0, 0.0)
    opts = FwdOptions(_ptr(z), _ptr(dt_bias), 1 if kw.get("dt_softplus") else 0, lo, hi)
    n = lib().ssd_chunk_scan_fwd_ex_workspace_size(ctypes.byref(shape), chunk_size,
                                                  ctypes.byref(opts))
    if n == 0:
        raise SSDError(SSD_ERR_INVALID_ARG, last_error())
    return torch.empty(n, dtype=torch.uint8, device=x.device)


def varlen_workspace_size(shape: Shape, nseq: int, chunk_size: int) -> int:
    n = lib().ssd_chunk_scan_varlen_workspace_size(ctypes.byref(shape), nseq, chunk_size)
    if n == 0:
        raise SSDError(SSD_ERR_INVALID_ARG, last_error())
    return n


def chunk_scan_varlen_fwd(x, dt, A, B, C, D, cu_seqlens, chunk_size: int = 256,
                          init_states=None, return_final_states: bool = True, y=None,
                          final_states=None, workspace=None, stream=None):
    """Packed variable-length scan.  x (1, T, H, P), dt (1, T, H) f32, B/C (1, T, G, N),
    cu_seqlens (nseq + 1,) int32 on the device, init_states (nseq, H, P, N) f32 or None.
    Returns (y, final_states or None); sequence s is tokens cu_seqlens[s] .. cu_seqlens[s+1]-1
    and carries its own state."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    code = _dtype_code(x)
    for t, n in ((x, "x"), (B, "B"), (C, "C")):
        _require(t, n, x.dtype, dev)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D")):
        _require(t, n, torch.float32, dev)
    _require(cu_seqlens, "cu_seqlens", torch.int32, dev)
    nseq = cu_seqlens.numel() - 1
    if init_states is not None:
        _require(init_states, "init_states", torch.float32, dev)
    shape = make_shape(b, L, H, P, N, G, code)
    if y is None:
        y = torch.empty_like(x)
    if final_states is None and return_final_states:
        final_states = torch.empty((nseq, H, P, N), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = torch.empty(varlen_workspace_size(shape, nseq, chunk_size),
                                dtype=torch.uint8, device=dev)
    _check(lib().ssd_chunk_scan_varlen_fwd(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), chunk_size,
        _ptr(cu_seqlens), nseq, _ptr(init_states), _ptr(y), _ptr(final_states), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)))
    return y, final_states


# ---------------------------------------------------------------- sequence parallelism
def bwd_workspace_size(shape: Shape, chunk_size: int) -> int:
    n = lib().ssd_chunk_scan_bwd_workspace_size(ctypes.byref(shape), chunk_size)
    if n == 0:
        raise SSDError(SSD_ERR_UNSUPPORTED, last_error())
    return n


def chunk_scan_bwd(x, dt, A, B, C, D, dy, chunk_size: int = 256, init_state=None, dfinal=None,
                   return_dinit: bool = True, workspace=None, stream=None):
    """Gradients of the chunked scan (ssd_chunk_scan_bwd): given dy (like y) and dfinal
    (b, H, P, N) f32 or None, returns a dict of float32 tensors dx (b, L, H, P), ddt (b, L, H),
    dA (H,), dB and dC (b, L, G, N), dD (H,) and dinit (b, H, P, N) (None unless
    return_dinit).  bf16 tensor-core shapes only."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    for t, n in ((x, "x"), (B, "B"), (C, "C"), (dy, "dy")):
        _require(t, n, x.dtype, dev)
    for t, n in ((dt, "dt"), (A, "A"), (D, "D")):
        _require(t, n, torch.float32, dev)
    for t, n in ((init_state, "init_state"), (dfinal, "dfinal")):
        if t is not None:
            _require(t, n, torch.float32, dev)
    if tuple(dy.shape) != tuple(x.shape):
        raise ValueError(f"dy must have x's shape {tuple(x.shape)}, got {tuple(dy.shape)}")
    shape = make_shape(b, L, H, P, N, G, _dtype_code(x))
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(shape, chunk_size), dtype=torch.uint8,
                                device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    g = dict(dx=torch.empty((b, L, H, P), **f32), ddt=torch.empty((b, L, H), **f32),
             dA=torch.empty((H,), **f32), dB=torch.empty((b, L, G, N), **f32),
             dC=torch.empty((b, L, G, N), **f32), dD=torch.empty((H,), **f32),
             dinit=torch.empty((b, H, P, N), **f32) if return_dinit else None)
    _check(lib().ssd_chunk_scan_bwd(
        ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), chunk_size,
        _ptr(init_state), _ptr(dy), _ptr(dfinal), _ptr(g["dx"]), _ptr(g["ddt"]), _ptr(g["dA"]),
        _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g["dD"]), _ptr(g["dinit"]), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)))
    return g


def seqpar_local(x, dt, A, B, chunk_size: int = 256, workspace=None, stream=None):
    """Phase 1 on this rank's segment: (h_loc (b, H, P, N) f32, log_decay (b, H) f32,
    workspace to pass on to seqpar_finish)."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    shape = make_shape(b, L, H, P, N, G, _dtype_code(x))
    if workspace is None:
        n = lib().ssd_seqpar_workspace_size(ctypes.byref(shape), chunk_size)
        if n == 0:
            raise SSDError(SSD_ERR_INVALID_ARG, last_error())
        workspace = torch.empty(n, dtype=torch.uint8, device=dev)
    h_loc = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    log_decay = torch.empty((b, H), dtype=torch.float32, device=dev)
    _check(lib().ssd_seqpar_local(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B),
                                  chunk_size, _ptr(h_loc), _ptr(log_decay), _ptr(workspace),
                                  workspace.numel(), _stream_handle(stream)))
    return h_loc, log_decay, workspace


def seqpar_finish(x, B, C, D, workspace, h_loc_all, log_decay_all, rank: int,
                  chunk_size: int = 256, init_state=None, y=None, final_state=None,
                  return_final_state: bool = True, stream=None):
    """Phase 3 on this rank's segment, after the exchange: (y, final_state or None)."""
    torch = _torch()
    b, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dev = x.device
    shape = make_shape(b, L, H, P, N, G, _dtype_code(x))
    nranks = h_loc_all.shape[0]
    if y is None:
        y = torch.empty_like(x)
    if final_state is None and return_final_state:
        final_state = torch.empty((b, H, P, N), dtype=torch.float32, device=dev)
    _check(lib().ssd_seqpar_finish(ctypes.byref(shape), _ptr(x), _ptr(B), _ptr(C), _ptr(D),
                                   chunk_size, _ptr(h_loc_all), _ptr(log_decay_all), nranks,
                                   rank, _ptr(init_state), _ptr(y), _ptr(final_state),
                                   _ptr(workspace), workspace.numel(), _stream_handle(stream)))
    return y, final_state


def exchange_states(h_loc, log_decay, group=None):
    """The one exchange of the sequence-parallel scan: every rank's local final state and
    segment log-decay, gathered in rank order (torch.distributed all_gather; NCCL over NVLink on
    GPUs, gloo on CPU).  Returns (h_loc_all [nranks, ...], log_decay_all [nranks, ...])."""
    torch = _torch()
    import torch.distributed as dist
    n = dist.get_world_size(group)
    hs = [torch.empty_like(h_loc) for _ in range(n)]
    ls = [torch.empty_like(log_decay) for _ in range(n)]
    dist.all_gather(hs, h_loc.contiguous(), group=group)
    dist.all_gather(ls, log_decay.contiguous(), group=group)
    return torch.stack(hs), torch.stack(ls)


def seqpar_scan(x, dt, A, B, C, D, chunk_size: int = 256, init_state=None, group=None,
                stream=None):
    """Sequence-parallel scan of this rank's contiguous segment (ranks hold the segments in
    order): local phase, one all-gather of states, finish.  Returns (y, final_state); the final
    state of the whole sequence is the last rank's."""
    import torch.distributed as dist
    h_loc, log_decay, ws = seqpar_local(x, dt, A, B, chunk_size, stream=stream)
    h_all, l_all = exchange_states(h_loc, log_decay, group)
    return seqpar_finish(x, B, C, D, ws, h_all, l_all, dist.get_rank(group), chunk_size,
                         init_state=init_state, stream=stream)


def state_update(state, x, dt, A, B, C, D, y=None, stream=None, z=None, dt_bias=None,
                 dt_softplus: bool = False, dt_limit=None):
    """One decode step.  state (b, H, P, N) f32 (in place), x (b, H, P), dt (b, H) f32,
    B/C (b, G, N).  Returns y (b, H, P).  z, dt_bias, dt_softplus, dt_limit: the block's fused
    steps (ssd_state_update_ex)."""
    torch = _torch()
    b, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    dev = x.device
    code = _dtype_code(x)
    for t, n in ((x, "x"), (B, "B"), (C, "C")):
        _require(t, n, x.dtype, dev)
    for t, n in ((state, "state"), (dt, "dt"), (A, "A"), (D, "D")):
        _require(t, n, torch.float32, dev)
    shape = make_shape(b, 1, H, P, N, G, code)
    if y is None:
        y = torch.empty_like(x)
    args = (ctypes.byref(shape), _ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C),
            _ptr(D), _ptr(y), _stream_handle(stream))
    if z is None and dt_bias is None and not dt_softplus and dt_limit is None:
        _check(lib().ssd_state_update(*args))
    else:
        if z is not None:
            _require(z, "z", x.dtype, dev)
        lo, hi = dt_limit if dt_limit is not None else (0.0, 0.0)
        opts = FwdOptions(_ptr(z), _ptr(dt_bias), 1 if dt_softplus else 0, lo, hi)
        _check(lib().ssd_state_update_ex(*args, ctypes.byref(opts)))
    return y


def workspace_status(workspace, stream=None) -> int:
    """Synchronise and return the status word the last scan on ``workspace`` left (0 = OK)."""
    return lib().ssd_workspace_status(_ptr(workspace), workspace.numel(), _stream_handle(stream))
