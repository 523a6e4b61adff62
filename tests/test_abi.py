"""Host-side checks of the C ABI that need no GPU: the library loads, exports every function the
header declares, sizes its workspace, and rejects bad arguments before touching the device."""
import ctypes
import subprocess

import pytest

from mamba_ssd_layer_scan_b200 import build, ssd


@pytest.fixture(scope="module")
def L():
    build.build()
    return ssd.lib()


def test_exports_every_declared_function(L):
    declared = ssd.declared_functions()
    assert {"ssd_chunk_scan_fwd", "ssd_state_update", "ssd_chunk_scan_workspace_size",
            "ssd_chunk_scan_varlen_fwd", "ssd_chunk_scan_varlen_workspace_size",
            "ssd_last_error"} <= set(declared)
    out = subprocess.run(["nm", "-D", "--defined-only", ssd.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    for name in declared:
        assert name in exported, name
        assert hasattr(L, name)


def test_testing_header_exported_and_validated(L):
    import re
    text = open(ssd.HEADER.replace("ssd.h", "ssd_testing.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = sorted(set(re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)))
    assert names == ["ssd_testing_skip_stage"]
    for name in names:
        assert hasattr(L, name)
    f = L.ssd_testing_skip_stage
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int, ctypes.c_int]
    assert f(7, 0) == ssd.SSD_ERR_INVALID_ARG
    assert f(2, -1) == ssd.SSD_ERR_INVALID_ARG


def test_version(L):
    assert b"sm_100a" in L.ssd_version()


def _shape(**kw):
    d = dict(batch=4, seqlen=4096, nheads=80, headdim=64, dstate=128, ngroups=1,
             dtype=ssd.SSD_BF16)
    d.update(kw)
    return ssd.make_shape(**d)


def test_workspace_size_layout():
    b, L_, H, P, N, Q = 4, 4096, 80, 64, 128, 256
    c = L_ // Q
    ws = ssd.workspace_size(_shape(), Q)
    # status word + cs (f32) + per-chunk dt rows (f32) + chunk states (f32) + bf16 entering
    # states (the last two regions only on the tensor-core path)
    expect = 256 + 2 * b * c * H * Q * 4 + b * c * H * P * N * 4 + b * c * H * P * N * 2
    assert ws == expect
    # float32 inputs run the CUDA-core path, which keeps the entering state in place (no bf16 copy)
    ws32 = ssd.workspace_size(_shape(dtype=ssd.SSD_F32), Q)
    assert ws32 == 256 + b * c * H * Q * 4 + b * c * H * P * N * 4
    # a ragged length rounds the chunk count up
    assert ssd.workspace_size(_shape(seqlen=4097), Q) > ws


@pytest.mark.parametrize("kw,code", [
    (dict(ngroups=3), ssd.SSD_ERR_INVALID_ARG),
    (dict(nheads=0), ssd.SSD_ERR_INVALID_ARG),
    (dict(batch=-1), ssd.SSD_ERR_INVALID_ARG),
    (dict(dtype=7), ssd.SSD_ERR_INVALID_ARG),
    (dict(headdim=129), ssd.SSD_ERR_UNSUPPORTED),
    (dict(dstate=48), ssd.SSD_ERR_UNSUPPORTED),
    (dict(headdim=128, dstate=256), ssd.SSD_ERR_UNSUPPORTED),
])
def test_bad_shapes_rejected(L, kw, code):
    sh = _shape(**kw)
    fake = ctypes.c_void_p(1 << 20)
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), fake, fake, fake, fake, fake, fake, 256, None,
                              fake, None, fake, 1 << 40, None)
    assert rc == code
    assert ssd.last_error()
    assert L.ssd_chunk_scan_workspace_size(ctypes.byref(sh), 256) == 0


def test_bad_chunk_and_pointers_rejected(L):
    sh = _shape()
    ok = ctypes.c_void_p(1 << 20)
    mis = ctypes.c_void_p((1 << 20) + 8)
    big = 1 << 40
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, 100, None, ok, None, ok,
                              big, None)
    assert rc == ssd.SSD_ERR_UNSUPPORTED and "chunk_size" in ssd.last_error()
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), None, ok, ok, ok, ok, ok, 256, None, ok, None,
                              ok, big, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "NULL" in ssd.last_error()
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), mis, ok, ok, ok, ok, ok, 256, None, ok, None, ok,
                              big, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "aligned" in ssd.last_error()
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, 256, None, ok, None,
                              ctypes.c_void_p((1 << 20) + 16), big, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "256-byte" in ssd.last_error()
    rc = L.ssd_chunk_scan_fwd(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, 256, None, ok, None, ok,
                              1024, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "workspace too small" in ssd.last_error()
    rc = L.ssd_chunk_scan_fwd(None, ok, ok, ok, ok, ok, ok, 256, None, ok, None, ok, big, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG


def test_empty_batch_is_a_no_op(L):
    sh = _shape(batch=0)
    assert L.ssd_chunk_scan_fwd(ctypes.byref(sh), None, None, None, None, None, None, 256, None,
                                None, None, None, 0, None) == ssd.SSD_OK
    assert L.ssd_state_update(ctypes.byref(sh), None, None, None, None, None, None, None, None,
                              None) == ssd.SSD_OK


def test_state_update_rejects_bad_args(L):
    ok = ctypes.c_void_p(1 << 20)
    sh = _shape(batch=128)
    rc = L.ssd_state_update(ctypes.byref(sh), None, ok, ok, ok, ok, ok, ok, ok, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG
    rc = L.ssd_state_update(ctypes.byref(sh), ctypes.c_void_p((1 << 20) + 4), ok, ok, ok, ok, ok,
                            ok, ok, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG
    sh = _shape(batch=128, dstate=100)
    rc = L.ssd_state_update(ctypes.byref(sh), ok, ok, ok, ok, ok, ok, ok, ok, None)
    assert rc == ssd.SSD_ERR_UNSUPPORTED


def test_product_path_has_no_cpu_fallback(tmp_path, monkeypatch):
    """With the shared library absent, the binding raises instead of computing anything."""
    monkeypatch.setattr(ssd, "_lib", None)
    monkeypatch.setattr(ssd, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        ssd.lib()


def test_varlen_workspace_size_layout():
    T, H, P, N, Q, nseq = 16384, 80, 64, 128, 256, 12
    slots = T // Q + nseq                  # chunks of any split of T tokens into nseq sequences
    r = lambda v: (v + 255) // 256 * 256
    rows = slots * H
    expect = (256 + r(slots * 8) + r((nseq + 1) * 4) + 2 * r(rows * Q * 4) + r(rows * P * N * 4)
              + r(rows * P * N * 2))
    assert ssd.varlen_workspace_size(_shape(batch=1, seqlen=T), nseq, Q) == expect


@pytest.mark.parametrize("kw,nseq,chunk,code", [
    (dict(batch=2), 3, 256, ssd.SSD_ERR_INVALID_ARG),         # packed input is one row
    (dict(batch=1), 0, 256, ssd.SSD_ERR_INVALID_ARG),         # no sequence
    (dict(batch=1, dtype=ssd.SSD_F32), 3, 256, ssd.SSD_ERR_UNSUPPORTED),
    (dict(batch=1), 3, 64, ssd.SSD_ERR_UNSUPPORTED),          # tensor-core chunk sizes only
])
def test_varlen_rejects_bad_arguments(L, kw, nseq, chunk, code):
    sh = _shape(**kw)
    assert L.ssd_chunk_scan_varlen_workspace_size(ctypes.byref(sh), nseq, chunk) == 0
    p = ctypes.c_void_p(1 << 20)
    rc = L.ssd_chunk_scan_varlen_fwd(ctypes.byref(sh), p, p, p, p, p, p, chunk, p, nseq, None, p,
                                     None, p, 1 << 40, None)
    assert rc == code
    assert ssd.last_error()


def test_fused_options_workspace_and_validation(L):
    sh = _shape()
    base = ssd.workspace_size(sh, 256)
    gate_only = ssd.FwdOptions(1 << 20, None, 0, 0.0, 0.0)
    assert L.ssd_chunk_scan_fwd_ex_workspace_size(ctypes.byref(sh), 256,
                                                  ctypes.byref(gate_only)) == base
    pro = ssd.FwdOptions(None, None, 1, 1e-3, 0.1)   # the prologue needs one dt per token-head
    r = lambda v: (v + 255) // 256 * 256
    assert L.ssd_chunk_scan_fwd_ex_workspace_size(ctypes.byref(sh), 256, ctypes.byref(pro)) == \
        base + r(4 * 4096 * 80 * 4)
    p = ctypes.c_void_p(1 << 20)
    bad = ssd.FwdOptions(ctypes.c_void_p((1 << 20) + 2), None, 0, 0.0, 0.0)   # misaligned z
    rc = L.ssd_chunk_scan_fwd_ex(ctypes.byref(sh), p, p, p, p, p, p, 256, None, p, None, p,
                                 1 << 40, None, ctypes.byref(bad))
    assert rc == ssd.SSD_ERR_INVALID_ARG and "z must" in ssd.last_error()
    inv = ssd.FwdOptions(None, None, 1, 0.5, 0.1)   # dt_min > dt_max
    rc = L.ssd_chunk_scan_fwd_ex(ctypes.byref(sh), p, p, p, p, p, p, 256, None, p, None, p,
                                 1 << 40, None, ctypes.byref(inv))
    assert rc == ssd.SSD_ERR_INVALID_ARG and "dt_min" in ssd.last_error()


def test_seqpar_workspace_and_rejections(L):
    sh = _shape()
    assert ssd.lib().ssd_seqpar_workspace_size(ctypes.byref(sh), 256) == \
        ssd.workspace_size(sh, 256) + 4 * 80 * 64 * 128 * 4
    f32 = _shape(dtype=ssd.SSD_F32)
    assert L.ssd_seqpar_workspace_size(ctypes.byref(f32), 256) == 0   # tensor-core path only
    p = ctypes.c_void_p(1 << 20)
    rc = L.ssd_seqpar_finish(ctypes.byref(sh), p, p, p, p, 256, p, p, 2, 2, None, p, None, p,
                             1 << 40, None)
    assert rc == ssd.SSD_ERR_INVALID_ARG and "rank" in ssd.last_error()


def test_backward_workspace_and_rejections(L):
    sh = _shape()
    n = L.ssd_chunk_scan_bwd_workspace_size(ctypes.byref(sh), 256)
    # two tensor-core scans' workspaces at least, plus the reversed operands
    assert n >= 2 * ssd.workspace_size(sh, 256) + 4 * 4096 * 80 * 64 * 2
    assert n % 256 == 0
    f32 = _shape(dtype=ssd.SSD_F32)
    assert L.ssd_chunk_scan_bwd_workspace_size(ctypes.byref(f32), 256) == 0
    assert L.ssd_chunk_scan_bwd_workspace_size(ctypes.byref(sh), 64) == 0
    p = ctypes.c_void_p(1 << 20)
    args = lambda **kw: [kw.get(k, p) for k in ("x", "dt", "A", "B", "C", "D")] + [256, None] + \
        [kw.get(k, p) for k in ("dy",)] + [None] + \
        [kw.get(k, p) for k in ("dx", "ddt", "dA", "dB", "dC", "dD")] + [None, p,
                                                                          kw.get("ws_bytes", n),
                                                                          None]
    rc = L.ssd_chunk_scan_bwd(ctypes.byref(f32), *args())
    assert rc == ssd.SSD_ERR_UNSUPPORTED
    rc = L.ssd_chunk_scan_bwd(ctypes.byref(sh), *args(dA=None))
    assert rc == ssd.SSD_ERR_INVALID_ARG
    rc = L.ssd_chunk_scan_bwd(ctypes.byref(sh), *args(dy=None))
    assert rc == ssd.SSD_ERR_INVALID_ARG and "dy" in ssd.last_error()
    rc = L.ssd_chunk_scan_bwd(ctypes.byref(sh), *args(dy=ctypes.c_void_p((1 << 20) + 2)))
    assert rc == ssd.SSD_ERR_INVALID_ARG and "aligned" in ssd.last_error()
    rc = L.ssd_chunk_scan_bwd(ctypes.byref(sh), *args(ws_bytes=n - 256))
    assert rc == ssd.SSD_ERR_INVALID_ARG and "workspace" in ssd.last_error()
