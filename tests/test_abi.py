"""The C-ABI library: it loads, exports every symbol include/ssm.h declares,
and rejects bad arguments before touching a GPU.  Runs without a GPU: every
call here returns during host-side validation (or is a no-op on empty sizes),
so nothing is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssm.h")


@pytest.fixture(scope="module")
def b():
    from selective_state_space_36_b200 import build
    build.build()
    from selective_state_space_36_b200 import binding
    return binding


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssm_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(b):
    names = declared_functions()
    assert set(names) == set(b.EXPORTED)
    for n in names:
        assert hasattr(b.lib, n), f"{n} not exported"
    assert b.lib.ssm_version() >= 100
    assert b.lib.ssm_status_string(0) == b"ok"


def _scan(b, dims, io=1, ptrs=None, softplus=1, opts=None):
    # ptrs: u, delta, A, B, C, D, z, bias, out, last_state
    p = dict(u=0x10000, delta=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None,
             bias=None, out=0x60000, state=None)
    p.update(ptrs or {})
    args = [b.SSMDims(*dims), io, p["u"], p["delta"], p["A"], p["B"], p["C"], p["D"], p["z"],
            p["bias"], softplus, p["out"], p["state"]]
    if opts is None:
        return b.lib.ssm_selective_scan_fwd(*args, None)
    return b.lib.ssm_selective_scan_fwd_ex(*args, ctypes.byref(opts), None)


def test_scan_argument_validation(b):
    ok = (2, 16, 8, 16)
    assert _scan(b, ok, io=7) == b.SSM_ERR_INVALID_ARG
    assert b"io dtype" in b.lib.ssm_last_error()
    assert _scan(b, (2, -1, 8, 16)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, (2, 16, 8, 0)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, (2, 16, 8, 65)) == b.SSM_ERR_UNSUPPORTED
    assert _scan(b, ok, softplus=2) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, ok, ptrs=dict(u=None)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, ok, ptrs=dict(out=None)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, ok, ptrs=dict(C=None)) == b.SSM_ERR_INVALID_ARG
    # misaligned: bf16 needs 2-byte, float32 params 4-byte alignment
    assert _scan(b, ok, ptrs=dict(u=0x10001)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, ok, ptrs=dict(A=0x30002)) == b.SSM_ERR_INVALID_ARG
    assert _scan(b, ok, io=0, ptrs=dict(z=0x70002)) == b.SSM_ERR_INVALID_ARG
    assert b"aligned" in b.lib.ssm_last_error()
    # overflow of the index space
    assert _scan(b, (1 << 40, 1 << 40, 8, 16)) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(9, 0)
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(2, -3)
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(1, 0, 3)
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(1, 0, 0, 5)
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(1, 0, 0, 0)
    opts.reserved[1] = 1
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(1, 0, 0, 0, 0, 7)  # unknown discretization
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    opts = b.SSMScanOpts(1, 0, 0, 2, 2, 1)  # exact ZOH with two channels per lane
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_UNSUPPORTED
    opts = b.SSMScanOpts(1, 0, 0, 0, 3)  # channels per lane must be 0, 1 or 2
    assert _scan(b, ok, opts=opts) == b.SSM_ERR_INVALID_ARG
    # staged kernel on rows that are not 16-byte multiples: refused before launch
    opts = b.SSMScanOpts(1, 0, 0, 2)
    assert _scan(b, (2, 16, 37, 16), opts=opts) == b.SSM_ERR_UNSUPPORTED


def test_scan_empty_sizes_are_noops(b):
    # nothing is dereferenced or launched when there is no work
    for dims in [(0, 16, 8, 16), (2, 0, 8, 16), (2, 16, 0, 16)]:
        assert _scan(b, dims, ptrs=dict(u=None, delta=None, A=None, B=None, C=None, out=None)) == b.SSM_OK


def test_state_update_argument_validation(b):
    f = b.lib.ssm_selective_state_update
    good = dict(state=0x10000, x=0x20000, dt=0x30000, A=0x40000, B=0x50000, C=0x60000, D=None,
                z=None, out=0x70000)

    def call(dims, io=1, **kw):
        p = dict(good, **kw)
        return f(b.SSMDims(*dims), io, p["state"], p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"],
                 p["z"], p["out"], None)

    assert call((4, 0, 8, 16), io=5) == b.SSM_ERR_INVALID_ARG
    assert call((4, 0, 8, 99)) == b.SSM_ERR_UNSUPPORTED
    assert call((4, 0, -8, 16)) == b.SSM_ERR_INVALID_ARG
    assert call((4, 0, 8, 16), state=None) == b.SSM_ERR_INVALID_ARG
    assert call((4, 0, 8, 16), state=0x10002) == b.SSM_ERR_INVALID_ARG
    assert call((0, 0, 8, 16), state=None, x=None) == b.SSM_OK


def test_python_binding_rejects_bad_tensors(b):
    import torch
    u = torch.zeros(1, 4, 8)
    A = torch.zeros(8, 16)
    with pytest.raises(TypeError):
        b.selective_scan_fwd(u.double(), u.double(), A, torch.zeros(1, 4, 16), torch.zeros(1, 4, 16))
    with pytest.raises(ValueError):
        b.selective_scan_fwd(u, u[:, :2], A, torch.zeros(1, 4, 16), torch.zeros(1, 4, 16))


def _bwd(b, dims, io=1, opts=None, softplus=1, **kw):
    # inputs u, delta, A, B, C, D, z, bias; h0, dout; outputs du, ddelta, dz,
    # dA, dB, dC, dD, ddelta_bias, dh0 -- distinct fake, 256-byte aligned addresses
    names = ["u", "delta", "A", "B", "C", "D", "z", "bias", "h0", "dout", "du", "ddelta", "dz",
             "dA", "dB", "dC", "dD", "dbias", "dh0"]
    p = {n: 0x100000 * (i + 1) for i, n in enumerate(names)}
    for n in ("D", "z", "bias", "h0", "dz", "dD", "dbias", "dh0"):
        p[n] = None
    p.update(kw)
    args = [b.SSMDims(*dims), io] + [p[n] for n in names[:8]] + [softplus] + [p[n] for n in names[8:]]
    if opts is None:
        return b.lib.ssm_selective_scan_bwd(*args, None)
    return b.lib.ssm_selective_scan_bwd_ex(*args, ctypes.byref(opts), None)


def test_bwd_argument_validation(b):
    ok = (2, 16, 64, 16)
    assert _bwd(b, ok, io=3) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, (2, 16, 64, 65)) == b.SSM_ERR_UNSUPPORTED
    assert _bwd(b, (2, -16, 64, 16)) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, softplus=5) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, dout=None) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, dB=None) == b.SSM_ERR_INVALID_ARG
    # dz exactly when z, dD exactly when D
    assert _bwd(b, ok, z=0x7000000) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, dz=0x7000000) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, D=0x7000000) == b.SSM_ERR_INVALID_ARG
    assert b"dD" in b.lib.ssm_last_error()
    assert _bwd(b, ok, du=0x7000001) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, dA=0x7000002) == b.SSM_ERR_INVALID_ARG
    assert b"aligned" in b.lib.ssm_last_error()
    # options: only the kernel family may be set; ZOH has no backward
    assert _bwd(b, ok, opts=b.SSMScanOpts(1)) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, opts=b.SSMScanOpts(0, 0, 0, 9)) == b.SSM_ERR_INVALID_ARG
    assert _bwd(b, ok, opts=b.SSMScanOpts(0, 0, 0, 0, 0, 1)) == b.SSM_ERR_UNSUPPORTED
    # the staged family on rows that are not 16-byte multiples, or N > 16
    assert _bwd(b, (2, 16, 37, 16), opts=b.SSMScanOpts(0, 0, 0, 2)) == b.SSM_ERR_UNSUPPORTED
    assert _bwd(b, (2, 16, 64, 32), opts=b.SSMScanOpts(0, 0, 0, 2)) == b.SSM_ERR_UNSUPPORTED
    assert b"staged backward" in b.lib.ssm_last_error()


def test_bwd_empty_sizes_without_outputs_are_noops(b):
    none = dict(u=None, delta=None, A=None, B=None, C=None, dout=None, du=None, ddelta=None,
                dA=None, dB=None, dC=None)
    for dims in [(0, 16, 8, 16), (2, 0, 8, 16), (2, 16, 0, 16)]:
        assert _bwd(b, dims, **none) == b.SSM_OK


def _ssd(b, dims, io=1, ptrs=None, softplus=1):
    # ptrs: x, dt, A, B, C, D, z, dt_bias, out, state (fake, never dereferenced)
    p = dict(x=0x10000, dt=0x20000, A=0x30000, B=0x40000, C=0x50000, D=None, z=None, bias=None,
             out=0x60000, state=None)
    p.update(ptrs or {})
    return b.lib.ssm_ssd_scan_fwd(b.SSMSsdDims(*dims), io, p["x"], p["dt"], p["A"], p["B"], p["C"], p["D"],
                                  p["z"], p["bias"], softplus, p["out"], p["state"], None)


def test_ssd_argument_validation(b):
    # (batch, seqlen, heads, headdim, groups, dstate)
    ok = (2, 256, 4, 64, 2, 128)
    assert _ssd(b, ok, io=7) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, ok, io=0) == b.SSM_ERR_UNSUPPORTED          # float32: the tensor-core path is bf16
    assert b"bf16" in b.lib.ssm_last_error()
    assert _ssd(b, (2, 256, 4, 32, 2, 128)) == b.SSM_ERR_UNSUPPORTED   # headdim 32
    assert _ssd(b, (2, 256, 4, 64, 2, 96)) == b.SSM_ERR_UNSUPPORTED   # dstate 96
    assert _ssd(b, (2, 256, 4, 64, 3, 128)) == b.SSM_ERR_INVALID_ARG  # heads not a multiple of groups
    assert _ssd(b, (2, 256, 4, 64, 0, 128)) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, (2, -1, 4, 64, 2, 128)) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, ok, softplus=2) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, ok, ptrs=dict(dt=None)) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, ok, ptrs=dict(out=None)) == b.SSM_ERR_INVALID_ARG
    assert _ssd(b, ok, ptrs=dict(dt=0x20001)) == b.SSM_ERR_INVALID_ARG   # dt not aligned to bf16
    assert _ssd(b, ok, ptrs=dict(x=0x10008)) == b.SSM_ERR_UNSUPPORTED    # x not 16-byte aligned (TMA)
    assert _ssd(b, ok, ptrs=dict(z=0x70004)) == b.SSM_ERR_UNSUPPORTED
    # empty problems: nothing to compute, nothing enqueued
    for dims in [(0, 256, 4, 64, 2, 128), (2, 0, 4, 64, 2, 128), (2, 256, 0, 64, 2, 128)]:
        assert _ssd(b, dims, ptrs=dict(x=None, out=None)) == b.SSM_OK


def test_build_info(b):
    info = b.build_info()
    assert 0 <= info["sfu_decays_per_16"] <= 16 and info["sfu_decays_per_16"] % 4 == 0
    p1 = info["split_pass1_sfu_decays_per_16"]
    assert 0 <= p1 <= 16 and p1 % 4 == 0
