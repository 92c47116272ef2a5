"""Thin ctypes binding of the C ABI in include/ssm.h.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libssm_b200.so.  torch supplies device memory and the stream.  If
the library is missing this module raises at import; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssm_b200.so")

SSM_OK, SSM_ERR_INVALID_ARG, SSM_ERR_UNSUPPORTED, SSM_ERR_CUDA = 0, 1, 2, 3
SSM_F32, SSM_BF16 = 0, 1
VARIANTS = {"auto": 0, "slab": 1, "split": 2}
FAMILIES = {"auto": 0, "generic": 1, "staged": 2}

# every symbol include/ssm.h declares
EXPORTED = ("ssm_selective_scan_fwd", "ssm_selective_scan_fwd_ex", "ssm_selective_scan_fwd_noalloc",
            "ssm_selective_scan_fwd_complex",
            "ssm_selective_scan_bwd", "ssm_selective_scan_bwd_ex", "ssm_selective_state_update",
            "ssm_scan_plan", "ssm_get_device_status", "ssm_test_inject_decode_wait_timeout",
            "ssm_status_string", "ssm_last_error", "ssm_version", "ssm_get_build_info", "ssm_ssd_scan_fwd",
            "ssm_test_exp2_poly")
NOALLOC_SCRATCH_BYTES = 16 * 1024 * 1024


class SSMDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("dim", ctypes.c_int64), ("dstate", ctypes.c_int64)]


class SSMScanOpts(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("segments", ctypes.c_int32),
                ("lanes", ctypes.c_int32), ("family", ctypes.c_int32),
                ("channels_per_lane", ctypes.c_int32), ("discretization", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 2)]


class SSMScanPlanInfo(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("segments", ctypes.c_int32),
                ("lanes", ctypes.c_int32), ("family", ctypes.c_int32),
                ("launches", ctypes.c_int32), ("channels_per_lane", ctypes.c_int32),
                ("workspace_bytes", ctypes.c_int64)]


class SSMSsdDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("heads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("groups", ctypes.c_int64), ("dstate", ctypes.c_int64)]


class SSMBuildInfo(ctypes.Structure):
    _fields_ = [("sfu_decays_per_16", ctypes.c_int32), ("split_pass1_sfu_decays_per_16", ctypes.c_int32),
                ("reserved", ctypes.c_int32 * 6)]


class SSMError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        super().__init__(f"{_status_str(status)}: {detail}")


_vp = ctypes.c_void_p


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m selective_state_space_36_b200.build` (no CPU fallback exists)")
    lib = ctypes.CDLL(LIB_PATH)
    scan_args = [SSMDims, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_int, _vp, _vp]
    lib.ssm_selective_scan_fwd.argtypes = scan_args + [_vp]
    lib.ssm_selective_scan_fwd.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd_ex.argtypes = scan_args + [ctypes.POINTER(SSMScanOpts), _vp]
    lib.ssm_selective_scan_fwd_ex.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd_noalloc.argtypes = scan_args + [ctypes.c_int, _vp]
    lib.ssm_selective_scan_fwd_noalloc.restype = ctypes.c_int
    lib.ssm_selective_scan_fwd_complex.argtypes = scan_args + [_vp]
    lib.ssm_selective_scan_fwd_complex.restype = ctypes.c_int
    lib.ssm_selective_scan_bwd.argtypes = ([SSMDims, ctypes.c_int] + [_vp] * 8 + [ctypes.c_int] +
                                           [_vp] * 11 + [_vp])
    lib.ssm_selective_scan_bwd.restype = ctypes.c_int
    lib.ssm_selective_scan_bwd_ex.argtypes = ([SSMDims, ctypes.c_int] + [_vp] * 8 + [ctypes.c_int] +
                                              [_vp] * 11 + [ctypes.POINTER(SSMScanOpts), _vp])
    lib.ssm_selective_scan_bwd_ex.restype = ctypes.c_int
    lib.ssm_selective_state_update.argtypes = [SSMDims, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp,
                                               _vp, _vp, _vp, _vp]
    lib.ssm_selective_state_update.restype = ctypes.c_int
    lib.ssm_scan_plan.argtypes = [SSMDims, ctypes.c_int, _vp, _vp, _vp, _vp, _vp, _vp,
                                  ctypes.POINTER(SSMScanOpts), ctypes.POINTER(SSMScanPlanInfo)]
    lib.ssm_scan_plan.restype = ctypes.c_int
    lib.ssm_get_device_status.argtypes = [_vp, ctypes.POINTER(ctypes.c_uint32)]
    lib.ssm_get_device_status.restype = ctypes.c_int
    lib.ssm_test_inject_decode_wait_timeout.argtypes = [ctypes.c_int32]
    lib.ssm_test_inject_decode_wait_timeout.restype = None
    lib.ssm_status_string.argtypes = [ctypes.c_int]
    lib.ssm_status_string.restype = ctypes.c_char_p
    lib.ssm_last_error.argtypes = []
    lib.ssm_last_error.restype = ctypes.c_char_p
    lib.ssm_version.argtypes = []
    lib.ssm_version.restype = ctypes.c_int
    lib.ssm_get_build_info.argtypes = [ctypes.POINTER(SSMBuildInfo)]
    lib.ssm_get_build_info.restype = None
    lib.ssm_ssd_scan_fwd.argtypes = [SSMSsdDims, ctypes.c_int] + [_vp] * 8 + [ctypes.c_int, _vp, _vp, _vp]
    lib.ssm_ssd_scan_fwd.restype = ctypes.c_int
    lib.ssm_test_exp2_poly.argtypes = [_vp, _vp, _vp, ctypes.c_int64, _vp]
    lib.ssm_test_exp2_poly.restype = ctypes.c_int
    return lib


lib = _load()


def _status_str(s: int) -> str:
    return lib.ssm_status_string(s).decode()


def check(status: int) -> None:
    if status != SSM_OK:
        raise SSMError(status, lib.ssm_last_error().decode())


def _io_of(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSM_F32
    if t.dtype == torch.bfloat16:
        return SSM_BF16
    raise TypeError(f"unsupported I/O dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, shape=None, device=None) -> Optional[int]:
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() else None


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def selective_scan_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                       out=None, last_state=None, variant: str = "auto", segments: int = 0,
                       lanes: int = 0, family: str = "auto", cpl: int = 0, zoh_b: bool = False,
                       stream=None):
    """Selective scan forward on CUDA tensors; returns ``out``.

    u, delta, z: (batch, seqlen, dim); B, C: (batch, seqlen, dstate) -- all
    float32 or all bfloat16.  A (dim, dstate), D and delta_bias (dim,) float32.
    last_state (batch, dim, dstate) float32 is read as h_0 and overwritten with
    h_L.  ``variant``/``segments``/``lanes``/``family``/``cpl`` force an
    execution choice (sequence split, lanes per channel, generic or staged
    kernel, channels per lane); ``zoh_b`` selects the exact zero-order hold
    for B instead of the Euler form.
    """
    io = _io_of(u)
    batch, seqlen, dim = u.shape
    dstate = A.shape[1]
    dev = u.device
    if out is None:
        out = torch.empty_like(u)
    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate)
    args = [
        _ptr(u, "u", u.dtype, seq, dev), _ptr(delta, "delta", u.dtype, seq, dev),
        _ptr(A, "A", torch.float32, (dim, dstate), dev), _ptr(B, "B", u.dtype, bc, dev),
        _ptr(C, "C", u.dtype, bc, dev), _ptr(D, "D", torch.float32, (dim,), dev),
        _ptr(z, "z", u.dtype, seq, dev), _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev),
        int(bool(delta_softplus)), _ptr(out, "out", u.dtype, seq, dev),
        _ptr(last_state, "last_state", torch.float32, (batch, dim, dstate), dev),
    ]
    dims = SSMDims(batch, seqlen, dim, dstate)
    if variant == "auto" and not segments and not lanes and family == "auto" and not cpl and not zoh_b:
        check(lib.ssm_selective_scan_fwd(dims, io, *args, _stream_handle(stream)))
    else:
        opts = SSMScanOpts(VARIANTS[variant], int(segments), int(lanes), FAMILIES[family], int(cpl),
                           int(bool(zoh_b)))
        check(lib.ssm_selective_scan_fwd_ex(dims, io, *args, ctypes.byref(opts), _stream_handle(stream)))
    return out


def _pairs(t, name):
    """A complex tensor as its (re, im) float view; real tensors pass through."""
    if t is not None and torch.is_complex(t):
        return torch.view_as_real(t.contiguous())
    return t


def selective_scan_fwd_complex(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                               out=None, last_state=None, stream=None):
    """Selective scan with complex A, B, C; returns ``out`` (real).

    A (dim, dstate) complex64 or (dim, dstate, 2) float32; B, C (batch,
    seqlen, dstate) complex64 or (batch, seqlen, dstate, 2) in the dtype of u;
    last_state (batch, dim, dstate, 2) float32 (or a complex64 tensor, whose
    storage is updated in place) read as h_0 and overwritten with h_L.
    """
    io = _io_of(u)
    batch, seqlen, dim = u.shape
    A, B, C = _pairs(A, "A"), _pairs(B, "B"), _pairs(C, "C")
    if last_state is not None and torch.is_complex(last_state):
        if not last_state.is_contiguous():
            raise ValueError("last_state must be contiguous")
        last_state = torch.view_as_real(last_state)
    dstate = A.shape[1]
    dev = u.device
    if out is None:
        out = torch.empty_like(u)
    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate, 2)
    args = [
        _ptr(u, "u", u.dtype, seq, dev), _ptr(delta, "delta", u.dtype, seq, dev),
        _ptr(A, "A", torch.float32, (dim, dstate, 2), dev), _ptr(B, "B", u.dtype, bc, dev),
        _ptr(C, "C", u.dtype, bc, dev), _ptr(D, "D", torch.float32, (dim,), dev),
        _ptr(z, "z", u.dtype, seq, dev), _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev),
        int(bool(delta_softplus)), _ptr(out, "out", u.dtype, seq, dev),
        _ptr(last_state, "last_state", torch.float32, (batch, dim, dstate, 2), dev),
    ]
    check(lib.ssm_selective_scan_fwd_complex(SSMDims(batch, seqlen, dim, dstate), io, *args,
                                             _stream_handle(stream)))
    return out


def selective_scan_bwd(u, delta, A, B, C, dout, D=None, z=None, delta_bias=None,
                       delta_softplus=True, h0=None, want_dh0=False, family: str = "auto",
                       stream=None):
    """Gradients of sum(dout * out) of one forward scan (Euler Bbar).

    Arguments as for ``selective_scan_fwd``; ``h0`` (batch, dim, dstate)
    float32 is the state that forward pass started from (None: zero).  Returns
    a dict: du, ddelta, dz (io dtype, dz None without z); dA (dim, dstate), dB,
    dC (batch, seqlen, dstate), dD (None without D), ddelta_bias (None without
    delta_bias) float32; dh0 (batch, dim, dstate) float32 if ``want_dh0`` (or
    h0 is given), else None.  ``family`` forces the generic or the staged
    kernels.
    """
    io = _io_of(u)
    batch, seqlen, dim = u.shape
    dstate = A.shape[1]
    dev = u.device
    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate)
    f32 = dict(dtype=torch.float32, device=dev)
    g = {"du": torch.empty_like(u), "ddelta": torch.empty_like(u),
         "dz": torch.empty_like(u) if z is not None else None,
         "dA": torch.empty((dim, dstate), **f32), "dB": torch.empty(bc, **f32),
         "dC": torch.empty(bc, **f32),
         "dD": torch.empty((dim,), **f32) if D is not None else None,
         "ddelta_bias": torch.empty((dim,), **f32) if delta_bias is not None else None,
         "dh0": torch.empty((batch, dim, dstate), **f32) if (want_dh0 or h0 is not None) else None}
    args = [
        _ptr(u, "u", u.dtype, seq, dev), _ptr(delta, "delta", u.dtype, seq, dev),
        _ptr(A, "A", torch.float32, (dim, dstate), dev), _ptr(B, "B", u.dtype, bc, dev),
        _ptr(C, "C", u.dtype, bc, dev), _ptr(D, "D", torch.float32, (dim,), dev),
        _ptr(z, "z", u.dtype, seq, dev), _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev),
        int(bool(delta_softplus)),
        _ptr(h0, "h0", torch.float32, (batch, dim, dstate), dev), _ptr(dout, "dout", u.dtype, seq, dev),
    ] + [_ptr(g[k], k) for k in ("du", "ddelta", "dz", "dA", "dB", "dC", "dD", "ddelta_bias", "dh0")]
    dims = SSMDims(batch, seqlen, dim, dstate)
    if family == "auto":
        check(lib.ssm_selective_scan_bwd(dims, io, *args, _stream_handle(stream)))
    else:
        opts = SSMScanOpts(0, 0, 0, FAMILIES[family])
        check(lib.ssm_selective_scan_bwd_ex(dims, io, *args, ctypes.byref(opts), _stream_handle(stream)))
    return g


def selective_scan_fwd_noalloc(u, delta, A, B, C, D=None, z=None, delta_bias=None,
                               delta_softplus=True, out=None, last_state=None, segments: int = 0,
                               stream=None):
    """The sequence-split scan without device allocation (carries live in the
    library's static scratch; see ssm_selective_scan_fwd_noalloc in ssm.h).
    ``out`` must be given by callers that cannot allocate (torch.empty_like
    is used otherwise)."""
    io = _io_of(u)
    batch, seqlen, dim = u.shape
    dstate = A.shape[1]
    dev = u.device
    if out is None:
        out = torch.empty_like(u)
    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate)
    check(lib.ssm_selective_scan_fwd_noalloc(
        SSMDims(batch, seqlen, dim, dstate), io,
        _ptr(u, "u", u.dtype, seq, dev), _ptr(delta, "delta", u.dtype, seq, dev),
        _ptr(A, "A", torch.float32, (dim, dstate), dev), _ptr(B, "B", u.dtype, bc, dev),
        _ptr(C, "C", u.dtype, bc, dev), _ptr(D, "D", torch.float32, (dim,), dev),
        _ptr(z, "z", u.dtype, seq, dev), _ptr(delta_bias, "delta_bias", torch.float32, (dim,), dev),
        int(bool(delta_softplus)), _ptr(out, "out", u.dtype, seq, dev),
        _ptr(last_state, "last_state", torch.float32, (batch, dim, dstate), dev),
        int(segments), _stream_handle(stream)))
    return out


def ssd_scan_fwd(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, out=None, last_state=None,
                 stream=None):
    """Mamba-2 SSD layer on CUDA bf16 tensors; returns ``out``.

    x, z: (batch, seqlen, heads, headdim); dt: (batch, seqlen, heads);
    B, C: (batch, seqlen, groups, dstate); A, D, dt_bias: (heads,) float32;
    last_state (batch, heads, headdim, dstate) float32 is read as H_0 and
    overwritten with H_L."""
    batch, seqlen, heads, headdim = x.shape
    groups, dstate = B.shape[2], B.shape[3]
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    seq, bc = (batch, seqlen, heads, headdim), (batch, seqlen, groups, dstate)
    check(lib.ssm_ssd_scan_fwd(
        SSMSsdDims(batch, seqlen, heads, headdim, groups, dstate), _io_of(x),
        _ptr(x, "x", x.dtype, seq, dev), _ptr(dt, "dt", x.dtype, (batch, seqlen, heads), dev),
        _ptr(A, "A", torch.float32, (heads,), dev), _ptr(B, "B", x.dtype, bc, dev), _ptr(C, "C", x.dtype, bc, dev),
        _ptr(D, "D", torch.float32, (heads,), dev), _ptr(z, "z", x.dtype, seq, dev),
        _ptr(dt_bias, "dt_bias", torch.float32, (heads,), dev), int(bool(dt_softplus)),
        _ptr(out, "out", x.dtype, seq, dev),
        _ptr(last_state, "last_state", torch.float32, (batch, heads, headdim, dstate), dev),
        _stream_handle(stream)))
    return out


def test_exp2_poly(x: torch.Tensor, stream=None):
    """(FMA-pipe exp2, SFU ex2.approx) of the float32 CUDA tensor x."""
    x = x.contiguous()
    poly, sfu = torch.empty_like(x), torch.empty_like(x)
    dev = x.device
    check(lib.ssm_test_exp2_poly(_ptr(x, "x", torch.float32, None, dev), _ptr(poly, "poly", torch.float32, None, dev),
                                 _ptr(sfu, "sfu", torch.float32, None, dev), x.numel(), _stream_handle(stream)))
    return poly, sfu


def build_info() -> dict:
    """Build parameters of the loaded library (ssm_get_build_info)."""
    info = SSMBuildInfo()
    lib.ssm_get_build_info(ctypes.byref(info))
    return {"sfu_decays_per_16": int(info.sfu_decays_per_16),
            "split_pass1_sfu_decays_per_16": int(info.split_pass1_sfu_decays_per_16)}


def scan_plan(batch: int, seqlen: int, dim: int, dstate: int, io: str = "bf16",
              variant: str = "auto", segments: int = 0, lanes: int = 0, family: str = "auto",
              cpl: int = 0, aligned: bool = True) -> dict:
    """What ssm_selective_scan_fwd would do for this shape (no GPU work).
    ``aligned`` describes the data pointers (16-byte aligned or not)."""
    base = 0x100000 if aligned else 0x100002
    opts = SSMScanOpts(VARIANTS[variant], int(segments), int(lanes), FAMILIES[family], int(cpl))
    info = SSMScanPlanInfo()
    check(lib.ssm_scan_plan(SSMDims(batch, seqlen, dim, dstate), SSM_BF16 if io == "bf16" else SSM_F32,
                            base, base, base, base, base, base, ctypes.byref(opts), ctypes.byref(info)))
    inv_v = {v: k for k, v in VARIANTS.items()}
    inv_f = {v: k for k, v in FAMILIES.items()}
    return {"variant": inv_v.get(info.variant, "none"), "segments": info.segments, "lanes": info.lanes,
            "family": inv_f.get(info.family, "none"), "launches": info.launches,
            "channels_per_lane": info.channels_per_lane,
            "workspace_bytes": info.workspace_bytes}


def device_status(stream=None) -> int:
    """Synchronises ``stream`` and returns (and clears) the device status word:
    bit 0 = a bounded wait in the decode kernel gave up."""
    v = ctypes.c_uint32(0)
    check(lib.ssm_get_device_status(_stream_handle(stream), ctypes.byref(v)))
    return int(v.value)


def selective_state_update(state, x, dt, A, B, C, D=None, z=None, out=None, stream=None):
    """One decode step on CUDA tensors; ``state`` is updated in place; returns ``out``.

    state (batch, dim, dstate) float32; x, dt, z (batch, dim) and B, C
    (batch, dstate) float32 or bfloat16; A (dim, dstate), D (dim,) float32.
    """
    io = _io_of(x)
    batch, dim = x.shape
    dstate = A.shape[1]
    dev = x.device
    if out is None:
        out = torch.empty_like(x)
    bd, bn = (batch, dim), (batch, dstate)
    check(lib.ssm_selective_state_update(
        SSMDims(batch, 0, dim, dstate), io,
        _ptr(state, "state", torch.float32, (batch, dim, dstate), dev),
        _ptr(x, "x", x.dtype, bd, dev), _ptr(dt, "dt", x.dtype, bd, dev),
        _ptr(A, "A", torch.float32, (dim, dstate), dev), _ptr(B, "B", x.dtype, bn, dev),
        _ptr(C, "C", x.dtype, bn, dev), _ptr(D, "D", torch.float32, (dim,), dev),
        _ptr(z, "z", x.dtype, bd, dev), _ptr(out, "out", x.dtype, bd, dev), _stream_handle(stream)))
    return out
