"""fp64 CPU oracle of the selective SSM scan and decode step.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The library code under
``selective_state_space_36_b200`` never imports this package, and this package
imports nothing from it.

The arithmetic lives in ``ssm_oracle.c`` (plain C, double precision, one
sequential loop per channel); this module compiles it with gcc on first use
and marshals numpy arrays.  Every function takes and returns float64 arrays;
inputs held as bf16 bits or float32 must be widened exactly first (see
``selective_state_space_36_b200.inputs.to_f64``).

Parity status of each function (what pins it lives in tests/test_oracle_pins.py):
  scan(..., zoh_b=False)  pinned: brute-force unrolled sum, N=1 closed form,
                          LTI convolution, Delta -> 0, split/resume, softplus
                          and bias placement, skip and gate special cases.
  scan(..., zoh_b=True)   pinned: brute force (ZOH form), Theorem 1.
  state_update            pinned: 1000 decode steps == scan over 1000 steps,
                          one-step brute force.
  scan_bwd                pinned: central finite differences of scan (every
                          input), torch autograd of an independent fp64 loop.
  scan_complex            pinned: bit-identical to scan when every imaginary
                          part is zero, brute-force complex unrolled sum, LTI
                          convolution with a complex kernel, pure-rotation
                          closed form (sign of the phase).
  ssd_scan                pinned: equal to scan with A[d, :] = A_head and the
                          head's Delta for every channel of the head; the
                          quadratic (masked attention) form; the chunked block
                          decomposition at several chunk lengths; Delta -> 0;
                          split/resume.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssm_oracle.c")
_LIB = os.path.join(_HERE, "libssm_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ssm_oracle.c into libssm_oracle.so (gcc, -O2, IEEE semantics)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                               "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _LIB)
    return _LIB


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_selective_scan.restype = ctypes.c_int
    lib.oracle_selective_scan.argtypes = [_i64, _i64, _i64, _i64,
                                          _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
                                          ctypes.c_int, ctypes.c_int, _dp, _dp, ctypes.c_int]
    lib.oracle_state_update.restype = ctypes.c_int
    lib.oracle_state_update.argtypes = [_i64, _i64, _i64, _dp, _dp, _dp, _dp,
                                        _dp, _dp, _dp, _dp, _dp]
    lib.oracle_default_threads.restype = ctypes.c_int
    lib.oracle_default_threads.argtypes = []
    lib.oracle_selective_scan_complex.restype = ctypes.c_int
    lib.oracle_selective_scan_complex.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 8 + [ctypes.c_int, _dp, _dp]
    lib.oracle_selective_scan_bwd.restype = ctypes.c_int
    lib.oracle_selective_scan_bwd.argtypes = [_i64, _i64, _i64, _i64] + [_dp] * 8 + [ctypes.c_int] + [_dp] * 11
    lib.oracle_ssd_scan.restype = ctypes.c_int
    lib.oracle_ssd_scan.argtypes = [_i64] * 6 + [_dp] * 8 + [ctypes.c_int, _dp, _dp]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = _bind(_LIB)
    return _lib


def default_threads() -> int:
    """Threads the oracle uses when ``nthreads`` is 0."""
    return int(_load().oracle_default_threads())


def _c64(a: Optional[np.ndarray], shape: Tuple[int, ...], name: str):
    if a is None:
        return None, None
    arr = np.ascontiguousarray(a, dtype=np.float64)
    if arr.shape != shape:
        raise ValueError(f"{name}: expected shape {shape}, got {arr.shape}")
    return arr, arr.ctypes.data_as(_dp)


def scan(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
         h0=None, zoh_b: bool = False, nthreads: int = 0, _lib_handle=None):
    """Selective scan in fp64.

    u, delta, z: (batch, seqlen, dim); B, C: (batch, seqlen, dstate);
    A: (dim, dstate); D, delta_bias: (dim,); h0: (batch, dim, dstate) or None.
    Returns (out (batch, seqlen, dim), last_state (batch, dim, dstate)).
    """
    u = np.asarray(u)
    batch, seqlen, dim = u.shape
    dstate = np.asarray(A).shape[1]
    keep = []

    def p(a, shape, name):
        arr, ptr = _c64(a, shape, name)
        keep.append(arr)
        return ptr

    pu = p(u, (batch, seqlen, dim), "u")
    pd = p(delta, (batch, seqlen, dim), "delta")
    pA = p(A, (dim, dstate), "A")
    pB = p(B, (batch, seqlen, dstate), "B")
    pC = p(C, (batch, seqlen, dstate), "C")
    pD = p(D, (dim,), "D")
    pz = p(z, (batch, seqlen, dim), "z")
    pb = p(delta_bias, (dim,), "delta_bias")
    out = np.zeros((batch, seqlen, dim), dtype=np.float64)
    state = (np.zeros((batch, dim, dstate), dtype=np.float64) if h0 is None
             else np.array(h0, dtype=np.float64, order="C", copy=True).reshape(batch, dim, dstate))
    rc = (_lib_handle or _load()).oracle_selective_scan(batch, seqlen, dim, dstate, pu, pd, pA, pB, pC, pD, pz, pb,
                                       int(bool(delta_softplus)), int(bool(zoh_b)),
                                       out.ctypes.data_as(_dp), state.ctypes.data_as(_dp),
                                       int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_selective_scan failed with code {rc}")
    return out, state


def _pairs(a, shape, name):
    """A complex array as a contiguous float64 (..., 2) array of (re, im)."""
    if a is None:
        return None
    c = np.ascontiguousarray(a, dtype=np.complex128)
    if c.shape != shape:
        raise ValueError(f"{name}: expected shape {shape}, got {c.shape}")
    return c.view(np.float64).reshape(shape + (2,))


def scan_complex(u, delta, A, B, C, D=None, z=None, delta_bias=None, delta_softplus=True,
                 h0=None, _lib_handle=None):
    """Selective scan with complex A, B, C in fp64 (real u, delta, z, D, bias).

    A: (dim, dstate) complex; B, C: (batch, seqlen, dstate) complex; h0:
    (batch, dim, dstate) complex or None.  y_t = Re(sum_n C_t,n h_t,n) + D u_t.
    Returns (out (batch, seqlen, dim) real, last_state (batch, dim, dstate) complex).
    """
    u = np.asarray(u)
    batch, seqlen, dim = u.shape
    dstate = np.asarray(A).shape[1]
    keep = []

    def p(a, shape, name):
        arr, ptr = _c64(a, shape, name)
        keep.append(arr)
        return ptr

    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate)
    Ap, Bp, Cp = _pairs(A, (dim, dstate), "A"), _pairs(B, bc, "B"), _pairs(C, bc, "C")
    ins = [p(u, seq, "u"), p(delta, seq, "delta"), p(Ap, (dim, dstate, 2), "A"), p(Bp, bc + (2,), "B"),
           p(Cp, bc + (2,), "C"), p(D, (dim,), "D"), p(z, seq, "z"), p(delta_bias, (dim,), "delta_bias")]
    out = np.zeros(seq, dtype=np.float64)
    st = np.zeros((batch, dim, dstate), dtype=np.complex128) if h0 is None else \
        np.array(h0, dtype=np.complex128, order="C", copy=True).reshape(batch, dim, dstate)
    stp = st.view(np.float64)
    rc = (_lib_handle or _load()).oracle_selective_scan_complex(
        batch, seqlen, dim, dstate, *ins, int(bool(delta_softplus)), out.ctypes.data_as(_dp),
        stp.ctypes.data_as(_dp))
    if rc != 0:
        raise RuntimeError(f"oracle_selective_scan_complex failed with code {rc}")
    return out, st


def scan_bwd(u, delta, A, B, C, dout, D=None, z=None, delta_bias=None, delta_softplus=True,
             h0=None, _lib_handle=None):
    """Gradients of sum(dout * out) of the scan (Euler Bbar) in fp64.

    Returns a dict: du, ddelta, dz (batch, seqlen, dim) [dz None without z],
    dA (dim, dstate), dB, dC (batch, seqlen, dstate), dD, ddelta_bias (dim,),
    dh0 (batch, dim, dstate).
    """
    u = np.asarray(u)
    batch, seqlen, dim = u.shape
    dstate = np.asarray(A).shape[1]
    keep = []

    def p(a, shape, name):
        arr, ptr = _c64(a, shape, name)
        keep.append(arr)
        return ptr

    seq, bc = (batch, seqlen, dim), (batch, seqlen, dstate)
    ins = [p(u, seq, "u"), p(delta, seq, "delta"), p(A, (dim, dstate), "A"), p(B, bc, "B"),
           p(C, bc, "C"), p(D, (dim,), "D"), p(z, seq, "z"), p(delta_bias, (dim,), "delta_bias")]
    ph0 = p(h0, (batch, dim, dstate), "h0")
    pdo = p(dout, seq, "dout")
    out = {"du": np.zeros(seq), "ddelta": np.zeros(seq), "dA": np.zeros((dim, dstate)),
           "dB": np.zeros(bc), "dC": np.zeros(bc), "dD": np.zeros(dim),
           "dz": np.zeros(seq) if z is not None else None, "ddelta_bias": np.zeros(dim),
           "dh0": np.zeros((batch, dim, dstate))}
    ptr = lambda k: out[k].ctypes.data_as(_dp) if out[k] is not None else None
    rc = (_lib_handle or _load()).oracle_selective_scan_bwd(
        batch, seqlen, dim, dstate, *ins, int(bool(delta_softplus)), ph0, pdo,
        ptr("du"), ptr("ddelta"), ptr("dA"), ptr("dB"), ptr("dC"), ptr("dD"), ptr("dz"),
        ptr("ddelta_bias"), ptr("dh0"))
    if rc != 0:
        raise RuntimeError(f"oracle_selective_scan_bwd failed with code {rc}")
    return out


def state_update(state, x, dt, A, B, C, D=None, z=None, _lib_handle=None):
    """One decode step in fp64.  Returns (out (batch, dim), new_state)."""
    st = np.array(state, dtype=np.float64, order="C", copy=True)
    batch, dim, dstate = st.shape
    keep = []

    def p(a, shape, name):
        arr, ptr = _c64(a, shape, name)
        keep.append(arr)
        return ptr

    px = p(x, (batch, dim), "x")
    pdt = p(dt, (batch, dim), "dt")
    pA = p(A, (dim, dstate), "A")
    pB = p(B, (batch, dstate), "B")
    pC = p(C, (batch, dstate), "C")
    pD = p(D, (dim,), "D")
    pz = p(z, (batch, dim), "z")
    out = np.zeros((batch, dim), dtype=np.float64)
    rc = (_lib_handle or _load()).oracle_state_update(batch, dim, dstate, st.ctypes.data_as(_dp), px, pdt, pA,
                                     pB, pC, pD, pz, out.ctypes.data_as(_dp))
    if rc != 0:
        raise RuntimeError(f"oracle_state_update failed with code {rc}")
    return out, st


def ssd_scan(x, dt, A, B, C, D=None, z=None, dt_bias=None, dt_softplus=True, h0=None,
             _lib_handle=None):
    """Mamba-2 SSD layer (linear / recurrent form) in fp64.

    x, z: (batch, seqlen, heads, headdim); dt: (batch, seqlen, heads) (raw);
    A, D, dt_bias: (heads,); B, C: (batch, seqlen, groups, dstate);
    h0: (batch, heads, headdim, dstate) or None.
    Returns (out (batch, seqlen, heads, headdim), last_state (batch, heads, headdim, dstate)).
    """
    x = np.asarray(x)
    batch, seqlen, heads, headdim = x.shape
    groups, dstate = np.asarray(B).shape[2:]
    keep = []

    def p(a, shape, name):
        arr, ptr = _c64(a, shape, name)
        keep.append(arr)
        return ptr

    seq = (batch, seqlen, heads, headdim)
    bc = (batch, seqlen, groups, dstate)
    px, pdt = p(x, seq, "x"), p(dt, (batch, seqlen, heads), "dt")
    pA, pB, pC = p(A, (heads,), "A"), p(B, bc, "B"), p(C, bc, "C")
    pD, pz, pb = p(D, (heads,), "D"), p(z, seq, "z"), p(dt_bias, (heads,), "dt_bias")
    out = np.zeros(seq, dtype=np.float64)
    state = (np.zeros((batch, heads, headdim, dstate), dtype=np.float64) if h0 is None
             else np.array(h0, dtype=np.float64, order="C", copy=True).reshape(batch, heads, headdim, dstate))
    rc = (_lib_handle or _load()).oracle_ssd_scan(batch, seqlen, heads, headdim, groups, dstate, px, pdt, pA,
                                                  pB, pC, pD, pz, pb, int(bool(dt_softplus)),
                                                  out.ctypes.data_as(_dp), state.ctypes.data_as(_dp))
    if rc != 0:
        raise RuntimeError(f"oracle_ssd_scan failed with code {rc}")
    return out, state


class Variant:
    """The same API bound to another build of the oracle source (used by the
    mutation tests, which compile deliberately broken copies)."""

    def __init__(self, path: str):
        self._h = _bind(path)

    def scan(self, *a, **kw):
        return scan(*a, _lib_handle=self._h, **kw)

    def state_update(self, *a, **kw):
        return state_update(*a, _lib_handle=self._h, **kw)

    def scan_bwd(self, *a, **kw):
        return scan_bwd(*a, _lib_handle=self._h, **kw)

    def scan_complex(self, *a, **kw):
        return scan_complex(*a, _lib_handle=self._h, **kw)

    def ssd_scan(self, *a, **kw):
        return ssd_scan(*a, _lib_handle=self._h, **kw)


def compile_variant(source: str, path: str) -> "Variant":
    """Compile C source text (a modified copy of ssm_oracle.c) to ``path``."""
    src = path + ".c"
    with open(src, "w") as f:
        f.write(source)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
                           "-o", path, src, "-lm", "-lpthread"])
    return Variant(path)


def source() -> str:
    with open(_SRC) as f:
        return f.read()
