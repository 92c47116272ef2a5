"""Helpers shared by the GPU parity tests: device upload of generator arrays,
oracle runs on exact fp64 copies, and the tolerance checks.

Tolerances (stated with the target):
  fp32 I/O: |out - ref| <= 1e-5 (1 + |ref|) elementwise; the same form for
            the returned state.
  bf16 I/O: |out - ref| <= 2e-2 (1 + |ref|); the state "within 1e-3 relative",
            read as the relative error of each channel's state vector:
            max_n |h - h_ref| <= 1e-3 max_n |h_ref| for every (b, d).  An
            elementwise relative error is ill-conditioned where a state entry
            happens to cross zero: fp32 rounding alone leaves ~1e-6 rms of
            absolute error there.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from selective_state_space_36_b200 import inputs as I

TOL_OUT = {"f32": 1e-5, "bf16": 2e-2}
TOL_STATE = {"f32": 1e-5, "bf16": 1e-3}


def to_dev(arr, io: str, device="cuda"):
    if arr is None:
        return None
    if arr.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)


def from_dev(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def f64(arr, io):
    return I.to_f64(arr, io)


def out_err(got, ref) -> float:
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    return float(np.max(np.abs(got - ref) / (1.0 + np.abs(ref))))


def check_out(got, ref, io, what="out", tol=None):
    tol = TOL_OUT[io] if tol is None else tol
    e = out_err(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= tol, f"{what}: max err {e:.3e} > {tol:.1e} (1+|ref|)"
    return e


def check_state(got, ref, io, what="last_state", tol=None):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    if io == "f32":
        e = float(np.max(np.abs(got - ref) / (1.0 + np.abs(ref))))
    else:
        # per-channel (last axis = states) norm-wise relative error
        num = np.max(np.abs(got - ref), axis=-1)
        den = np.max(np.abs(ref), axis=-1) + 1e-30
        e = float(np.max(num / den))
    tol = TOL_STATE[io] if tol is None else tol
    assert e <= tol, f"{what}: max rel err {e:.3e} > {tol:.1e}"
    return e


def state_err_elementwise(got, ref) -> float:
    """The elementwise relative state error with an fp32-noise floor:
    max |h - h_ref| / (|h_ref| + 1e-3 rms(h_ref)) over all entries.  Reported
    beside the norm-wise figure that check_state bounds: entries that cross
    zero carry only fp32 rounding (~1e-6 rms), which the floor absorbs."""
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    floor = 1e-3 * float(np.sqrt(np.mean(ref ** 2))) + 1e-30
    return float(np.max(np.abs(got - ref) / (np.abs(ref) + floor)))


def oracle_scan(x: dict, io: str, nthreads: int = 0, zoh_b: bool = False):
    """Oracle on the exact fp64 values of a scan_inputs() dictionary."""
    return oracle.scan(f64(x["u"], io), f64(x["delta"], io), f64(x["A"], "f32"), f64(x["B"], io),
                       f64(x["C"], io), D=f64(x["D"], "f32"), z=f64(x["z"], io),
                       delta_bias=f64(x["delta_bias"], "f32"), delta_softplus=x["delta_softplus"],
                       h0=f64(x["h0"], "f32"), nthreads=nthreads, zoh_b=zoh_b)


def gpu_scan(x: dict, io: str, with_state=True, **kw):
    """Library scan on device copies of a scan_inputs() dictionary."""
    from selective_state_space_36_b200 import binding
    d = {k: to_dev(v, io) for k, v in x.items() if isinstance(v, np.ndarray)}
    state = None
    if with_state:
        u = x["u"]
        state = (d["h0"].clone() if x.get("h0") is not None
                 else torch.zeros((u.shape[0], u.shape[2], x["A"].shape[1]), dtype=torch.float32, device="cuda"))
    out = binding.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d.get("D"),
                                     z=d.get("z"), delta_bias=d.get("delta_bias"),
                                     delta_softplus=x["delta_softplus"], last_state=state, **kw)
    torch.cuda.synchronize()
    return out, state


def channel_subset(x: dict, dims_idx, batch_idx=None) -> dict:
    """The scan inputs restricted to channels dims_idx of batch rows batch_idx.
    Channels are independent, so the oracle on the subset equals the oracle's
    values for those channels of the full problem."""
    bi = slice(None) if batch_idx is None else np.asarray(batch_idx)
    di = np.asarray(dims_idx)
    sub = {}
    for k, v in x.items():
        if not isinstance(v, np.ndarray):
            sub[k] = v
        elif k in ("u", "delta", "z"):
            sub[k] = v[bi][:, :, di]
        elif k in ("B", "C"):
            sub[k] = v[bi]
        elif k == "A":
            sub[k] = v[di]
        elif k in ("D", "delta_bias"):
            sub[k] = v[di]
        elif k == "h0":
            sub[k] = v[bi][:, di]
        else:
            sub[k] = v
    return sub


# ------------------------------------------------------------------ backward
# Gradients are compared row by row (rows = every index but the last axis)
# with a norm-wise bound, max_j |g - g_ref| <= tol * max_j |g_ref|, for the
# same reason as the bf16 state: single entries of a gradient cross zero.
# The bounds (derivation with the backward kernel's description):
#   io outputs du, ddelta, dz: bf16 rounding of the result (2^-9 relative)
#   dominates, so 1e-2 for bf16; float32 sums (dA, dB, dC, dD, ddelta_bias,
#   dh0) and every fp32-I/O output carry only fp32 arithmetic, whose error in
#   the adjoint grows at most linearly with the decay's memory 1/(Delta |A|)
#   (<= ~1e3 steps at these inputs, i.e. <= ~6e-5 relative): 1e-4.
TOL_GRAD = {"io": {"f32": 1e-4, "bf16": 1e-2}, "f32": {"f32": 1e-4, "bf16": 1e-4}}
GRAD_IO = ("du", "ddelta", "dz")
GRAD_F32 = ("dA", "dB", "dC", "dD", "ddelta_bias", "dh0")


def grad_err(got, ref) -> float:
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    if got.size == 0:
        return 0.0
    g2 = got.reshape(-1, got.shape[-1]) if got.ndim > 1 else got.reshape(1, -1)
    r2 = ref.reshape(-1, ref.shape[-1]) if ref.ndim > 1 else ref.reshape(1, -1)
    floor = 1e-6 * float(np.max(np.abs(r2))) + 1e-30
    num = np.max(np.abs(g2 - r2), axis=1)
    den = np.max(np.abs(r2), axis=1) + floor
    return float(np.max(num / den))


def grad_keys(x: dict):
    """The gradients a call with these inputs returns (dh0 requested)."""
    ks = ["du", "ddelta", "dA", "dB", "dC", "dh0"]
    ks += ["dz"] if x.get("z") is not None else []
    ks += ["dD"] if x.get("D") is not None else []
    ks += ["ddelta_bias"] if x.get("delta_bias") is not None else []
    return ks


def check_grads(got: dict, ref: dict, io: str, keys) -> dict:
    errs = {}
    for k in keys:
        assert got.get(k) is not None, f"{k}: not returned"
        g = from_dev(got[k])
        assert g.shape == ref[k].shape, f"{k}: shape {g.shape} != {ref[k].shape}"
        assert np.all(np.isfinite(g)), f"{k}: non-finite values"
        tol = TOL_GRAD["io" if k in GRAD_IO else "f32"][io]
        e = grad_err(g, ref[k])
        assert e <= tol, f"{k}: max row-wise rel err {e:.3e} > {tol:.0e}"
        errs[k] = e
    return errs


def oracle_bwd(x: dict, io: str, dout):
    """Oracle gradients on the exact fp64 values of scan_inputs() + dout."""
    return oracle.scan_bwd(f64(x["u"], io), f64(x["delta"], io), f64(x["A"], "f32"), f64(x["B"], io),
                           f64(x["C"], io), f64(dout, io), D=f64(x["D"], "f32"), z=f64(x["z"], io),
                           delta_bias=f64(x["delta_bias"], "f32"), delta_softplus=x["delta_softplus"],
                           h0=f64(x["h0"], "f32"))


def gpu_bwd(x: dict, io: str, dout, want_dh0=True, family="auto"):
    """Library backward on device copies of scan_inputs() + dout."""
    from selective_state_space_36_b200 import binding
    d = {k: to_dev(v, io) for k, v in x.items() if isinstance(v, np.ndarray)}
    g = binding.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], to_dev(dout, io),
                                   D=d.get("D"), z=d.get("z"), delta_bias=d.get("delta_bias"),
                                   delta_softplus=x["delta_softplus"], h0=d.get("h0"),
                                   want_dh0=want_dh0, family=family)
    torch.cuda.synchronize()
    return g
