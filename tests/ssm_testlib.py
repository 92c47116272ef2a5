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


def check_out(got, ref, io, what="out"):
    e = out_err(got, ref)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    assert e <= TOL_OUT[io], f"{what}: max err {e:.3e} > {TOL_OUT[io]:.0e} (1+|ref|)"
    return e


def check_state(got, ref, io, what="last_state"):
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
    assert e <= TOL_STATE[io], f"{what}: max rel err {e:.3e} > {TOL_STATE[io]:.0e}"
    return e


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
