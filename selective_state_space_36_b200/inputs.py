"""Seeded synthetic inputs for the selective scan and the one-token decode step.

This module is the only code the CUDA path and the fp64 oracle have in common:
it draws random numbers and rounds them to the I/O type.  It holds none of the
scan's arithmetic (no discretisation, recurrence, readout or gate).  Two input
recipes need one elementwise transform each, and both are part of *drawing* an
input rather than of the method:

* the Delta bias is the inverse softplus of a per-channel time step dt0 drawn
  log-uniformly in [1e-3, 1e-1]; it initialises the learned parameter that the
  selection mechanism adds to the input-dependent projection before tau_Delta
  (【論文要約】Mamba: Linear-Time Sequence Modeling with Selective State Spaces,
  "S6" section, Algorithm 2);
* the decode step takes an already-positive Delta, so its recipe draws the raw
  value, adds the bias and applies numpy's ``logaddexp(0, .)`` before rounding
  to bf16.  Both sides then consume the same rounded value.

Layouts (dense, row-major):
  u, delta, z, out : (batch, seqlen, dim)      D contiguous
  B, C             : (batch, seqlen, dstate)   N contiguous
  A                : (dim, dstate) float32
  D, delta_bias    : (dim,) float32
  state / h0       : (batch, dim, dstate) float32

Every sequence tensor is drawn in blocks of ``CHUNK_ROWS`` time steps, each
block from its own PCG64 stream seeded by (seed, tensor, batch row, block).  A
slice [t0, t1) is therefore reproducible without drawing the rest, blocks can
be drawn in parallel, and long sequences can be streamed to the device.
bf16 values are float32 draws rounded to nearest even; the oracle consumes the
rounded values, upcast exactly.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace
from typing import Dict, Iterable, Optional, Tuple

import numpy as np

CHUNK_ROWS = 4096

# stream identifiers: one independent PCG64 family per drawn quantity
_TID = {"param": 0, "u": 1, "delta": 2, "z": 3, "B": 4, "C": 5, "h0": 6,
        "x": 7, "dt": 8, "dB": 9, "dC": 10, "dz": 11, "dout": 12,
        "B_im": 13, "C_im": 14, "h0_im": 15}

SEQ_NAMES = ("u", "delta", "z", "B", "C")


# --------------------------------------------------------------------------
# bf16 <-> float32, round to nearest even (pure bit manipulation)
# --------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + r) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bits (uint16) to float32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def to_f64(arr: Optional[np.ndarray], io: str) -> Optional[np.ndarray]:
    """Exact float64 view of an array held in the I/O representation."""
    if arr is None:
        return None
    if io == "bf16" and arr.dtype == np.uint16:
        return bf16_bits_to_f32(arr).astype(np.float64)
    return np.asarray(arr, dtype=np.float64)


def _round_io(x32: np.ndarray, io: str) -> np.ndarray:
    if io == "bf16":
        return f32_to_bf16_bits(x32)
    if io == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    raise ValueError(f"unknown io type {io!r}")


# --------------------------------------------------------------------------
# configurations
# --------------------------------------------------------------------------
@dataclass(frozen=True)
class ScanConfig:
    """One synthetic selective-scan workload.

    ``d_skip`` is ``"one"`` (D = 1) or ``"uniform"`` (D ~ U(0.5, 1.5));
    ``delta_sigma`` is the standard deviation of the raw Delta draws;
    ``h0_sigma`` (optional) draws an initial state N(0, h0_sigma^2).
    """
    name: str
    batch: int
    seqlen: int
    dim: int
    dstate: int = 16
    io: str = "bf16"
    seed: int = 0
    delta_sigma: float = 0.5
    d_skip: str = "one"
    softplus: bool = True
    has_z: bool = True
    has_d: bool = True
    has_bias: bool = True
    h0_sigma: Optional[float] = None
    dt_min: float = 1e-3
    dt_max: float = 1e-1

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.dim

    def with_(self, **kw) -> "ScanConfig":
        return replace(self, **kw)


@dataclass(frozen=True)
class DecodeConfig:
    """Synthetic workload for repeated one-token decode steps."""
    name: str
    batch: int
    dim: int
    dstate: int = 16
    steps: int = 1000
    io: str = "bf16"
    seed: int = 4
    delta_sigma: float = 0.5
    d_skip: str = "uniform"
    h0_sigma: float = 0.1
    has_z: bool = True
    has_d: bool = True
    dt_min: float = 1e-3
    dt_max: float = 1e-1


# The five workloads the library is specified on (sizes and distributions as
# stated with the target; "N(0, 0.25)" read as variance 0.25, sigma = 0.5).
TINY_F32 = ScanConfig("tiny_f32_b1_l256_d64_n16", 1, 256, 64, 16, io="f32", seed=0,
                      delta_sigma=0.5, d_skip="one")
MAMBA130M = ScanConfig("mamba130m_b8_l2048_d1536_n16", 8, 2048, 1536, 16, io="bf16",
                       seed=1, delta_sigma=0.5, d_skip="one")
MAMBA1P4B = ScanConfig("mamba1p4b_b8_l2048_d4096_n16", 8, 2048, 4096, 16, io="bf16",
                       seed=2, delta_sigma=0.5, d_skip="uniform")
LONGSEQ = ScanConfig("longseq_b1_l1048576_d1536_n16", 1, 1 << 20, 1536, 16, io="bf16",
                     seed=3, delta_sigma=0.5, d_skip="uniform")
DECODE = DecodeConfig("decode_b256_d5120_n16_x1000", 256, 5120, 16, steps=1000,
                      io="bf16", seed=4, delta_sigma=0.5, d_skip="uniform", h0_sigma=0.1)

SCAN_CONFIGS = {c.name: c for c in (TINY_F32, MAMBA130M, MAMBA1P4B, LONGSEQ)}


# --------------------------------------------------------------------------
# per-channel parameters
# --------------------------------------------------------------------------
def channel_params(seed: int, dim: int, dstate: int, d_skip: str,
                   dt_min: float = 1e-3, dt_max: float = 1e-1
                   ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """A (dim, dstate), D (dim,), delta_bias (dim,), all float32.

    A[d, n] = -(n + 1) (a real diagonal initialisation); dt0 log-uniform in
    [dt_min, dt_max]; delta_bias = inverse softplus of dt0, evaluated in
    float64 as dt0 + log(-expm1(-dt0)) and rounded to float32; D is 1 or
    U(0.5, 1.5) depending on ``d_skip``.  Draw order: dt0, then D.
    """
    rng = np.random.default_rng([seed, _TID["param"]])
    A = np.tile(-(np.arange(dstate, dtype=np.float32) + 1.0), (dim, 1)).astype(np.float32)
    dt0 = np.exp(rng.uniform(math.log(dt_min), math.log(dt_max), size=dim))
    bias = (dt0 + np.log(-np.expm1(-dt0))).astype(np.float32)
    if d_skip == "one":
        D = np.ones(dim, dtype=np.float32)
    elif d_skip == "uniform":
        D = rng.uniform(0.5, 1.5, size=dim).astype(np.float32)
    else:
        raise ValueError(d_skip)
    return A, D, bias


# --------------------------------------------------------------------------
# sequence tensors
# --------------------------------------------------------------------------
def _sigma(cfg: ScanConfig, name: str) -> float:
    return cfg.delta_sigma if name == "delta" else 1.0


def _width(cfg: ScanConfig, name: str) -> int:
    return cfg.dstate if name in ("B", "C", "B_im", "C_im") else cfg.dim


def _draw_block(cfg: ScanConfig, name: str, b: int, blk: int) -> np.ndarray:
    rows = min(CHUNK_ROWS, cfg.seqlen - blk * CHUNK_ROWS)
    rng = np.random.default_rng([cfg.seed, _TID[name], b, blk])
    x = rng.standard_normal((rows, _width(cfg, name)), dtype=np.float32)
    s = _sigma(cfg, name)
    if s != 1.0:
        x *= np.float32(s)
    return _round_io(x, cfg.io)


def _io_dtype(io: str):
    return np.uint16 if io == "bf16" else np.float32


def draw_rows(cfg: ScanConfig, name: str, b: int, t0: int, t1: int,
              out: Optional[np.ndarray] = None, threads: int = 0) -> np.ndarray:
    """Rows [t0, t1) of sequence tensor ``name`` for batch row ``b``."""
    w = _width(cfg, name)
    if out is None:
        out = np.empty((t1 - t0, w), dtype=_io_dtype(cfg.io))
    blocks = range(t0 // CHUNK_ROWS, (t1 + CHUNK_ROWS - 1) // CHUNK_ROWS) if t1 > t0 else range(0)

    def fill(blk):
        lo, hi = blk * CHUNK_ROWS, min((blk + 1) * CHUNK_ROWS, cfg.seqlen)
        data = _draw_block(cfg, name, b, blk)
        a, e = max(lo, t0), min(hi, t1)
        out[a - t0:e - t0] = data[a - lo:e - lo]

    nthreads = threads or min(len(blocks), os.cpu_count() or 1)
    if nthreads > 1 and len(blocks) > 1:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(fill, blocks))
    else:
        for blk in blocks:
            fill(blk)
    return out


def draw_tensor(cfg: ScanConfig, name: str, t0: int = 0, t1: Optional[int] = None,
                threads: int = 0) -> np.ndarray:
    """Full (batch, t1 - t0, width) slice of a sequence tensor."""
    t1 = cfg.seqlen if t1 is None else t1
    out = np.empty((cfg.batch, t1 - t0, _width(cfg, name)), dtype=_io_dtype(cfg.io))
    for b in range(cfg.batch):
        draw_rows(cfg, name, b, t0, t1, out=out[b], threads=threads)
    return out


def draw_h0(cfg, batch: int, dim: int, dstate: int, sigma: float) -> np.ndarray:
    """Initial state (batch, dim, dstate) float32 ~ N(0, sigma^2)."""
    out = np.empty((batch, dim, dstate), dtype=np.float32)
    for b in range(batch):
        rng = np.random.default_rng([cfg.seed, _TID["h0"], b])
        out[b] = rng.standard_normal((dim, dstate), dtype=np.float32) * np.float32(sigma)
    return out


def scan_inputs(cfg: ScanConfig, t0: int = 0, t1: Optional[int] = None,
                threads: int = 0) -> Dict[str, Optional[np.ndarray]]:
    """All inputs of one scan over time steps [t0, t1), in I/O representation.

    Keys: u, delta, z, B, C (sequence tensors), A, D, delta_bias (float32),
    h0 (float32 or None), and the flag delta_softplus.
    """
    A, D, bias = channel_params(cfg.seed, cfg.dim, cfg.dstate, cfg.d_skip, cfg.dt_min, cfg.dt_max)
    res: Dict[str, Optional[np.ndarray]] = {
        n: draw_tensor(cfg, n, t0, t1, threads) for n in SEQ_NAMES}
    if not cfg.has_z:
        res["z"] = None
    res["A"] = A
    res["D"] = D if cfg.has_d else None
    res["delta_bias"] = bias if cfg.has_bias else None
    res["h0"] = (draw_h0(cfg, cfg.batch, cfg.dim, cfg.dstate, cfg.h0_sigma)
                 if cfg.h0_sigma is not None else None)
    res["delta_softplus"] = cfg.softplus
    return res


def draw_dout(cfg: ScanConfig, t0: int = 0, t1: Optional[int] = None,
              threads: int = 0) -> np.ndarray:
    """Upstream gradient of the scan output: (batch, t1 - t0, dim) ~ N(0, 1)
    in I/O representation, from its own stream (the loss is sum(dout * out))."""
    return draw_tensor(cfg, "dout", t0, t1, threads)


# --------------------------------------------------------------------------
# complex diagonal A
# --------------------------------------------------------------------------
def complex_A(dim: int, dstate: int) -> np.ndarray:
    """A[d, n] = -1/2 + i pi n for every channel (the S4D-Lin initialisation),
    as float32 (re, im) pairs of shape (dim, dstate, 2)."""
    A = np.empty((dim, dstate, 2), dtype=np.float32)
    A[..., 0] = -0.5
    A[..., 1] = (np.pi * np.arange(dstate, dtype=np.float64)).astype(np.float32)[None, :]
    return A


def _interleave(re: np.ndarray, im: np.ndarray) -> np.ndarray:
    out = np.empty(re.shape + (2,), dtype=re.dtype)
    out[..., 0] = re
    out[..., 1] = im
    return out


def complex_scan_inputs(cfg: ScanConfig, t0: int = 0, t1: Optional[int] = None,
                        threads: int = 0) -> Dict[str, Optional[np.ndarray]]:
    """Inputs of a scan with complex A, B, C, in I/O representation.

    u, delta, z, D, delta_bias as in scan_inputs (same streams); A (dim,
    dstate, 2) float32 from complex_A; B and C (batch, t1 - t0, dstate, 2)
    (re, im) pairs, the real parts from the B and C streams and the imaginary
    parts ~ N(0, 1) from streams of their own; h0 (batch, dim, dstate, 2)
    float32 or None.
    """
    res = scan_inputs(cfg, t0, t1, threads)
    res["A"] = complex_A(cfg.dim, cfg.dstate)
    res["B"] = _interleave(res["B"], draw_tensor(cfg, "B_im", t0, t1, threads))
    res["C"] = _interleave(res["C"], draw_tensor(cfg, "C_im", t0, t1, threads))
    if res["h0"] is not None:
        im = np.empty_like(res["h0"])
        for b in range(cfg.batch):
            rng = np.random.default_rng([cfg.seed, _TID["h0_im"], b])
            im[b] = rng.standard_normal((cfg.dim, cfg.dstate), dtype=np.float32) * np.float32(cfg.h0_sigma)
        res["h0"] = _interleave(res["h0"], im)
    return res


def pairs_to_c128(arr: Optional[np.ndarray], io: str) -> Optional[np.ndarray]:
    """Exact complex128 values of an (..., 2) array of (re, im) pairs."""
    if arr is None:
        return None
    f = to_f64(arr, io)
    return f[..., 0] + 1j * f[..., 1]


# --------------------------------------------------------------------------
# decode workload
# --------------------------------------------------------------------------
def decode_params(cfg: DecodeConfig):
    """A, D, delta_bias for the decode workload (see channel_params)."""
    return channel_params(cfg.seed, cfg.dim, cfg.dstate, cfg.d_skip, cfg.dt_min, cfg.dt_max)


def decode_h0(cfg: DecodeConfig) -> np.ndarray:
    return draw_h0(cfg, cfg.batch, cfg.dim, cfg.dstate, cfg.h0_sigma)


def decode_step_inputs(cfg: DecodeConfig, step: int,
                       bias: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Fresh inputs of decode step ``step``: x, z, dt (batch, dim); B, C (batch, dstate).

    dt is drawn as round_bf16(logaddexp(0, r + bias)) with r ~ N(0, delta_sigma^2)
    evaluated in float64, i.e. an already-positive time step.
    """
    if bias is None:
        bias = decode_params(cfg)[2]

    def normal(tag, shape, sigma=1.0):
        rng = np.random.default_rng([cfg.seed, _TID[tag], step])
        x = rng.standard_normal(shape, dtype=np.float32)
        if sigma != 1.0:
            x *= np.float32(sigma)
        return x

    bd, bn = (cfg.batch, cfg.dim), (cfg.batch, cfg.dstate)
    r = normal("dt", bd, cfg.delta_sigma).astype(np.float64) + bias.astype(np.float64)[None, :]
    dt32 = np.logaddexp(0.0, r).astype(np.float32)
    return {
        "x": _round_io(normal("x", bd), cfg.io),
        "z": _round_io(normal("dz", bd), cfg.io) if cfg.has_z else None,
        "B": _round_io(normal("dB", bn), cfg.io),
        "C": _round_io(normal("dC", bn), cfg.io),
        "dt": _round_io(dt32, cfg.io),
    }


def iter_time_blocks(seqlen: int, block: int) -> Iterable[Tuple[int, int]]:
    for t0 in range(0, seqlen, block):
        yield t0, min(seqlen, t0 + block)


# --------------------------------------------------------------------------
# Mamba-2 SSD layer
# --------------------------------------------------------------------------
_SSD_TID = {"ssd_param": 20, "ssd_x": 21, "ssd_dt": 22, "ssd_B": 23, "ssd_C": 24, "ssd_z": 25, "ssd_h0": 26}


@dataclass(frozen=True)
class SsdConfig:
    """One SSD workload: x, z (batch, seqlen, heads, headdim), dt (batch,
    seqlen, heads), B, C (batch, seqlen, groups, dstate), all bf16; A, D,
    dt_bias (heads,) float32; state (batch, heads, headdim, dstate) float32."""
    name: str
    batch: int
    seqlen: int
    heads: int
    headdim: int
    groups: int
    dstate: int
    seed: int = 5
    dt_sigma: float = 0.5
    dt_min: float = 1e-3
    dt_max: float = 1e-1
    h0_sigma: Optional[float] = None
    has_z: bool = True

    @property
    def elements(self) -> int:
        return self.batch * self.seqlen * self.heads * self.headdim

    def with_(self, **kw) -> "SsdConfig":
        return replace(self, **kw)


# Mamba-2 at the 1.4B-layer shape: d_inner 4096 as 64 heads of 64, dstate 128,
# one group of B, C shared by every head.
MAMBA2_1P3B = SsdConfig("mamba2_b8_l2048_h64_p64_n128", 8, 2048, 64, 64, 1, 128, seed=5)


def ssd_params(cfg: SsdConfig) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """A, D, dt_bias (heads,) float32: A_h = -U(1, 16) (one scalar per head),
    D ~ U(0.5, 1.5), dt_bias = inverse softplus of dt0 log-uniform in
    [dt_min, dt_max] (as channel_params).  Draw order: A, dt0, D."""
    rng = np.random.default_rng([cfg.seed, _SSD_TID["ssd_param"]])
    A = (-rng.uniform(1.0, 16.0, size=cfg.heads)).astype(np.float32)
    dt0 = np.exp(rng.uniform(math.log(cfg.dt_min), math.log(cfg.dt_max), size=cfg.heads))
    bias = (dt0 + np.log(-np.expm1(-dt0))).astype(np.float32)
    D = rng.uniform(0.5, 1.5, size=cfg.heads).astype(np.float32)
    return A, D, bias


def ssd_rows(cfg: SsdConfig, name: str, b: int) -> np.ndarray:
    """Batch row b of an SSD sequence tensor ("x", "z", "dt", "B", "C") as bf16
    bits: x, z (seqlen, heads, headdim); dt (seqlen, heads) ~ N(0, dt_sigma^2)
    (the raw step); B, C (seqlen, groups, dstate); all others ~ N(0, 1)."""
    shape = {"x": (cfg.heads, cfg.headdim), "z": (cfg.heads, cfg.headdim), "dt": (cfg.heads,),
             "B": (cfg.groups, cfg.dstate), "C": (cfg.groups, cfg.dstate)}[name]
    rng = np.random.default_rng([cfg.seed, _SSD_TID["ssd_" + name], b])
    v = rng.standard_normal((cfg.seqlen,) + shape, dtype=np.float32)
    if name == "dt":
        v *= np.float32(cfg.dt_sigma)
    return f32_to_bf16_bits(v)


def ssd_inputs(cfg: SsdConfig) -> Dict[str, Optional[np.ndarray]]:
    """All inputs of one SSD call: x, dt, B, C, z (bf16 bits, with a batch
    axis), A, D, dt_bias (float32), h0 (float32 or None)."""
    res: Dict[str, Optional[np.ndarray]] = {
        k: np.stack([ssd_rows(cfg, k, b) for b in range(cfg.batch)]) for k in ("x", "dt", "B", "C", "z")}
    if not cfg.has_z:
        res["z"] = None
    res["A"], res["D"], res["dt_bias"] = ssd_params(cfg)
    if cfg.h0_sigma is not None:
        rng = np.random.default_rng([cfg.seed, _SSD_TID["ssd_h0"]])
        res["h0"] = (rng.standard_normal((cfg.batch, cfg.heads, cfg.headdim, cfg.dstate), dtype=np.float32)
                     * np.float32(cfg.h0_sigma))
    else:
        res["h0"] = None
    return res
