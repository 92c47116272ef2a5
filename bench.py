"""Benchmark: selective-scan forward throughput at the Mamba-1.4B layer shape.

One step = one ssm_selective_scan_fwd call over one batch of the workload
(batch 8, L 2048, dim 4096, N 16, bf16 I/O, fp32 state) -- the whole hot path:
softplus(Delta), discretisation, recurrence, readout, D skip, silu(z) gate, the
fp32 state in and out.  Inputs are seeded synthetic data of that shape.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload mamba1p4b|mamba130m|longseq|decode|mamba1p4b_bwd|mamba130m_complex|mamba2_ssd]

The other workloads measure the remaining hot-path kernels the same way:
mamba130m (batch 8, L 2048, dim 1536), longseq (batch 1, L 1,048,576, dim 1536:
the sequence-split variant) and decode (one ssm_selective_state_update step at
batch 256, dim 5120, N 16; two state buffers alternate so that the 84 MB state
cannot simply stay in the 126 MB L2) and mamba1p4b_bwd (one
ssm_selective_scan_bwd call on the 1.4B-layer workload with a seeded dout),
mamba130m_complex (the scan with a complex diagonal A) and mamba2_ssd (one
ssm_ssd_scan_fwd call: Mamba-2's SSD layer, batch 8, L 2048, 64 heads of 64,
dstate 128, on the tensor cores).

Prints one JSON line (rank 0).  With --gpus N > 1 the script starts N ranks
itself (torchrun, one process per GPU) unless it already runs under one.  The
N ranks share one global workload of N times the workload's batch, whose
batch rows are split over the ranks (selective_state_space_36_b200.shard):
weak scaling, no collective on the data path.  The timed region is bracketed
by a barrier and a device synchronisation and its length is the maximum over
ranks; value = the global workload's elements over that time.

The reference arm (--impl reference) times the fp64 CPU oracle on the host
cores on a bounded sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_36_b200 import inputs as I  # noqa: E402

METRIC = "selective-scan fwd Gelem/s (B·L·D) at 1.4B-layer shape; % of HBM roofline"
UNIT = "Gelem/s"
WORKLOAD = I.MAMBA1P4B
L2_BYTES = 126 * 1024 * 1024
WORKLOADS = {"mamba1p4b": I.MAMBA1P4B, "mamba130m": I.MAMBA130M, "longseq": I.LONGSEQ,
             "decode": I.DECODE, "mamba1p4b_bwd": I.MAMBA1P4B, "mamba130m_complex": I.MAMBA130M,
             "mamba2_ssd": I.MAMBA2_1P3B}
SCAN_METRICS = {
    "mamba1p4b": METRIC,
    "mamba130m": "selective-scan fwd Gelem/s (B·L·D) at 130M-layer shape; % of HBM roofline",
    "longseq": "selective-scan fwd Gelem/s (B·L·D) at L=1,048,576 (sequence split); % of HBM roofline",
}
DECODE_METRIC = "decode state-update steps/s at batch 256, dim 5120, N 16; % of HBM roofline"
BWD_METRIC = "selective-scan bwd Gelem/s (B·L·D) at 1.4B-layer shape"
COMPLEX_METRIC = "selective-scan fwd, complex A (S4D-Lin), Gelem/s (B·L·D) at 130M-layer shape"


def bwd_sfu_ceiling_per_sm_clock(dstate: int = 16) -> float:
    """Elements per SM clock the backward's SFU work allows (the SFU delivers
    16 results per SM clock): the checkpointing forward pass needs dstate
    decays and the softplus exponential per element, the reverse pass the
    dstate decays again (recomputed), the softplus exponential, and an
    exponential and a reciprocal for each of sigmoid(z) and sigmoid(delta +
    bias).  An upper bound: it ignores the issue slots the rest takes."""
    return 16.0 / ((dstate + 1) + (dstate + 1 + 4))


def bwd_algorithmic_bytes(cfg: I.ScanConfig, ckpt_every: int = 8) -> int:
    """Bytes the backward must move: u, delta read twice (both passes), z,
    dout, B, C read and du, ddelta, dz written once, dB, dC written in fp32,
    and the state checkpoints written and read once."""
    es = 2 if cfg.io == "bf16" else 4
    seq = cfg.elements * es * (2 * 2 + 2 + 3)
    bc = cfg.batch * cfg.seqlen * cfg.dstate * (es * 3 + 4 * 2)
    ck = cfg.batch * cfg.dim * ((cfg.seqlen + ckpt_every - 1) // ckpt_every) * cfg.dstate * 4 * 2
    return seq + bc + ck


def alu_ceiling_per_sm_clock(dstate: int = 16, sfu_decays=None) -> float:
    """Elements per SM clock that the arithmetic of the scan allows on B200.

    Model built from measured unit costs (B200 pipe rates: the SFU returns 16
    ex2 per SM clock; next to scalar FFMA an SFU instruction takes ~4 issue
    cycles of its SM sub-partition and its unit for 8 cycles per warp; an
    f32x2 op takes 1 issue cycle).  Per element the method needs dstate
    decays exp(Delta A_n), 2 SFU ops for softplus and silu, 2 packed FP32
    issue cycles per state (Delta A, Delta u B, state FMA, readout FMA) and
    ~14 more issue cycles (softplus polynomial, gate, loads, stores).  A
    decay costs 4 issue cycles on the SFU or ~4.5 as an FMA-pipe polynomial.
    With ``sfu_decays`` = m of the dstate decays on the SFU (the rest on the
    FMA pipe) the ceiling is that of the shipped code; with None, the best m.
    Four sub-partitions x 32 lanes per SM clock.
    """
    best = 0.0
    for m in (range(dstate + 1) if sfu_decays is None else [min(dstate, sfu_decays * dstate // 16)]):
        sfu_cycles = 8.0 * (m + 2)
        issue_cycles = 4.0 * (m + 2) + 4.5 * (dstate - m) + 2.0 * dstate + 14.0
        best = max(best, 128.0 / max(sfu_cycles, issue_cycles))
    return best


def algorithmic_bytes(cfg: I.ScanConfig) -> int:
    """Bytes the method must move once: u, delta, z, B, C read and out written
    (the fp32 state in/out and A, D, bias are excluded, as in the metric)."""
    es = 2 if cfg.io == "bf16" else 4
    return cfg.elements * es * 4 + cfg.batch * cfg.seqlen * cfg.dstate * es * 2


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0, "source": "fallback"}


SCAN_KERNEL_SOURCES = ("scan_fwd_staged.cuh", "scan_common.cuh", "scan_kernels.cuh", "ssm_device.cuh", "cp_async.cuh")


def kernel_source_sha() -> str:
    """Hash of the staged scan kernel's sources with comments and blank space
    removed: a committed ncu traffic figure is valid only for the code it was
    captured on."""
    import re
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "selective_state_space_36_b200", "csrc")
    for f in SCAN_KERNEL_SOURCES:
        if True:
            with open(os.path.join(csrc, f)) as fh:
                code = fh.read()
            code = re.sub(r"/\*.*?\*/", "", code, flags=re.S)
            code = re.sub(r"//[^\n]*", "", code)
            code = re.sub(r"\s+", " ", code)
            h.update(f.encode() + b"\0" + code.encode())
    return h.hexdigest()[:16]


def committed_traffic(sha: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", "scan_fwd_mamba1p4b_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    if d.get("kernel_source_sha") != sha:
        return None
    return d.get("dram_bytes_per_launch")


# ------------------------------------------------------------ multi-GPU logic
def sharded_workload(args, rank: int, world: int):
    """The global workload of a run on `world` GPUs and this rank's share.

    Weak scaling: the global batch is the workload's batch times the number
    of GPUs, and the batch rows are split over the ranks (scan_shard), so each
    GPU scans the workload's shape; a run on one GPU is the workload itself.
    Rows are drawn by their global index, so the gathered result of N ranks
    equals one process scanning the global batch."""
    from selective_state_space_36_b200.shard import scan_shard
    cfg = WORKLOADS[args.workload]
    if getattr(args, "batch", 0) or getattr(args, "seqlen", 0):
        b_, l_ = args.batch or cfg.batch, args.seqlen or cfg.seqlen
        cfg = cfg.with_(batch=b_, seqlen=l_, name=f"{args.workload}_b{b_}_l{l_}_d{cfg.dim}_n{cfg.dstate}")
    if world > 1:
        gb = cfg.batch * world
        cfg = cfg.with_(batch=gb, name=cfg.name.replace(f"_b{cfg.batch}_", f"_b{gb}_", 1))
    return cfg, scan_shard(cfg.batch, cfg.dim, world, rank)


def max_over_ranks(values, device=None):
    """Element-wise maximum of a few timings over all ranks (one all-reduce)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def whole_job_rate(world: int, elements_per_rank: int, ms_per_step: float) -> float:
    """Gelem/s of the whole job: every rank's elements over the slowest rank's time."""
    return world * elements_per_rank / (ms_per_step * 1e-3) / 1e9


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_index: int, period_s: float = 0.001):
        self.samples, self.reasons, self.ok = [], set(), False
        self._stop = threading.Event()
        self.period = period_s
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.ok = False
        self._t = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self) -> dict:
        if self._t:
            self._stop.set()
            self._t.join()
        med = statistics.median(self.samples) if self.samples else None
        return {"sm_mhz": med, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ oracle arm
# The oracle's sample, the same for the reference arm and the cpu_baseline of
# our arm: one batch row of the workload, its first REF_CHANNELS channels,
# every time step (channels are independent, so this is the workload's own
# arithmetic on a bounded part of it).
REF_CHANNELS = 1024


def _oracle_block(cfg: I.ScanConfig, b: int):
    """fp64 inputs of the sample block of batch row b."""
    A, D, bias = I.channel_params(cfg.seed, cfg.dim, cfg.dstate, cfg.d_skip, cfg.dt_min, cfg.dt_max)
    ch = slice(0, min(REF_CHANNELS, cfg.dim))
    x = {}
    for k in I.SEQ_NAMES:
        rows = I.to_f64(I.draw_rows(cfg, k, b, 0, cfg.seqlen), cfg.io)
        x[k] = np.ascontiguousarray((rows if k in ("B", "C") else rows[:, ch])[None])
    x.update(A=A[ch].astype(np.float64), D=D[ch].astype(np.float64), bias=bias[ch].astype(np.float64))
    return x


def _time_oracle_block(x) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.scan(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"], delta_bias=x["bias"],
                delta_softplus=True)
    return time.perf_counter() - t0


def oracle_rate(cfg: I.ScanConfig, budget_s: float):
    """The fp64 oracle, as it stands, on sample blocks of the workload (one
    per batch row in turn) until ``budget_s`` seconds have been spent (at
    least one block).  Returns (Gelem/s, threads, elements, seconds)."""
    import oracle
    threads = min(oracle.default_threads(), REF_CHANNELS, cfg.dim)
    done, spent, b = 0, 0.0, 0
    while b == 0 or (spent < budget_s and b < 64):
        x = _oracle_block(cfg, b % cfg.batch)
        spent += _time_oracle_block(x)
        done += x["u"].shape[1] * x["u"].shape[2]
        b += 1
    return done / spent / 1e9, threads, done, spent


def run_reference(args, rank: int) -> int:
    if rank != 0:
        return 0
    import oracle
    cfg = WORKLOAD
    xs = [_oracle_block(cfg, b) for b in range(min(2, cfg.batch))]
    threads = min(oracle.default_threads(), REF_CHANNELS)
    per_step = []
    for i in range(args.warmup + args.steps):
        dt = _time_oracle_block(xs[i % len(xs)])
        if i >= args.warmup:
            per_step.append(dt)
    secs = sum(per_step)
    el = args.steps * cfg.seqlen * min(REF_CHANNELS, cfg.dim)
    value = el / secs / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": cfg.name, "batch": cfg.batch, "seqlen": cfg.seqlen,
                   "dim": cfg.dim, "dstate": cfg.dstate, "io": cfg.io,
                   "parallelism": "host threads over channels"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"per step: one batch row x {REF_CHANNELS} channels x {cfg.seqlen} steps "
                                   f"of the {cfg.name} workload"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def _upload(a, dev):
    import torch
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def _scan_device_inputs(cfg: I.ScanConfig, dev, sh=None):
    """Device copies of a scan workload's inputs, or of one rank's shard of
    them (rows [b0, b1) and channels [d0, d1) of the global workload, drawn
    by their global indices).  Long sequences are drawn and copied block by
    block so that the host never holds them whole."""
    import torch
    from selective_state_space_36_b200.shard import Shard
    sh = sh or Shard(0, cfg.batch, 0, cfg.dim)
    A, D, bias = I.channel_params(cfg.seed, cfg.dim, cfg.dstate, cfg.d_skip, cfg.dt_min, cfg.dt_max)
    dt = torch.bfloat16 if cfg.io == "bf16" else torch.float32
    d = {}
    for k in I.SEQ_NAMES:
        bc = k in ("B", "C")
        w = cfg.dstate if bc else sh.dim
        d[k] = torch.empty((sh.batch, cfg.seqlen, w), dtype=dt, device=dev)
        for i, b in enumerate(range(sh.b0, sh.b1)):
            for t0, t1 in I.iter_time_blocks(cfg.seqlen, 1 << 16):
                rows = I.draw_rows(cfg, k, b, t0, t1)
                d[k][i, t0:t1].copy_(_upload(rows if bc else rows[:, sh.d0:sh.d1], dev))
    cs = slice(sh.d0, sh.d1)
    d.update(A=_upload(np.ascontiguousarray(A[cs]), dev), D=_upload(np.ascontiguousarray(D[cs]), dev),
             delta_bias=_upload(np.ascontiguousarray(bias[cs]), dev))
    return d


def _time_steps(step, steps, warmup, stream, dev, world, sample_clocks=True):
    """Warm-up, then K steps bracketed by barrier + synchronize, CUDA events on
    the launching stream around the region; max over ranks.  The steps run back
    to back, as a caller issues them: no event is recorded between them (an
    event pair around every step added 2-6 us per step and stopped a decode
    step's launch from overlapping the end of the step before it), so a step's
    average duration is the region's time over K."""
    import torch
    import torch.distributed as dist
    for _ in range(max(warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev.index or 0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sample_clocks:
        sampler.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    elapsed_ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0]
    return elapsed_ms, elapsed_ms / steps, clocks


def _e2e(step_with_copies, steps, stream, dev, world):
    import torch
    import torch.distributed as dist
    for _ in range(2):
        step_with_copies()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step_with_copies()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks([e0.elapsed_time(e1)], dev)[0] / steps
    if world > 1:
        dist.barrier()
    return ms


def _base_line(metric, unit, value, world, args, ms_per_step, higher=True, io="bf16"):
    # dtype: the arithmetic type (fp32 everywhere); io_dtype: the element type
    # of the tensors read and written (bf16 for the benchmark workloads)
    return {"metric": metric, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": max(args.warmup, 3), "ms_per_step": ms_per_step, "higher_is_better": higher,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "io_dtype": io, "data": "synthetic"}


def run_scan(args, rank, world, dev):
    import torch
    from selective_state_space_36_b200 import binding as lib

    gcfg, sh = sharded_workload(args, rank, world)
    cfg = gcfg.with_(batch=sh.batch, dim=sh.dim)  # this rank's part
    d = _scan_device_inputs(gcfg, dev, sh)
    state = torch.zeros(sh.batch, sh.dim, cfg.dstate, device=dev)
    out = torch.empty_like(d["u"])
    stream = torch.cuda.current_stream(dev)
    plan = lib.scan_plan(sh.batch, cfg.seqlen, sh.dim, cfg.dstate, cfg.io)

    # Each step scans one batch of the workload and resumes from the state the
    # previous step left in last_state (a continued sequence): the same work.
    def step():
        lib.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                               delta_bias=d["delta_bias"], out=out, last_state=state, stream=stream)

    elapsed_ms, kernel_ms, clocks = _time_steps(step, args.steps, args.warmup, stream, dev, world)
    ms_per_step = elapsed_ms / args.steps
    metric = SCAN_METRICS.get(args.workload, METRIC)
    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"metric": metric, "value": gcfg.elements / (ms_per_step * 1e-3) / 1e9,
                              "unit": UNIT, "kernel_ms": kernel_ms, "config": {"workload": gcfg.name},
                              "note": "profiling run: no e2e, no cpu baseline"}), flush=True)
        return 0

    e2e = None
    if cfg.elements <= 1 << 28:
        # End to end through the public call with host buffers: every step
        # copies this rank's pinned host inputs in, scans, and copies the
        # output and the final state back.  The batch rows are independent
        # scans, so the step is pipelined by row as a user would run it: row
        # b + 1's host->device copy (one stream) overlaps row b's scan (the
        # compute stream) and row b - 1's device->host copy (a third stream).
        host = {k: v.cpu().pin_memory() for k, v in d.items()}
        host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        host_state = torch.empty(state.shape, dtype=state.dtype, pin_memory=True)
        host_state0 = torch.zeros(state.shape, dtype=state.dtype, pin_memory=True)
        h2d = sum(v.numel() * v.element_size() for v in host.values()) + host_state0.numel() * 4
        d2h = host_out.numel() * host_out.element_size() + host_state.numel() * 4
        e2e_steps = max(3, min(args.steps, 20))
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        rows = cfg.batch
        ev_in = [torch.cuda.Event() for _ in range(rows)]
        ev_done = [torch.cuda.Event() for _ in range(rows)]

        def e2e_step():
            s_in.wait_stream(stream)  # the previous step is done with the buffers
            with torch.cuda.stream(s_in):
                for k in ("A", "D", "delta_bias"):
                    d[k].copy_(host[k], non_blocking=True)
                for b in range(rows):
                    for k in I.SEQ_NAMES:
                        d[k][b].copy_(host[k][b], non_blocking=True)
                    state[b].copy_(host_state0[b], non_blocking=True)
                    ev_in[b].record(s_in)
            for b in range(rows):
                stream.wait_event(ev_in[b])
                sl = slice(b, b + 1)
                lib.selective_scan_fwd(d["u"][sl], d["delta"][sl], d["A"], d["B"][sl], d["C"][sl], D=d["D"],
                                       z=d["z"][sl], delta_bias=d["delta_bias"], out=out[sl],
                                       last_state=state[sl], stream=stream)
                ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                for b in range(rows):
                    s_out.wait_event(ev_done[b])
                    host_out[b].copy_(out[b], non_blocking=True)
                    host_state[b].copy_(state[b], non_blocking=True)
            stream.wait_stream(s_out)  # the step ends when its results are on the host

        e2e_ms = _e2e(e2e_step, e2e_steps, stream, dev, world)
        e2e = {"value": gcfg.elements / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world, "steps": e2e_steps,
               "pipeline": "by batch row: copy in / scan / copy out on three streams"}

    if rank == 0:
        peaks = measured_peaks()
        abytes = algorithmic_bytes(cfg)  # one launch on this rank
        achieved_gbs = abytes / (kernel_ms * 1e-3) / 1e9
        sm_mhz = clocks["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        info = lib.build_info()
        per_clk = alu_ceiling_per_sm_clock(cfg.dstate, info["sfu_decays_per_16"])
        alu_note = f"{info['sfu_decays_per_16']} of 16 decays on the SFU"
        if plan["launches"] == 2:
            # the sequence split computes every decay twice: pass 1 (its own
            # SFU share) then pass 2; the passes' times add
            c1 = alu_ceiling_per_sm_clock(cfg.dstate, info["split_pass1_sfu_decays_per_16"])
            per_clk = 1.0 / (1.0 / c1 + 1.0 / per_clk)
            alu_note = (f"two passes, {info['split_pass1_sfu_decays_per_16']} then {info['sfu_decays_per_16']} "
                        f"of 16 decays on the SFU")
        alu_peak = per_clk * sms * sm_mhz * 1e6 / 1e9
        kernel_gelem = cfg.elements / (kernel_ms * 1e-3) / 1e9
        sha = kernel_source_sha()
        line = _base_line(metric, UNIT, gcfg.elements / (ms_per_step * 1e-3) / 1e9, world, args, ms_per_step,
                          io=cfg.io)
        line.update({
            "config": {"workload": gcfg.name, "global_batch": gcfg.batch, "batch": gcfg.batch,
                       "seqlen": cfg.seqlen, "dim": gcfg.dim, "dstate": cfg.dstate, "io": cfg.io,
                       "per_gpu": f"rows {sh.b0}..{sh.b1 - 1}, channels {sh.d0}..{sh.d1 - 1} on rank 0",
                       "parallelism": f"dp{world} (batch rows, no exchange)" if world > 1 else "single",
                       "l2": f"inputs {abytes / 1e6:.0f} MB per GPU > {L2_BYTES >> 20} MB L2; no flush",
                       "plan": plan},
            "roofline": {
                "bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved_gbs / peaks["hbm_gbs"],
                "peak_source": peaks["source"] + " (copy bandwidth)",
                "traffic": committed_traffic(sha) if args.workload == "mamba1p4b" and plan["launches"] == 1 else None,
                "kernel_ms": kernel_ms, "algorithmic_bytes_per_launch": abytes,
                "alu": {"achieved": kernel_gelem, "peak": alu_peak, "unit": "Gelem/s",
                        "frac": kernel_gelem / alu_peak,
                        "peak_source": (f"derived for the shipped arithmetic ({alu_note}): "
                                        f"{per_clk:.3f} elem/clk/SM x {sms} SMs x "
                                        f"{sm_mhz:.0f} MHz (measured SFU/FMA issue costs)")},
                "kernel_source_sha": sha},
            "e2e": e2e,
            "gpu_launches": args.steps * plan["launches"],
            "clocks": clocks,
        })
        if world == 1 and not args.no_cpu_baseline:
            v, threads, el, secs = oracle_rate(cfg, budget_s=args.cpu_budget)
            line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
                                    "sample": f"{el} elements of {cfg.name} in blocks of one batch row x "
                                              f"{REF_CHANNELS} channels x 2048 steps ({secs:.1f} s)"}
        print(json.dumps(line), flush=True)
    return 0


def run_decode(args, rank, world, dev):
    import torch
    from selective_state_space_36_b200 import binding as lib

    cfg = I.DECODE if rank == 0 else I.DecodeConfig(**{**I.DECODE.__dict__, "seed": I.DECODE.seed + 1000 * rank})
    A, D, bias = I.decode_params(cfg)
    st = I.decode_step_inputs(cfg, 0, bias)
    d = {k: _upload(v, dev) for k, v in st.items()}
    Ad, Dd = _upload(A, dev), _upload(D, dev)
    h0 = I.decode_h0(cfg)
    states = [_upload(h0, dev), _upload(h0, dev)]  # 2 x 84 MB > L2: alternate them
    out = torch.empty_like(d["x"])
    stream = torch.cuda.current_stream(dev)
    k = [0]

    def step():
        lib.selective_state_update(states[k[0] & 1], d["x"], d["dt"], Ad, d["B"], d["C"], D=Dd, z=d["z"],
                                   out=out, stream=stream)
        k[0] += 1

    elapsed_ms, kernel_ms, clocks = _time_steps(step, args.steps, args.warmup, stream, dev, world)
    ms_per_step = elapsed_ms / args.steps
    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"metric": DECODE_METRIC, "value": world * 1e3 / ms_per_step, "unit": "steps/s",
                              "kernel_ms": kernel_ms, "config": {"workload": cfg.name},
                              "note": "profiling run: no e2e, no cpu baseline"}), flush=True)
        return 0
    channels = cfg.batch * cfg.dim
    es = 2
    abytes = channels * (cfg.dstate * 4 * 2 + 4 * es) + cfg.batch * cfg.dstate * es * 2 + cfg.dim * cfg.dstate * 4
    host = {kk: v.cpu().pin_memory() for kk, v in d.items()}
    host_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = host_out.numel() * host_out.element_size()

    def e2e_step():
        for kk in d:
            d[kk].copy_(host[kk], non_blocking=True)
        step()
        host_out.copy_(out, non_blocking=True)

    e2e_ms = _e2e(e2e_step, max(3, min(args.steps, 50)), stream, dev, world)
    if rank == 0:
        peaks = measured_peaks()
        achieved = abytes / (kernel_ms * 1e-3) / 1e9
        line = _base_line(DECODE_METRIC, "steps/s", world * 1e3 / ms_per_step, world, args, ms_per_step)
        line.update({
            "config": {"workload": cfg.name, "batch": cfg.batch, "dim": cfg.dim, "dstate": cfg.dstate,
                       "io": cfg.io, "per_gpu": "one full decode batch per GPU",
                       "l2": "two 84 MB state buffers alternate (168 MB > 126 MB L2)"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel_ms": kernel_ms,
                         "algorithmic_bytes_per_launch": abytes,
                         "peak_source": peaks["source"] + " (copy bandwidth)"},
            "e2e": {"value": world * 1e3 / e2e_ms, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": args.steps,
            "clocks": clocks,
        })
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            h = h0.astype(np.float64)
            spent, n = 0.0, 0
            while spent < args.cpu_budget and n < 50:
                s_in = I.decode_step_inputs(cfg, n, bias)
                f = lambda a: I.to_f64(a, cfg.io)
                t0 = time.perf_counter()
                _, h = oracle.state_update(h, f(s_in["x"]), f(s_in["dt"]), A, f(s_in["B"]), f(s_in["C"]),
                                           D=D, z=f(s_in["z"]))
                spent += time.perf_counter() - t0
                n += 1
            line["cpu_baseline"] = {"value": n / spent, "unit": "steps/s", "cores": 1, "kind": "oracle",
                                    "sample": f"{n} full decode steps ({spent:.1f} s)"}
        print(json.dumps(line), flush=True)
    return 0


def run_bwd(args, rank, world, dev):
    """One step = one ssm_selective_scan_bwd over the 1.4B-layer workload with a
    seeded upstream gradient dout (both kernels, the zeroing of the summed
    gradients and the checkpoint workspace are inside the step)."""
    import torch
    from selective_state_space_36_b200 import binding as lib

    gcfg, sh = sharded_workload(args, rank, world)
    d = _scan_device_inputs(gcfg, dev, sh)
    cfg = gcfg.with_(batch=sh.batch, dim=sh.dim)  # this rank's part
    dout = torch.empty_like(d["u"])
    for i, b in enumerate(range(sh.b0, sh.b1)):
        for t0, t1 in I.iter_time_blocks(cfg.seqlen, 1 << 16):
            dout[i, t0:t1].copy_(_upload(I.draw_rows(gcfg, "dout", b, t0, t1)[:, sh.d0:sh.d1], dev))
    h0 = torch.zeros(cfg.batch, cfg.dim, cfg.dstate, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lib.selective_scan_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], dout, D=d["D"], z=d["z"],
                               delta_bias=d["delta_bias"], h0=h0, stream=stream)

    elapsed_ms, call_ms, clocks = _time_steps(step, args.steps, args.warmup, stream, dev, world)
    ms_per_step = elapsed_ms / args.steps
    value = gcfg.elements / (ms_per_step * 1e-3) / 1e9
    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"metric": BWD_METRIC, "value": value, "unit": UNIT, "kernel_ms": call_ms,
                              "config": {"workload": cfg.name},
                              "note": "profiling run: no e2e, no cpu baseline"}), flush=True)
        return 0
    if rank == 0:
        peaks = measured_peaks()
        sm_mhz = clocks["sm_mhz"] or peaks.get("sm_max_mhz", 1965.0)
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        sfu_peak = bwd_sfu_ceiling_per_sm_clock(cfg.dstate) * sms * sm_mhz * 1e6 / 1e9
        call_gelem = cfg.elements / (call_ms * 1e-3) / 1e9
        abytes = bwd_algorithmic_bytes(cfg)
        line = _base_line(BWD_METRIC, UNIT, value, world, args, ms_per_step)
        line.update({
            "config": {"workload": cfg.name + "_bwd", "batch": cfg.batch, "seqlen": cfg.seqlen,
                       "dim": cfg.dim, "dstate": cfg.dstate, "io": cfg.io,
                       "per_gpu": "one full workload per GPU",
                       "parallelism": f"dp{world}" if world > 1 else "single",
                       "l2": f"inputs {abytes / 1e6:.0f} MB moved per call > {L2_BYTES >> 20} MB L2; no flush"},
            "roofline": {
                "bound": "alu", "achieved": call_gelem, "peak": sfu_peak, "unit": "Gelem/s",
                "frac": call_gelem / sfu_peak, "traffic": None, "kernel_ms": call_ms,
                "scope": "the whole backward call (checkpointing forward pass + reverse pass)",
                "peak_source": (f"derived SFU bound: {bwd_sfu_ceiling_per_sm_clock(cfg.dstate):.3f} elem/clk/SM"
                                f" x {sms} SMs x {sm_mhz:.0f} MHz"),
                "hbm": {"achieved": abytes / (call_ms * 1e-3) / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": abytes / (call_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                        "algorithmic_bytes_per_call": abytes,
                        "peak_source": peaks["source"] + " (copy bandwidth)"}},
            "e2e": None,
            "gpu_launches": args.steps * 2,
            "clocks": clocks,
        })
        print(json.dumps(line), flush=True)
    return 0


def run_complex(args, rank, world, dev):
    """One step = one ssm_selective_scan_fwd_complex over the 130M-layer
    workload with complex A = -1/2 + i pi n and complex B, C."""
    import torch
    from selective_state_space_36_b200 import binding as lib

    cfg = WORKLOADS[args.workload]
    if rank:
        cfg = cfg.with_(seed=cfg.seed + 1000 * rank)
    x = I.complex_scan_inputs(cfg)
    d = {k: _upload(v, dev) for k, v in x.items() if isinstance(v, np.ndarray)}
    state = torch.zeros(cfg.batch, cfg.dim, cfg.dstate, 2, device=dev)
    out = torch.empty_like(d["u"])
    stream = torch.cuda.current_stream(dev)

    def step():
        lib.selective_scan_fwd_complex(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                                       delta_bias=d["delta_bias"], out=out, last_state=state, stream=stream)

    elapsed_ms, kernel_ms, clocks = _time_steps(step, args.steps, args.warmup, stream, dev, world)
    ms_per_step = elapsed_ms / args.steps
    if rank == 0:
        peaks = measured_peaks()
        es = 2 if cfg.io == "bf16" else 4
        abytes = cfg.elements * es * 4 + cfg.batch * cfg.seqlen * cfg.dstate * es * 4
        achieved = abytes / (kernel_ms * 1e-3) / 1e9
        line = _base_line(COMPLEX_METRIC, UNIT, whole_job_rate(world, cfg.elements, ms_per_step), world, args,
                          ms_per_step)
        line.update({
            "config": {"workload": cfg.name + "_complex", "batch": cfg.batch, "seqlen": cfg.seqlen,
                       "dim": cfg.dim, "dstate": cfg.dstate, "io": cfg.io, "A": "-1/2 + i pi n"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None, "kernel_ms": kernel_ms,
                         "algorithmic_bytes_per_launch": abytes,
                         "note": "arithmetic-bound (exp, sincos and complex products per state); "
                                 "the HBM fraction is context"},
            "e2e": None, "gpu_launches": args.steps, "clocks": clocks,
        })
        print(json.dumps(line), flush=True)
    return 0


SSD_METRIC = "SSD (Mamba-2) fwd Gelem/s (B·L·heads·headdim) at batch 8, L 2048, 64 heads x 64, dstate 128"
SSD_CHUNK = 128


def ssd_algorithmic_bytes(cfg: I.SsdConfig) -> int:
    """x, z, dt, B, C read and out written once (bf16)."""
    per_tok = 2 * (3 * cfg.heads * cfg.headdim + cfg.heads + 2 * cfg.groups * cfg.dstate)
    return cfg.batch * cfg.seqlen * per_tok


def ssd_flops(cfg: I.SsdConfig, q: int = SSD_CHUNK) -> int:
    """Dense products of the chunked decomposition at chunk length q, per
    (batch row, head, chunk): C B^T (2 q^2 N), M X (2 q^2 P), C H^T (2 q N P)
    and the chunk state B^T (w o X) (2 q N P)."""
    chunks = (cfg.seqlen + q - 1) // q
    n, p = cfg.dstate, cfg.headdim
    return cfg.batch * cfg.heads * chunks * (2 * q * q * n + 2 * q * q * p + 4 * q * n * p)


def run_ssd(args, rank, world, dev):
    """One step = one ssm_ssd_scan_fwd over the Mamba-2 workload (batch rows
    split over the ranks as for the scan workloads)."""
    import torch
    from selective_state_space_36_b200 import binding as lib
    from selective_state_space_36_b200.shard import scan_shard
    g = I.MAMBA2_1P3B
    if args.batch or args.seqlen:
        g = g.with_(batch=args.batch or g.batch, seqlen=args.seqlen or g.seqlen)
    if world > 1:
        g = g.with_(batch=g.batch * world, name=g.name.replace(f"_b{g.batch}_", f"_b{g.batch * world}_", 1))
    sh = scan_shard(g.batch, g.heads, world, rank)
    cfg = g.with_(batch=sh.batch)
    d = {}
    for k in ("x", "dt", "B", "C", "z"):
        rows = np.stack([I.ssd_rows(g, k, b) for b in range(sh.b0, sh.b1)])
        d[k] = _upload(rows, dev)
    A, D, bias = I.ssd_params(g)
    d.update(A=_upload(A, dev), D=_upload(D, dev), dt_bias=_upload(bias, dev))
    state = torch.zeros(cfg.batch, cfg.heads, cfg.headdim, cfg.dstate, device=dev)
    out = torch.empty_like(d["x"])
    stream = torch.cuda.current_stream(dev)

    def step():
        lib.ssd_scan_fwd(d["x"], d["dt"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"], dt_bias=d["dt_bias"],
                         out=out, last_state=state, stream=stream)

    elapsed_ms, kernel_ms, clocks = _time_steps(step, args.steps, args.warmup, stream, dev, world)
    ms_per_step = elapsed_ms / args.steps
    value = g.elements / (ms_per_step * 1e-3) / 1e9
    if args.no_e2e:
        if rank == 0:
            print(json.dumps({"metric": SSD_METRIC, "value": value, "unit": UNIT, "kernel_ms": kernel_ms,
                              "config": {"workload": g.name}, "note": "profiling run"}), flush=True)
        return 0
    if rank == 0:
        peaks = measured_peaks()
        abytes = ssd_algorithmic_bytes(cfg)
        flops = ssd_flops(cfg)
        gbs = abytes / (kernel_ms * 1e-3) / 1e9
        tfs = flops / (kernel_ms * 1e-3) / 1e12
        tpeak = peaks.get("bf16_tflops_sustained") or peaks["bf16_tflops"]
        line = _base_line(SSD_METRIC, UNIT, value, world, args, ms_per_step, io="bf16")
        line.update({
            "config": {"workload": g.name, "global_batch": g.batch, "seqlen": g.seqlen, "heads": g.heads,
                       "headdim": g.headdim, "groups": g.groups, "dstate": g.dstate, "chunk": SSD_CHUNK,
                       "parallelism": f"dp{world} (batch rows, no exchange)" if world > 1 else "single",
                       "l2": f"inputs {abytes / 1e6:.0f} MB per GPU > {L2_BYTES >> 20} MB L2; no flush"},
            "roofline": {
                "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"] + " (copy bandwidth)",
                "traffic": None, "kernel_ms": kernel_ms, "algorithmic_bytes_per_launch": abytes,
                "tensor": {"achieved": tfs, "peak": tpeak, "unit": "TFLOP/s", "frac": tfs / tpeak,
                           "flops_per_launch": flops,
                           "peak_source": peaks["source"] + (" bf16 dense, sustained"
                                                             if peaks.get("bf16_tflops_sustained") else " bf16 dense")}},
            "e2e": None, "gpu_launches": args.steps, "clocks": clocks,
        })
        print(json.dumps(line), flush=True)
    return 0


def run_ours(args, rank: int, world: int, local_rank: int) -> int:
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev)
    try:
        if args.workload == "decode":
            return run_decode(args, rank, world, dev)
        if args.workload == "mamba1p4b_bwd":
            return run_bwd(args, rank, world, dev)
        if args.workload == "mamba130m_complex":
            return run_complex(args, rank, world, dev)
        if args.workload == "mamba2_ssd":
            return run_ssd(args, rank, world, dev)
        return run_scan(args, rank, world, dev)
    finally:
        if world > 1:
            dist.destroy_process_group()


def main() -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling cases)")
    ap.add_argument("--seqlen", type=int, default=0, help="override the workload's length (profiling cases)")
    ap.add_argument("--no-e2e", action="store_true", help="device-timed loop only (profiling cases)")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mamba1p4b")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # one process per GPU: re-run this command under torchrun
        import socket
        import subprocess
        with socket.socket() as so:
            so.bind(("127.0.0.1", 0))
            port = so.getsockname()[1]
        cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
               "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
        return subprocess.call(cmd)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "ours" and world != args.gpus and "WORLD_SIZE" in os.environ:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE {world}; using {world}", file=sys.stderr)
    if args.impl == "reference":
        return run_reference(args, rank)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
