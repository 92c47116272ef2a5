"""Host-side figures that bench.py reports beside its measurements: the
algorithmic byte count of the roofline, the arithmetic ceiling model and the
committed DRAM traffic lookup (no GPU)."""
import json
import os

import pytest

import bench
from selective_state_space_36_b200 import inputs as I

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_of_the_workloads():
    # u, delta, z read and out written in bf16 (8 bytes per element), plus
    # the B and C rows (2 x N x 2 bytes per (b, t))
    assert bench.algorithmic_bytes(I.MAMBA1P4B) == 8 * 2048 * 4096 * 8 + 8 * 2048 * 16 * 4
    assert bench.algorithmic_bytes(I.MAMBA1P4B) == 537_919_488
    assert bench.algorithmic_bytes(I.MAMBA130M) == 8 * 2048 * 1536 * 8 + 8 * 2048 * 16 * 4


def test_arithmetic_ceiling_model():
    # every decay on the SFU: 16 decays + softplus + silu = 18 SFU operations
    # per element at 16 per SM clock -> 16 / 18 elements per clock per SM
    assert bench.alu_ceiling_per_sm_clock(16, 16) == pytest.approx(16 / 18)
    # a quarter of the decays on the FMA pipe: the issue slots bind first
    # (4 x 14 + 4.5 x 4 + 2 x 16 + 14 = 120 cycles of a sub-partition per 128
    # elements' worth of lanes)
    assert bench.alu_ceiling_per_sm_clock(16, 12) == pytest.approx(128 / 120)
    # the best split the model allows is at least the SFU-only one
    assert bench.alu_ceiling_per_sm_clock(16) >= bench.alu_ceiling_per_sm_clock(16, 16)


def test_whole_job_rate_counts_every_rank():
    assert bench.whole_job_rate(4, 10**9, 1000.0) == pytest.approx(4.0)
    assert bench.whole_job_rate(1, 67_108_864, 0.4) == pytest.approx(167.77216)


def test_committed_traffic_is_tied_to_the_kernel_sources():
    with open(os.path.join(ROOT, "profiles", "scan_fwd_mamba1p4b_traffic.json")) as f:
        d = json.load(f)
    launches = d["launches"]
    mean = round(sum(x["dram_bytes_read"] for x in launches) / len(launches)) + \
        round(sum(x["dram_bytes_write"] for x in launches) / len(launches))
    assert d["dram_bytes_per_launch"] == mean
    assert bench.committed_traffic(d["kernel_source_sha"]) == d["dram_bytes_per_launch"]
    assert bench.committed_traffic("0" * 16) is None
    # the sources the hash covers exist, and the hash ignores comments
    sha = bench.kernel_source_sha()
    assert len(sha) == 16 and sha == bench.kernel_source_sha()
