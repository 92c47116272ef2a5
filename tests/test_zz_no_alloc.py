"""ssm_selective_scan_fwd_noalloc: the sequence-split scan for callers that
cannot allocate device memory at call time (its carries live in a static
scratch array inside the library instead of coming from cudaMallocAsync).

Checked through the C ABI against the allocating entry point
ssm_selective_scan_fwd, within the parity tolerances the other GPU tests use,
on two calls in a row (different inputs, so stale scratch contents from the
first call would show up in the second).  This file is collected last so that
a run stopping at its first failure has already run every other test; it also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

from selective_state_space_36_b200 import inputs as I
from tests import ssm_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from selective_state_space_36_b200 import binding
    return binding


def _dev(x, io):
    return {k: T.to_dev(v, io) for k, v in x.items() if isinstance(v, np.ndarray)}


def _run(lib, fn, d, x, segments):
    state = d["h0"].clone()
    out = torch.empty_like(d["u"])
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=x["delta_softplus"],
              out=out, last_state=state)
    if fn == "noalloc":
        lib.selective_scan_fwd_noalloc(d["u"], d["delta"], d["A"], d["B"], d["C"], segments=segments, **kw)
    else:
        lib.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], variant="split",
                               segments=segments, **kw)
    torch.cuda.synchronize()
    return out, state


@pytest.mark.parametrize("io", ["bf16", "f32"])
def test_noalloc_matches_allocating_entry_point_on_two_calls(lib, io):
    # two different problems back to back through the same static scratch
    cfgs = [I.ScanConfig("na1", 2, 5000, 96, 16, io=io, seed=31, h0_sigma=0.3, d_skip="uniform"),
            I.ScanConfig("na2", 1, 9000, 200, 16, io=io, seed=32, h0_sigma=0.5)]
    for cfg, segments in zip(cfgs, (7, 0)):
        x = I.scan_inputs(cfg)
        d = _dev(x, io)
        ref_out, ref_state = _run(lib, "alloc", d, x, segments)
        out, state = _run(lib, "noalloc", d, x, segments)
        T.check_out(T.from_dev(out), T.from_dev(ref_out), io)
        T.check_state(T.from_dev(state), T.from_dev(ref_state), io)


def test_noalloc_rejects_a_split_larger_than_its_scratch(lib):
    # batch 8 x dim 4096 x 16 states: 2 MiB of carries per segment -> 9 don't fit
    cfg = I.ScanConfig("big", 8, 4096, 4096, 16, io="bf16", seed=1)
    u = torch.zeros(cfg.batch, cfg.seqlen, cfg.dim, dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros(cfg.batch, cfg.seqlen, cfg.dstate, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(cfg.dim, cfg.dstate, device="cuda")
    out = torch.full_like(u, 7.0)
    with pytest.raises(lib.SSMError) as ei:
        lib.selective_scan_fwd_noalloc(u, u, A, Bm, Bm, out=out, segments=9)
    assert ei.value.status == lib.SSM_ERR_UNSUPPORTED
    assert b"static scratch" in lib.lib.ssm_last_error()
    torch.cuda.synchronize()
    assert torch.all(out == 7.0)  # nothing was launched


def _oracle_rows(x, io, dsel):
    sub = T.channel_subset(x, dsel)
    return T.oracle_scan(sub, io)


@pytest.mark.parametrize("shape,split_segments", [
    # batch 8 x dim 8192 x 16 states: the automatic split (3 segments) needs
    # 17.5 MB of carries; 2 segments (13.1 MB) fit the 16 MiB scratch
    ((8, 512, 8192), 2),
    # batch 32 x dim 4096: even 2 segments need 26 MB, so one pass runs
    ((32, 256, 4096), 1),
])
def test_noalloc_automatic_segments_fit_the_scratch(lib, shape, split_segments):
    batch, seqlen, dim = shape
    scratch = 16 * 1024 * 1024
    auto = lib.scan_plan(batch, seqlen, dim, 16, "bf16", variant="split")
    assert auto["workspace_bytes"] > scratch  # the default split would not fit
    if split_segments >= 2:
        fits = lib.scan_plan(batch, seqlen, dim, 16, "bf16", variant="split", segments=split_segments)
        over = lib.scan_plan(batch, seqlen, dim, 16, "bf16", variant="split", segments=split_segments + 1)
        assert fits["workspace_bytes"] <= scratch < over["workspace_bytes"]
    cfg = I.ScanConfig("na_auto", batch, seqlen, dim, 16, io="bf16", seed=33, h0_sigma=0.3, d_skip="uniform")
    x = I.scan_inputs(cfg)
    d = _dev(x, "bf16")
    for _ in range(2):  # two calls in a row through the same scratch
        out, state = _run(lib, "noalloc", d, x, 0)
        ref_state = d["h0"].clone()
        ref_out = lib.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"], z=d["z"],
                                         delta_bias=d["delta_bias"], last_state=ref_state)
        torch.cuda.synchronize()
        T.check_out(T.from_dev(out), T.from_dev(ref_out), "bf16")
        T.check_state(T.from_dev(state), T.from_dev(ref_state), "bf16")
    # sampled channels of every batch row against the fp64 oracle
    dsel = np.array([0, 1, 127, 128, dim // 2 + 5, dim - 1])
    ro, rs = _oracle_rows(x, "bf16", dsel)
    ds = torch.as_tensor(dsel, device="cuda")
    T.check_out(T.from_dev(out[:, :, ds]), ro, "bf16")
    T.check_state(T.from_dev(state[:, ds]), rs, "bf16")
