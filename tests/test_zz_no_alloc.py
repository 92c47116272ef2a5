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
