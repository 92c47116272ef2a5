"""The long-sequence workload (batch 1, L = 1,048,576, dim 1536, N 16, bf16):
one call (the sequence-split variant is chosen automatically), and the same
sequence as 16 resumed calls of 65,536 steps through last_state.

Inputs (about 10 GB) are streamed to the device block by block; the host keeps
only B, C and the columns of the sampled channels, on which the fp64 oracle
runs over all 1,048,576 steps.
"""
import numpy as np
import pytest
import torch

from selective_state_space_36_b200 import inputs as I
from tests import ssm_testlib as T

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SEG = 65536


@pytest.fixture(scope="module")
def longseq():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cfg = I.LONGSEQ
    L, Dm = cfg.seqlen, cfg.dim
    rng = np.random.default_rng(0)
    dsel = np.unique(np.concatenate([[0, 127, 128, Dm - 1], rng.choice(Dm, 4, replace=False)]))
    dev = {k: torch.empty((1, L, Dm), dtype=torch.bfloat16, device="cuda") for k in ("u", "delta", "z")}
    host_cols = {k: np.empty((1, L, len(dsel)), dtype=np.uint16) for k in ("u", "delta", "z")}
    host_bc = {k: I.draw_tensor(cfg, k) for k in ("B", "C")}
    for t0, t1 in I.iter_time_blocks(L, SEG):
        for k in ("u", "delta", "z"):
            blk = I.draw_rows(cfg, k, 0, t0, t1)
            host_cols[k][0, t0:t1] = blk[:, dsel]
            dev[k][0, t0:t1].copy_(T.to_dev(blk, "bf16"))
    A, D, bias = I.channel_params(cfg.seed, Dm, cfg.dstate, cfg.d_skip)
    dev.update({k: T.to_dev(v, "bf16") for k, v in host_bc.items()})
    dev.update({"A": torch.from_numpy(A).cuda(), "D": torch.from_numpy(D).cuda(),
                "delta_bias": torch.from_numpy(bias).cuda()})
    sub = dict(host_cols, B=host_bc["B"], C=host_bc["C"], A=A[dsel], D=D[dsel],
               delta_bias=bias[dsel], h0=None, delta_softplus=True)
    ref_out, ref_state = T.oracle_scan(sub, "bf16")
    return cfg, dev, dsel, ref_out, ref_state


def _scan(lib, dev, sl=slice(None), state=None, **kw):
    return lib.selective_scan_fwd(dev["u"][:, sl], dev["delta"][:, sl], dev["A"], dev["B"][:, sl],
                                  dev["C"][:, sl], D=dev["D"], z=dev["z"][:, sl],
                                  delta_bias=dev["delta_bias"], last_state=state, **kw)


def test_one_call(longseq):
    from selective_state_space_36_b200 import binding as lib
    cfg, dev, dsel, ref_out, ref_state = longseq
    state = torch.zeros((1, cfg.dim, cfg.dstate), device="cuda")
    out = _scan(lib, dev, state=state)
    torch.cuda.synchronize()
    ds = torch.as_tensor(dsel, device="cuda")
    T.check_out(T.from_dev(out[:, :, ds]), ref_out, "bf16")
    T.check_state(T.from_dev(state[:, ds]), ref_state, "bf16")
    del out


def test_sixteen_resumed_segments_equal_one_pass(longseq):
    from selective_state_space_36_b200 import binding as lib
    cfg, dev, dsel, ref_out, ref_state = longseq
    one_state = torch.zeros((1, cfg.dim, cfg.dstate), device="cuda")
    one = _scan(lib, dev, state=one_state)
    state = torch.zeros_like(one_state)
    ds = torch.as_tensor(dsel, device="cuda")
    for s in range(cfg.seqlen // SEG):
        sl = slice(s * SEG, (s + 1) * SEG)
        part = _scan(lib, dev, sl, state=state)
        # this segment vs the one-pass result, every element (GPU-side compare)
        ref = one[:, sl].float()
        err = ((part.float() - ref).abs() / (1 + ref.abs())).max().item()
        assert err <= T.TOL_OUT["bf16"], f"segment {s}: {err:.3e}"
        T.check_out(T.from_dev(part[:, :, ds]), ref_out[:, sl], "bf16", what=f"segment {s} vs oracle")
        del part
    torch.cuda.synchronize()
    T.check_state(T.from_dev(state), T.from_dev(one_state), "bf16", what="resumed vs one-pass state")
    T.check_state(T.from_dev(state[:, ds]), ref_state, "bf16")
