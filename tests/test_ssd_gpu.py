"""Mamba-2 SSD layer on the GPU (ssm_ssd_scan_fwd, tensor cores) against the
fp64 oracle (oracle.ssd_scan, the linear form, pinned in test_oracle_pins).

Tolerances: the bf16 ones of the selective scan -- out within
2e-2 (1 + |ref|), the returned state within 1e-3 of each state row's largest
value (norm-wise over dstate).  The arithmetic they cover: a bf16 intra-chunk
matrix (~2^-9 relative), fp32 accumulation, a state carried in fp32 whose
products (update and inter-chunk output) take two-term bf16 splits (~2^-17).
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_36_b200 import inputs as I
from tests import ssm_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from selective_state_space_36_b200 import binding
    return binding


def _f64(a):
    return None if a is None else I.to_f64(a, "bf16")


def _oracle(x, heads=None, softplus=True):
    hs = slice(None) if heads is None else np.asarray(heads)
    sub = lambda a: None if a is None else a[:, :, hs]
    return oracle.ssd_scan(_f64(sub(x["x"])), _f64(sub(x["dt"])), x["A"][hs].astype(float), _f64(x["B"]),
                           _f64(x["C"]), D=x["D"][hs].astype(float), z=_f64(sub(x["z"])),
                           dt_bias=x["dt_bias"][hs].astype(float), dt_softplus=softplus,
                           h0=None if x["h0"] is None else x["h0"][:, hs].astype(float))


def _gpu(lib, x, softplus=True, state=None):
    d = {k: T.to_dev(v, "bf16") for k, v in x.items() if isinstance(v, np.ndarray) and v.dtype == np.uint16}
    f = {k: torch.from_numpy(np.ascontiguousarray(x[k])).cuda() for k in ("A", "D", "dt_bias")}
    if state is None and x["h0"] is not None:
        state = torch.from_numpy(x["h0"]).cuda()
    out = lib.ssd_scan_fwd(d["x"], d["dt"], f["A"], d["B"], d["C"], D=f["D"], z=d.get("z"),
                           dt_bias=f["dt_bias"], dt_softplus=softplus, last_state=state)
    torch.cuda.synchronize()
    return out, state


CASES = [
    # (batch, seqlen, heads, groups, dstate, gate, h0)
    (2, 300, 3, 1, 128, True, 0.3),   # three chunks, ragged tail, initial state
    (1, 256, 4, 2, 64, False, None),  # dstate 64, two groups, no gate
    (2, 77, 2, 1, 128, True, 0.5),    # shorter than one chunk
    (1, 1, 2, 1, 128, True, 0.5),     # one token
    (3, 129, 2, 2, 128, True, None),  # one step into the second chunk
]


@pytest.mark.parametrize("batch,seqlen,heads,groups,dstate,gate,h0", CASES)
def test_ssd_matches_oracle(lib, batch, seqlen, heads, groups, dstate, gate, h0):
    cfg = I.SsdConfig("t", batch, seqlen, heads, 64, groups, dstate, seed=11, h0_sigma=h0, has_z=gate)
    x = I.ssd_inputs(cfg)
    out, state = _gpu(lib, x)
    ro, rs = _oracle(x)
    T.check_out(T.from_dev(out), ro, "bf16")
    if state is not None:
        T.check_state(T.from_dev(state), rs, "bf16")


def test_ssd_without_softplus(lib):
    # Delta = dt itself: small positive steps, no bias (the workload's bias is
    # the inverse softplus of a small dt0, i.e. negative, and would make the
    # decays grow without softplus)
    cfg = I.SsdConfig("t", 1, 200, 2, 64, 1, 128, seed=12, h0_sigma=0.2)
    x = I.ssd_inputs(cfg)
    x["dt"] = I.f32_to_bf16_bits(np.abs(I.to_f64(x["dt"], "bf16")).astype(np.float32) * 0.05)
    x["dt_bias"] = np.zeros_like(x["dt_bias"])
    out, state = _gpu(lib, x, softplus=False)
    ro, rs = _oracle(x, softplus=False)
    T.check_out(T.from_dev(out), ro, "bf16")
    T.check_state(T.from_dev(state), rs, "bf16")


def test_ssd_resume_equals_one_pass(lib):
    cfg = I.SsdConfig("t", 2, 640, 2, 64, 1, 128, seed=13, h0_sigma=0.3)
    x = I.ssd_inputs(cfg)
    out, state = _gpu(lib, x)
    cut = 384
    first = {k: (v[:, :cut] if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v) for k, v in x.items()}
    second = {k: (v[:, cut:] if isinstance(v, np.ndarray) and v.dtype == np.uint16 else v) for k, v in x.items()}
    o1, s1 = _gpu(lib, first)
    o2, s2 = _gpu(lib, second, state=s1)
    T.check_out(T.from_dev(torch.cat([o1, o2], 1)), T.from_dev(out), "bf16")
    T.check_state(T.from_dev(s2), T.from_dev(state), "bf16")


@pytest.mark.slow
def test_ssd_mamba2_workload_sampled_heads(lib):
    """The benchmark workload (batch 8, L 2048, 64 heads of 64, dstate 128)
    in the launch the benchmark times; the oracle on 4 heads of every row."""
    cfg = I.MAMBA2_1P3B.with_(h0_sigma=0.2)
    x = I.ssd_inputs(cfg)
    out, state = _gpu(lib, x)
    hsel = [0, 17, 42, 63]
    ro, rs = _oracle(x, heads=hsel)
    hs = torch.as_tensor(hsel, device="cuda")
    T.check_out(T.from_dev(out[:, :, hs]), ro, "bf16")
    T.check_state(T.from_dev(state[:, hs]), rs, "bf16")
    assert lib.device_status() == 0


def test_ssd_empty_and_rejected_shapes(lib):
    cfg = I.SsdConfig("t", 1, 0, 2, 64, 1, 128, seed=1)
    x = torch.zeros(1, 0, 2, 64, dtype=torch.bfloat16, device="cuda")
    dt = torch.zeros(1, 0, 2, dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros(1, 0, 1, 128, dtype=torch.bfloat16, device="cuda")
    A = -torch.ones(2, device="cuda")
    st = torch.full((1, 2, 64, 128), 3.0, device="cuda")
    lib.ssd_scan_fwd(x, dt, A, Bm, Bm, last_state=st)
    torch.cuda.synchronize()
    assert torch.all(st == 3.0)  # seqlen 0: state unchanged
    x = torch.zeros(1, 8, 2, 32, dtype=torch.bfloat16, device="cuda")
    dt = torch.zeros(1, 8, 2, dtype=torch.bfloat16, device="cuda")
    Bm = torch.zeros(1, 8, 1, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.SSMError) as ei:
        lib.ssd_scan_fwd(x, dt, A, Bm, Bm)
    assert ei.value.status == lib.SSM_ERR_UNSUPPORTED
