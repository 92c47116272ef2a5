"""GPU parity of ssm_selective_scan_fwd against the fp64 oracle.

Every case compares the CUDA path (called through the C ABI) element by
element with the oracle on the same seeded inputs: small shapes spanning
several chunks, blocks and ragged tails for every kernel layout and variant,
and the tiny fp32, Mamba-130M and Mamba-1.4B workloads in full (the last in
the launch configuration the benchmark times).  The L = 1,048,576 workload is
in test_longseq_gpu.py.
"""
import numpy as np
import pytest
import torch

from selective_state_space_36_b200 import inputs as I
from tests import ssm_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from selective_state_space_36_b200 import binding
    return binding


def _case(io, batch, L, dim, N, seed, **kw):
    cfg = I.ScanConfig("case", batch, L, dim, N, io=io, seed=seed, **kw)
    return cfg, I.scan_inputs(cfg)


def _check(x, io, report=None, **kw):
    out, state = T.gpu_scan(x, io, **kw)
    ref_out, ref_state = T.oracle_scan(x, io)
    e1 = T.check_out(T.from_dev(out), ref_out, io)
    e2 = T.check_state(T.from_dev(state), ref_state, io)
    if report:
        e3 = T.state_err_elementwise(T.from_dev(state), ref_state)
        print(f"[{report}] out {e1:.2e} (1+|y|); state norm-wise {e2:.2e}, elementwise with floor {e3:.2e}")
    return e1, e2


# ------------------------------------------------------------- named workloads
def test_tiny_fp32_workload():
    x = I.scan_inputs(I.TINY_F32)
    _check(x, "f32")


def test_tiny_fp32_workload_with_h0_and_every_variant():
    x = I.scan_inputs(I.TINY_F32.with_(h0_sigma=0.5))
    for kw in [dict(variant="slab", lanes=1), dict(variant="slab", lanes=2),
               dict(variant="slab", lanes=4), dict(variant="split", segments=3),
               dict(variant="split", segments=4, lanes=4)]:
        _check(x, "f32", **kw)


@pytest.mark.slow
def test_mamba130m_workload_full():
    x = I.scan_inputs(I.MAMBA130M)
    _check(x, "bf16", report="mamba130m")


@pytest.mark.slow
def test_mamba1p4b_workload_full():
    """The benchmark's workload and launch configuration, every element."""
    x = I.scan_inputs(I.MAMBA1P4B)
    _check(x, "bf16", report="mamba1p4b")


# ------------------------------------------------------ layouts and variants
LAYOUTS = [dict(variant="slab", lanes=1), dict(variant="slab", lanes=2), dict(variant="slab", lanes=4),
           dict(variant="split", segments=2), dict(variant="split", segments=5, lanes=2),
           dict(variant="split", segments=7, lanes=4)]


FAMILIES = {"generic": dict(family="generic"), "staged": dict(family="staged", cpl=1),
            "staged_cpl2": dict(family="staged", cpl=2)}


@pytest.mark.parametrize("family", sorted(FAMILIES))
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("layout", range(len(LAYOUTS)))
def test_layouts_ragged(io, layout, family):
    # dim 200: full channel tiles + a ragged one; L 333 = several chunks + a tail
    _, x = _case(io, 3, 333, 200, 16, seed=10 + layout, h0_sigma=0.3, d_skip="uniform")
    _check(x, io, **FAMILIES[family], **LAYOUTS[layout])


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 5, 8, 13, 16, 17, 24, 32, 33, 64])
def test_state_sizes(io, N):
    # dim 37: no 16-byte rows, so the generic kernel runs
    _, x = _case(io, 2, 130, 37, N, seed=N, h0_sigma=0.2)
    _check(x, io)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [8, 16, 24, 32, 64])
@pytest.mark.parametrize("lanes", [1, 2, 4])
@pytest.mark.parametrize("cpl", [1, 2])
def test_state_sizes_staged(io, N, lanes, cpl):
    _, x = _case(io, 2, 130, 40, N, seed=N + lanes, h0_sigma=0.2)
    _check(x, io, family="staged", lanes=lanes, variant="slab", cpl=cpl)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("flags", ["no_z", "no_d", "no_bias", "no_softplus", "bare"])
def test_optional_inputs(io, flags):
    kw = dict(has_z=flags not in ("no_z", "bare"), has_d=flags not in ("no_d", "bare"),
              has_bias=flags not in ("no_bias", "bare"), softplus=flags not in ("no_softplus",))
    if flags == "no_softplus":
        kw["delta_sigma"] = 0.02  # keep raw + bias (the Delta itself) mostly positive
    _, x = _case(io, 2, 150, 70, 16, seed=3, **kw)
    if flags == "no_softplus":
        # without softplus Delta = raw + bias; make the bias small and positive
        x["delta_bias"] = np.abs(x["delta_bias"]).astype(np.float32) * 0.01
    _check(x, io)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_single_step_and_single_channel(io):
    for (batch, L, dim) in [(1, 1, 1), (1, 1, 300), (2, 65, 1), (1, 64, 129), (5, 2, 3)]:
        _, x = _case(io, batch, L, dim, 16, seed=L + dim, h0_sigma=0.5)
        _check(x, io)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_split_equals_slab_long(io):
    """Sequence split vs one pass at many segment counts, both vs the oracle."""
    _, x = _case(io, 1, 4 * 1024 + 77, 24, 16, seed=7, h0_sigma=0.3)
    ref_out, ref_state = T.oracle_scan(x, io)
    for fam in ("generic", "staged", "staged_cpl2"):
        for seg in (2, 3, 16, 65):
            out, st = T.gpu_scan(x, io, variant="split", segments=seg, **FAMILIES[fam])
            T.check_out(T.from_dev(out), ref_out, io)
            T.check_state(T.from_dev(st), ref_state, io)


def test_delta_zero_keeps_state_bit_exact():
    """Delta = 0 (raw 0, no bias, softplus off): Abar = 1 and Bbar = 0, so the
    state comes back bit for bit and out = C h0 + D u."""
    for io in ("f32", "bf16"):
        _, x = _case(io, 2, 100, 50, 16, seed=2, h0_sigma=1.0, softplus=False, has_bias=False, has_z=False)
        x["delta"] = np.zeros_like(x["delta"])
        out, st = T.gpu_scan(x, io)
        assert np.array_equal(st.cpu().numpy(), x["h0"])
        ref_out, _ = T.oracle_scan(x, io)
        T.check_out(T.from_dev(out), ref_out, io)


def test_resume_from_last_state_equals_one_pass():
    """Scanning [0, k) then [k, L) from the returned state equals one pass."""
    for io in ("f32", "bf16"):
        _, x = _case(io, 2, 700, 96, 16, seed=5)
        full_out, full_st = T.gpu_scan(x, io)
        parts, st = [], torch.zeros_like(full_st)
        for t0, t1 in [(0, 1), (1, 200), (200, 333), (333, 700)]:
            sl = {k: (v[:, t0:t1] if isinstance(v, np.ndarray) and v.ndim == 3 and k != "h0" else v)
                  for k, v in x.items()}
            from selective_state_space_36_b200 import binding
            d = {k: T.to_dev(v, io) for k, v in sl.items() if isinstance(v, np.ndarray)}
            parts.append(binding.selective_scan_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], D=d["D"],
                                                    z=d["z"], delta_bias=d["delta_bias"], last_state=st))
        out = torch.cat(parts, dim=1)
        ref_out, ref_st = T.oracle_scan(x, io)
        T.check_out(T.from_dev(out), ref_out, io)
        T.check_state(T.from_dev(st), ref_st, io)
        # and against the one-pass GPU result
        T.check_out(T.from_dev(out), T.from_dev(full_out), io)


def test_empty_inputs_leave_state_untouched(lib):
    for (batch, L, dim) in [(2, 0, 8), (0, 5, 8), (2, 5, 0)]:
        u = torch.zeros(batch, L, dim, device="cuda", dtype=torch.bfloat16)
        A = -torch.ones(dim, 16, device="cuda")
        Bm = torch.zeros(batch, L, 16, device="cuda", dtype=torch.bfloat16)
        st = torch.randn(batch, dim, 16, device="cuda")
        st0 = st.clone()
        out = lib.selective_scan_fwd(u, u, A, Bm, Bm, last_state=st)
        torch.cuda.synchronize()
        assert out.shape == (batch, L, dim) and torch.equal(st, st0)


def test_failed_call_leaves_no_cuda_error_behind(lib):
    """A call that fails inside a CUDA runtime call returns SSM_ERR_CUDA and
    leaves the runtime's error state clean for the caller (torch shares it).
    Here the sequence split asks cudaMallocAsync for ~1 TB of carries, which
    fails before anything is launched; the data pointers are never used."""
    import ctypes
    dims = lib.SSMDims(1, 65536, 1 << 24, 16)
    opts = lib.SSMScanOpts(2, 1024, 1, 1, 0)  # split, 1024 segments, 1 lane, generic
    fake = 0x100000
    rc = lib.lib.ssm_selective_scan_fwd_ex(dims, lib.SSM_BF16, fake, fake, fake, fake, fake, None, None,
                                           None, 1, fake, None, ctypes.byref(opts), None)
    assert rc == lib.SSM_ERR_CUDA
    assert b"workspace" in lib.lib.ssm_last_error()
    torch.cuda.synchronize()
    assert torch.ones(8, device="cuda").sum().item() == 8.0


# ----------------------------------------------- exact zero-order hold on B
@pytest.mark.parametrize("family", ["generic", "staged"])
@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("layout", [dict(variant="slab", lanes=1), dict(variant="slab", lanes=4),
                                    dict(variant="split", segments=3)])
def test_zoh_b_matches_oracle(io, family, layout):
    """Bbar = (Delta A)^-1 (exp(Delta A) - 1) Delta B (【論文要約】Mamba notes,
    数式解説 3) against the oracle's ZOH mode, including Delta A near 0 (series
    branch) and larger Delta A (direct branch)."""
    _, x = _case(io, 2, 300, 96, 16, seed=41, h0_sigma=0.3, d_skip="uniform", dt_max=0.5)
    out, st = T.gpu_scan(x, io, family=family, zoh_b=True, **layout)
    ref_out, ref_st = T.oracle_scan(x, io, zoh_b=True)
    T.check_out(T.from_dev(out), ref_out, io)
    T.check_state(T.from_dev(st), ref_st, io)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_theorem1_gated_rnn_on_gpu(io):
    """N = 1, A = -1, B = C = 1, no skip, no gate, Delta = softplus(raw + bias),
    exact ZOH: the scan is the gated RNN h_t = (1 - g_t) h_{t-1} + g_t x_t with
    g_t = sigmoid(raw_t + bias) (【論文要約】Mamba notes, 数式解説 4, Theorem 1),
    computed here in fp64 from the rounded inputs, independently of the oracle."""
    from scipy.special import expit
    cfg, x = _case(io, 2, 200, 40, 1, seed=43, h0_sigma=0.5, has_z=False, has_d=False)
    x["A"] = -np.ones_like(x["A"])
    ones = np.ones_like(I.to_f64(x["B"], io))
    x["B"] = x["C"] = (I.f32_to_bf16_bits(ones.astype(np.float32)) if io == "bf16"
                       else ones.astype(np.float32))
    out, st = T.gpu_scan(x, io, zoh_b=True)
    u, raw = I.to_f64(x["u"], io), I.to_f64(x["delta"], io)
    g = expit(raw + x["delta_bias"].astype(np.float64)[None, None, :])
    h = x["h0"][:, :, 0].astype(np.float64)
    ref = np.zeros_like(u)
    for t in range(cfg.seqlen):
        h = (1.0 - g[:, t]) * h + g[:, t] * u[:, t]
        ref[:, t] = h
    T.check_out(T.from_dev(out), ref, io)
    T.check_state(T.from_dev(st)[:, :, 0:1], h[:, :, None], io)
