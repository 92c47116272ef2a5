"""GPU parity of ssm_selective_scan_fwd_complex (complex diagonal A) against
the fp64 oracle's complex scan: shapes spanning several chunks, 32-channel
blocks and ragged tails, every state-size layout, each optional input absent
or present, resumption through the returned state, and the 130M-layer shape
with S4D-Lin A.

Tolerances: those of the real scan, except that the fp32 bound grows with
max |Im A|.  The phase Delta Im A of every step is formed in fp32: Delta
carries up to ~2 ulp from the fp32 softplus and the product 0.5 ulp, an
absolute phase error of ~2.5 eps Delta |Im A| per step.  A contribution to
the state has been rotated through sum Delta steps' phases and weighs
exp(-|Re A| sum Delta), so the weighted phase error of a state is
~2.5 eps |Im A| / |Re A| = 5 eps |Im A| at Re A = -1/2 (S4D-Lin), independent
of Delta.  The readout sums N such terms, and its error is measured against
1 + |y|, with |y| up to ~sqrt(N) smaller than the sum of the terms' sizes
(about 4 at N = 16): the fp32 bound used is max(1e-5, 20 eps max|Im A|),
eps = 2^-24 (4.5e-5 at N = 16, 1.9e-4 at N = 64).  The bf16 bounds (2e-2 on
out, 1e-3 on the state) are far above it.
"""
import numpy as np
import pytest
import torch

import oracle
from selective_state_space_36_b200 import inputs as I
from tests import ssm_testlib as T

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from selective_state_space_36_b200 import binding
    return binding


def _oracle(x, io):
    return oracle.scan_complex(T.f64(x["u"], io), T.f64(x["delta"], io), I.pairs_to_c128(x["A"], "f32"),
                               I.pairs_to_c128(x["B"], io), I.pairs_to_c128(x["C"], io),
                               D=T.f64(x["D"], "f32"), z=T.f64(x["z"], io),
                               delta_bias=T.f64(x["delta_bias"], "f32"), delta_softplus=x["delta_softplus"],
                               h0=I.pairs_to_c128(x["h0"], "f32"))


def _gpu(lib, x, io, state=None):
    d = {k: T.to_dev(v, io) for k, v in x.items() if isinstance(v, np.ndarray)}
    A = torch.from_numpy(np.ascontiguousarray(x["A"], dtype=np.float32)).cuda()
    if state is None:
        u = x["u"]
        state = (torch.from_numpy(np.ascontiguousarray(x["h0"], dtype=np.float32)).cuda() if x["h0"] is not None
                 else torch.zeros((u.shape[0], u.shape[2], x["A"].shape[1], 2), device="cuda"))
    out = lib.selective_scan_fwd_complex(d["u"], d["delta"], A, d["B"], d["C"], D=d.get("D"), z=d.get("z"),
                                         delta_bias=d.get("delta_bias"), delta_softplus=x["delta_softplus"],
                                         last_state=state)
    torch.cuda.synchronize()
    return out, state


def _check(lib, io, batch, L, dim, N, seed, **kw):
    cfg = I.ScanConfig("cx", batch, L, dim, N, io=io, seed=seed, **kw)
    x = I.complex_scan_inputs(cfg)
    out, state = _gpu(lib, x, io)
    ref_out, ref_state = _oracle(x, io)
    tol_out = tol_state = None
    if io == "f32":
        tol_out = tol_state = max(1e-5, 20 * 2.0 ** -24 * float(np.abs(x["A"][..., 1]).max()))
    e1 = T.check_out(T.from_dev(out), ref_out, io, tol=tol_out)
    st = T.from_dev(state)
    got_state = st[..., 0] + 1j * st[..., 1]
    # the real scan's state check applied to the complex error: |h - h_ref|
    # against |h_ref| (elementwise for fp32, channel-wise for bf16)
    e2 = T.check_state(np.abs(got_state - ref_state) + np.abs(ref_state), np.abs(ref_state), io,
                       what="last_state (complex)", tol=tol_state)
    return e1, e2


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_complex_small_all_inputs(lib, io):
    _check(lib, io, 2, 100, 40, 16, 3, h0_sigma=0.5)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 8, 16, 17, 32, 33, 64])
def test_complex_state_sizes(lib, io, N):
    _check(lib, io, 1, 45, 33, N, 40 + N, h0_sigma=0.3)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("opt", [dict(has_z=False), dict(has_d=False), dict(has_bias=False),
                                 dict(has_z=False, has_d=False, has_bias=False), dict(h0_sigma=None)])
def test_complex_optional_inputs(lib, io, opt):
    _check(lib, io, 2, 70, 36, 16, 8, **opt)


def test_complex_resume_equals_one_pass(lib):
    cfg = I.ScanConfig("cx", 2, 96, 64, 16, io="f32", seed=12, h0_sigma=0.5)
    x = I.complex_scan_inputs(cfg)
    out_full, st_full = _gpu(lib, x, "f32")
    x1 = I.complex_scan_inputs(cfg, 0, 40)
    x2 = I.complex_scan_inputs(cfg, 40, 96)
    o1, st = _gpu(lib, x1, "f32")
    o2, st = _gpu(lib, x2, "f32", state=st)
    got = np.concatenate([T.from_dev(o1), T.from_dev(o2)], axis=1)
    assert np.array_equal(got, T.from_dev(out_full))
    assert torch.equal(st, st_full)


@pytest.mark.slow
def test_complex_mamba130m_shape(lib):
    # the 130M-layer shape with S4D-Lin A, against the oracle on 64 channels
    cfg = I.MAMBA130M.with_(dim=64)
    _check(lib, "bf16", cfg.batch, cfg.seqlen, cfg.dim, cfg.dstate, cfg.seed)


# The staged kernel (bf16, N = 16, dim a multiple of 8): several chunks of
# 32 steps, ragged chunk and tile tails, channels past the last full tile.
@pytest.mark.parametrize("batch,L,dim", [(1, 1, 8), (2, 31, 40), (1, 33, 64), (2, 100, 72), (1, 257, 96)])
def test_complex_staged_shapes(lib, batch, L, dim):
    _check(lib, "bf16", batch, L, dim, 16, 70 + L, h0_sigma=0.4)


@pytest.mark.parametrize("opt", [dict(has_z=False), dict(has_d=False), dict(has_bias=False),
                                 dict(has_z=False, has_d=False, has_bias=False), dict(h0_sigma=None),
                                 # Delta as given: small steps of either sign, no bias
                                 dict(softplus=False, has_bias=False, delta_sigma=0.05)])
def test_complex_staged_optional_inputs(lib, opt):
    _check(lib, "bf16", 2, 77, 48, 16, 9, **opt)


def test_complex_staged_resume_equals_one_pass(lib):
    # splits at multiples of 8 steps keep every step's owning lane, so the
    # two calls reproduce the one-pass result bit for bit
    cfg = I.ScanConfig("cx", 2, 136, 64, 16, io="bf16", seed=14, h0_sigma=0.5)
    x = I.complex_scan_inputs(cfg)
    out_full, st_full = _gpu(lib, x, "bf16")
    for cut in (40, 64):
        o1, st = _gpu(lib, I.complex_scan_inputs(cfg, 0, cut), "bf16")
        o2, st = _gpu(lib, I.complex_scan_inputs(cfg, cut, 136), "bf16", state=st)
        got = np.concatenate([T.from_dev(o1), T.from_dev(o2)], axis=1)
        assert np.array_equal(got, T.from_dev(out_full))
        assert torch.equal(st, st_full)


@pytest.mark.slow
def test_complex_mamba130m_full_sampled_channels(lib):
    """The benchmark's launch (batch 8, L 2048, dim 1536, N 16, bf16: the
    staged kernel) against the oracle on 12 channels spread over the 48
    32-channel tiles, every batch row."""
    cfg = I.MAMBA130M.with_(h0_sigma=0.3)
    x = I.complex_scan_inputs(cfg)
    out, state = _gpu(lib, x, "bf16")
    sel = np.array([0, 1, 31, 100, 257, 511, 640, 777, 1023, 1200, 1502, 1535])
    xs = dict(x)
    for k in ("u", "delta", "z"):
        xs[k] = np.ascontiguousarray(x[k][:, :, sel])
    for k in ("D", "delta_bias"):
        xs[k] = np.ascontiguousarray(x[k][sel])
    xs["A"] = np.ascontiguousarray(x["A"][sel])
    xs["h0"] = np.ascontiguousarray(x["h0"][:, sel])
    ref_out, ref_state = _oracle(xs, "bf16")
    idx = torch.as_tensor(sel, device="cuda")
    T.check_out(T.from_dev(out[:, :, idx]), ref_out, "bf16")
    st = T.from_dev(state[:, idx])
    got_state = st[..., 0] + 1j * st[..., 1]
    T.check_state(np.abs(got_state - ref_state) + np.abs(ref_state), np.abs(ref_state), "bf16",
                  what="last_state (complex)")
