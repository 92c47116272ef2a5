"""Pins of the fp64 oracle to facts fixed by the pages and by mathematics.

None of these re-types the oracle's loop: each compares it with an independent
route to the same number (an unrolled closed sum, a closed form, a library
convolution, a library softplus/sigmoid, an exact invariant), so a dropped
term, a wrong sign, a wrong index or a transposed operand in the oracle fails
at least one of them.  No GPU is involved.

Sources: NL-345, Mamba: Linear-Time Sequence Modeling with Selective State
Spaces (section 2: eq. (2) recurrence, eq. (3) convolution, "Linear Time
Invariance", "Structure and Dimensions"; section 1: recurrent inference);
【論文要約】Mamba notes (数式解説 3 ZOH; 4 Theorem 1; S6 Algorithm 2).
"""
import math

import numpy as np
import pytest
from scipy.special import expit

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _rand_case(rng, batch=2, L=11, dim=3, N=4, softplus=True, bias=True, gate=True,
               dskip=True, h0=True):
    u = rng.standard_normal((batch, L, dim))
    delta = rng.standard_normal((batch, L, dim)) * 0.7
    A = -rng.uniform(0.2, 2.5, size=(dim, N))
    B = rng.standard_normal((batch, L, N))
    C = rng.standard_normal((batch, L, N))
    D = rng.standard_normal(dim) if dskip else None
    z = rng.standard_normal((batch, L, dim)) if gate else None
    bvec = rng.standard_normal(dim) * 0.5 if bias else None
    hh = rng.standard_normal((batch, dim, N)) if h0 else None
    return dict(u=u, delta=delta, A=A, B=B, C=C, D=D, z=z, delta_bias=bvec,
                delta_softplus=softplus, h0=hh)


def _brute(case, zoh_b=False):
    """Fully unrolled y_t = sum_{s<=t} C_t (prod_{r=s+1..t} Abar_r) Bbar_s x_s
    + C_t (prod_{r<=t} Abar_r) h0 + D x_t, then the silu(z) gate; pure-Python
    loops with explicit products (no running state)."""
    u, delta, A, B, C = case["u"], case["delta"], case["A"], case["B"], case["C"]
    batch, L, dim = u.shape
    N = A.shape[1]
    out = np.zeros_like(u)
    last = np.zeros((batch, dim, N))
    for b in range(batch):
        for d in range(dim):
            dl = []
            for t in range(L):
                s = delta[b, t, d] + (case["delta_bias"][d] if case["delta_bias"] is not None else 0.0)
                dl.append(math.log1p(math.exp(s)) if case["delta_softplus"] else s)
            abar = [[math.exp(dl[t] * A[d, n]) for n in range(N)] for t in range(L)]
            if zoh_b:
                bbar = [[(math.exp(dl[t] * A[d, n]) - 1.0) / (dl[t] * A[d, n]) * dl[t] * B[b, t, n]
                         for n in range(N)] for t in range(L)]
            else:
                bbar = [[dl[t] * B[b, t, n] for n in range(N)] for t in range(L)]

            def state_at(t, n):
                tot = 0.0
                if case["h0"] is not None:
                    p = 1.0
                    for r in range(0, t + 1):
                        p *= abar[r][n]
                    tot += p * case["h0"][b, d, n]
                for s in range(t + 1):
                    p = 1.0
                    for r in range(s + 1, t + 1):
                        p *= abar[r][n]
                    tot += p * bbar[s][n] * u[b, s, d]
                return tot

            for t in range(L):
                y = sum(C[b, t, n] * state_at(t, n) for n in range(N))
                if case["D"] is not None:
                    y += case["D"][d] * u[b, t, d]
                if case["z"] is not None:
                    zz = case["z"][b, t, d]
                    y *= zz * expit(zz)
                out[b, t, d] = y
            for n in range(N):
                last[b, d, n] = state_at(L - 1, n)
    return out, last


def _run(oracle_mod, case, **kw):
    return oracle_mod.scan(case["u"], case["delta"], case["A"], case["B"], case["C"],
                           D=case["D"], z=case["z"], delta_bias=case["delta_bias"],
                           delta_softplus=case["delta_softplus"], h0=case["h0"], **kw)


def _close(a, b, tol):
    a, b = np.asarray(a), np.asarray(b)
    err = np.max(np.abs(a - b) / (1.0 + np.abs(b))) if a.size else 0.0
    assert err <= tol, f"max rel err {err:.3e} > {tol:.1e}"


@pytest.mark.parametrize("zoh_b", [False, True])
@pytest.mark.parametrize("variant", ["full", "no_softplus", "no_gate_no_skip", "no_bias_no_h0"])
def test_brute_force_unrolled_sum(oracle_mod, zoh_b, variant):
    rng = np.random.default_rng(100 + 7 * zoh_b + len(variant))
    kw = {}
    if variant == "no_softplus":
        kw = dict(softplus=False)
    elif variant == "no_gate_no_skip":
        kw = dict(gate=False, dskip=False)
    elif variant == "no_bias_no_h0":
        kw = dict(bias=False, h0=False)
    case = _rand_case(rng, **kw)
    if variant == "no_softplus":
        case["delta"] = np.abs(case["delta"]) + 0.05  # keep Delta positive
    out, last = _run(oracle_mod, case, zoh_b=zoh_b)
    ref_out, ref_last = _brute(case, zoh_b=zoh_b)
    _close(out, ref_out, 1e-12)
    _close(last, ref_last, 1e-12)


def test_brute_force_distinguishes_transposes(oracle_mod):
    """B and C swapped, or A read transposed, must be visible: the pins use
    dim != dstate != seqlen and asymmetric data."""
    rng = np.random.default_rng(5)
    case = _rand_case(rng, batch=1, L=7, dim=2, N=5)
    out, _ = _run(oracle_mod, case)
    swapped = dict(case, B=case["C"], C=case["B"])
    ref_swapped, _ = _brute(swapped)
    assert np.max(np.abs(out - ref_swapped)) > 1e-3


def test_n1_closed_form_constant_input(oracle_mod):
    """N=1, constant Delta, A, B, C, x, h0 = 0:
    h_t = Delta B x (1 - a^{t+1}) / (1 - a), a = exp(Delta A)."""
    L, dlt, a_c, b_c, c_c, x_c, d_c = 40, 0.37, -0.8, 1.3, 0.9, 0.6, 0.25
    u = np.full((1, L, 1), x_c)
    delta = np.full((1, L, 1), dlt)
    out, last = oracle_mod.scan(u, delta, np.array([[a_c]]), np.full((1, L, 1), b_c),
                                np.full((1, L, 1), c_c), D=np.array([d_c]), delta_softplus=False)
    a = math.exp(dlt * a_c)
    t = np.arange(L)
    h = dlt * b_c * x_c * (1 - a ** (t + 1)) / (1 - a)
    _close(out[0, :, 0], c_c * h + d_c * x_c, 1e-13)
    _close(last[0, 0, 0], h[-1], 1e-13)


def test_n1_closed_form_impulse(oracle_mod):
    """Impulse x_0 = 1: h_t = a^t Delta B."""
    L, dlt, a_c = 30, 0.21, -1.7
    u = np.zeros((1, L, 1)); u[0, 0, 0] = 1.0
    out, _ = oracle_mod.scan(u, np.full((1, L, 1), dlt), np.array([[a_c]]),
                             np.ones((1, L, 1)), np.ones((1, L, 1)), delta_softplus=False)
    a = math.exp(dlt * a_c)
    _close(out[0, :, 0], dlt * a ** np.arange(L), 1e-14)


@pytest.mark.parametrize("softplus", [False, True])
def test_lti_equals_convolution(oracle_mod, softplus):
    """With Delta, B, C constant in time the recurrence is the convolution
    y = x * K + D x, K_k = sum_n C_n exp(k Delta A_n) Delta B_n (NL-345
    section 2, eq. (3) and "Linear Time Invariance"); numpy.convolve is the
    independent route."""
    rng = np.random.default_rng(11)
    batch, L, dim, N = 2, 64, 3, 5
    A = -rng.uniform(0.1, 3.0, size=(dim, N))
    Bv, Cv = rng.standard_normal((batch, N)), rng.standard_normal((batch, N))
    draw = rng.uniform(-2.0, 0.5, size=(batch, dim))
    bias = rng.uniform(-0.5, 0.5, size=dim)
    D = rng.standard_normal(dim)
    u = rng.standard_normal((batch, L, dim))
    delta = np.repeat(draw[:, None, :], L, axis=1)
    B = np.repeat(Bv[:, None, :], L, axis=1)
    C = np.repeat(Cv[:, None, :], L, axis=1)
    out, _ = oracle_mod.scan(u, delta, A, B, C, D=D, delta_bias=bias, delta_softplus=softplus)
    k = np.arange(L)
    for b in range(batch):
        for d in range(dim):
            s = draw[b, d] + bias[d]
            dlt = np.logaddexp(0.0, s) if softplus else s
            K = sum(Cv[b, n] * np.exp(k * dlt * A[d, n]) * dlt * Bv[b, n] for n in range(N))
            ref = np.convolve(u[b, :, d], K)[:L] + D[d] * u[b, :, d]
            _close(out[b, :, d], ref, 1e-12)


def test_delta_zero_keeps_state_exactly(oracle_mod):
    """Delta = 0 (raw 0, no bias, softplus off): Abar = 1, Bbar = 0, so the state
    is kept bit for bit and y = C h0 + D u (NL-345 section 2 / the notes: Delta
    controls how much is remembered)."""
    rng = np.random.default_rng(3)
    batch, L, dim, N = 2, 20, 4, 6
    h0 = rng.standard_normal((batch, dim, N))
    u = rng.standard_normal((batch, L, dim))
    C = rng.standard_normal((batch, L, N))
    D = rng.standard_normal(dim)
    out, last = oracle_mod.scan(u, np.zeros((batch, L, dim)), -rng.uniform(0.5, 2, (dim, N)),
                                rng.standard_normal((batch, L, N)), C, D=D,
                                delta_softplus=False, h0=h0)
    assert np.array_equal(last, h0)
    ref = np.einsum("btn,bdn->btd", C, h0) + D[None, None, :] * u
    _close(out, ref, 1e-14)


@pytest.mark.parametrize("zoh_b", [False, True])
def test_split_and_resume_equals_one_pass(oracle_mod, zoh_b):
    """Running [0, k) then [k, L) from the returned state is one pass."""
    rng = np.random.default_rng(21)
    case = _rand_case(rng, batch=2, L=37, dim=5, N=3)
    full_out, full_last = _run(oracle_mod, case, zoh_b=zoh_b)
    for k in (1, 9, 36):
        first = {key: (v[:, :k] if isinstance(v, np.ndarray) and v.ndim == 3 and v.shape[1] == 37 else v)
                 for key, v in case.items()}
        second = {key: (v[:, k:] if isinstance(v, np.ndarray) and v.ndim == 3 and v.shape[1] == 37 else v)
                  for key, v in case.items()}
        o1, s1 = _run(oracle_mod, first, zoh_b=zoh_b)
        second["h0"] = s1
        o2, s2 = _run(oracle_mod, second, zoh_b=zoh_b)
        assert np.array_equal(np.concatenate([o1, o2], axis=1), full_out)
        assert np.array_equal(s2, full_last)


def test_theorem1_gated_rnn_under_zoh(oracle_mod):
    """N=1, A=-1, B=C=1, Delta = softplus(raw + bias): under exact ZOH the scan is
    h_t = (1 - g_t) h_{t-1} + g_t x_t with g_t = sigmoid(raw_t + bias)
    (【論文要約】Mamba notes, 数式解説 4, Theorem 1).  Under Euler it is not."""
    rng = np.random.default_rng(8)
    L, dim = 50, 3
    raw = rng.standard_normal((1, L, dim))
    bias = rng.standard_normal(dim)
    x = rng.standard_normal((1, L, dim))
    h0 = rng.standard_normal((1, dim, 1))
    args = (x, raw, -np.ones((dim, 1)), np.ones((1, L, 1)), np.ones((1, L, 1)))
    out_zoh, last_zoh = oracle_mod.scan(*args, delta_bias=bias, delta_softplus=True, h0=h0, zoh_b=True)
    out_eul, _ = oracle_mod.scan(*args, delta_bias=bias, delta_softplus=True, h0=h0, zoh_b=False)
    ref = np.zeros((L, dim))
    h = h0[0, :, 0].copy()
    for t in range(L):
        g = expit(raw[0, t] + bias)
        h = (1.0 - g) * h + g * x[0, t]
        ref[t] = h
    _close(out_zoh[0], ref, 1e-13)
    _close(last_zoh[0, :, 0], ref[-1], 1e-13)
    assert np.max(np.abs(out_eul[0] - ref)) > 1e-2


def test_softplus_and_bias_placement(oracle_mod):
    """N=1, A=0 (Abar = 1), B=C=u=1: y_t = sum_{s<=t} Delta_s with
    Delta_s = softplus(raw_s + bias) -- the bias goes inside tau_Delta
    (Algorithm 2).  np.logaddexp is the independent softplus, including
    arguments far outside the range where log(1 + e^s) is safe."""
    L = 64
    raw = np.linspace(-60.0, 60.0, L).reshape(1, L, 1)
    bias = np.array([0.75])
    out, _ = oracle_mod.scan(np.ones((1, L, 1)), raw, np.zeros((1, 1)), np.ones((1, L, 1)),
                             np.ones((1, L, 1)), delta_bias=bias, delta_softplus=True)
    ref = np.cumsum(np.logaddexp(0.0, raw[0, :, 0] + bias[0]))
    _close(out[0, :, 0] / (1 + ref), ref / (1 + ref), 1e-14)
    wrong = np.cumsum(np.logaddexp(0.0, raw[0, :, 0]) + bias[0])
    assert np.max(np.abs(out[0, :, 0] - wrong)) > 1e-3


def test_skip_and_gate(oracle_mod):
    """No input into the state (B = 0, h0 = 0): out = D u silu(z) with the
    library sigmoid; C = 0 leaves the same; D absent gives 0."""
    rng = np.random.default_rng(4)
    batch, L, dim, N = 2, 9, 3, 4
    u, z = rng.standard_normal((batch, L, dim)), rng.standard_normal((batch, L, dim)) * 3
    D = rng.standard_normal(dim)
    A = -rng.uniform(0.5, 2, (dim, N))
    zeros_bn = np.zeros((batch, L, N))
    out, _ = oracle_mod.scan(u, rng.standard_normal((batch, L, dim)), A, zeros_bn,
                             rng.standard_normal((batch, L, N)), D=D, z=z)
    _close(out, D * u * z * expit(z), 1e-15)
    out0, _ = oracle_mod.scan(u, rng.standard_normal((batch, L, dim)), A, zeros_bn, zeros_bn, z=z)
    assert np.array_equal(out0, np.zeros_like(out0))


def test_thread_count_and_channel_subset_invariance(oracle_mod):
    """Channels are independent (NL-345 section 2, "Structure and Dimensions"):
    any thread count, and any subset of channels, reproduces the same bits."""
    rng = np.random.default_rng(6)
    case = _rand_case(rng, batch=3, L=25, dim=7, N=4)
    o1, s1 = _run(oracle_mod, case, nthreads=1)
    o8, s8 = _run(oracle_mod, case, nthreads=8)
    assert np.array_equal(o1, o8) and np.array_equal(s1, s8)
    sel = [1, 4, 6]
    sub = dict(case)
    for key in ("u", "delta", "z"):
        sub[key] = case[key][:, :, sel]
    sub["A"], sub["D"], sub["delta_bias"] = case["A"][sel], case["D"][sel], case["delta_bias"][sel]
    sub["h0"] = case["h0"][:, sel]
    os_, ss = _run(oracle_mod, sub)
    assert np.array_equal(os_, o1[:, :, sel]) and np.array_equal(ss, s1[:, sel])


def test_decode_one_step_brute_force(oracle_mod):
    rng = np.random.default_rng(9)
    batch, dim, N = 3, 5, 4
    h = rng.standard_normal((batch, dim, N))
    x, dt, z = rng.standard_normal((batch, dim)), rng.uniform(0.01, 0.5, (batch, dim)), rng.standard_normal((batch, dim))
    A = -rng.uniform(0.5, 3, (dim, N))
    B, C, D = rng.standard_normal((batch, N)), rng.standard_normal((batch, N)), rng.standard_normal(dim)
    out, hn = oracle_mod.state_update(h, x, dt, A, B, C, D=D, z=z)
    for b in range(batch):
        for d in range(dim):
            newh = [math.exp(dt[b, d] * A[d, n]) * h[b, d, n] + dt[b, d] * B[b, n] * x[b, d] for n in range(N)]
            y = sum(C[b, n] * newh[n] for n in range(N)) + D[d] * x[b, d]
            y *= z[b, d] * expit(z[b, d])
            assert abs(out[b, d] - y) <= 1e-14 * (1 + abs(y))
            assert np.allclose(hn[b, d], newh, rtol=1e-15, atol=0)


def test_decode_steps_equal_scan(oracle_mod):
    """Recurrent mode (NL-345 section 1: constant time per step, no cache of
    past elements): 1000 decode steps equal one scan over the same 1000 steps,
    same Delta (softplus off, no bias), starting from the same state."""
    rng = np.random.default_rng(12)
    batch, dim, N, L = 2, 3, 4, 1000
    h0 = rng.standard_normal((batch, dim, N)) * 0.1
    x, z = rng.standard_normal((batch, L, dim)), rng.standard_normal((batch, L, dim))
    dt = np.logaddexp(0.0, rng.standard_normal((batch, L, dim)) * 0.5 - 4.0)
    B, C = rng.standard_normal((batch, L, N)), rng.standard_normal((batch, L, N))
    A = -np.tile(np.arange(1, N + 1, dtype=float), (dim, 1))
    D = rng.uniform(0.5, 1.5, dim)
    out_scan, last_scan = oracle_mod.scan(x, dt, A, B, C, D=D, z=z, delta_softplus=False, h0=h0)
    h = h0
    outs = []
    for t in range(L):
        o, h = oracle_mod.state_update(h, x[:, t], dt[:, t], A, B[:, t], C[:, t], D=D, z=z[:, t])
        outs.append(o)
    assert np.array_equal(np.stack(outs, axis=1), out_scan)
    assert np.array_equal(h, last_scan)


def test_empty_and_degenerate_shapes(oracle_mod):
    rng = np.random.default_rng(1)
    # seqlen 0: no output, state passes through
    h0 = rng.standard_normal((2, 3, 4))
    out, last = oracle_mod.scan(np.zeros((2, 0, 3)), np.zeros((2, 0, 3)), -np.ones((3, 4)),
                                np.zeros((2, 0, 4)), np.zeros((2, 0, 4)), h0=h0)
    assert out.shape == (2, 0, 3) and np.array_equal(last, h0)
    # dstate 0: y = D u silu(z)
    u, z = rng.standard_normal((1, 5, 2)), rng.standard_normal((1, 5, 2))
    out, last = oracle_mod.scan(u, rng.standard_normal((1, 5, 2)), np.zeros((2, 0)),
                                np.zeros((1, 5, 0)), np.zeros((1, 5, 0)), D=np.array([2.0, -1.0]), z=z)
    _close(out, np.array([2.0, -1.0]) * u * z * expit(z), 1e-15)


# ------------------------------------------------------------------ backward
def _bwd_case(seed, softplus=True, gate=True):
    rng = np.random.default_rng(seed)
    case = _rand_case(rng, batch=2, L=6, dim=3, N=3, softplus=softplus, gate=gate)
    if not softplus:
        case["delta"] = np.abs(case["delta"]) + 0.1
    dout = rng.standard_normal(case["u"].shape)
    return case, dout


_GRAD_OF = {"u": "du", "delta": "ddelta", "z": "dz", "A": "dA", "B": "dB", "C": "dC", "D": "dD",
            "delta_bias": "ddelta_bias", "h0": "dh0"}


def _loss(oracle_mod, case, dout):
    out, _ = _run(oracle_mod, case)
    return float(np.sum(out * dout))


@pytest.mark.parametrize("softplus", [True, False])
@pytest.mark.parametrize("gate", [True, False])
def test_bwd_matches_central_differences(oracle_mod, softplus, gate):
    """Every gradient of sum(dout * out) against central differences of the
    (separately pinned) forward oracle, eps = 1e-6."""
    case, dout = _bwd_case(60 + 2 * softplus + gate, softplus, gate)
    g = oracle_mod.scan_bwd(case["u"], case["delta"], case["A"], case["B"], case["C"], dout,
                            D=case["D"], z=case["z"], delta_bias=case["delta_bias"],
                            delta_softplus=softplus, h0=case["h0"])
    eps = 1e-6
    for name, gname in _GRAD_OF.items():
        if case[name] is None:
            continue
        base = case[name]
        for idx in np.ndindex(base.shape):
            plus, minus = dict(case), dict(case)
            plus[name] = base.copy(); plus[name][idx] += eps
            minus[name] = base.copy(); minus[name][idx] -= eps
            fd = (_loss(oracle_mod, plus, dout) - _loss(oracle_mod, minus, dout)) / (2 * eps)
            assert abs(fd - g[gname][idx]) <= 2e-7 * (1 + abs(fd)), (name, idx, fd, g[gname][idx])


def test_bwd_matches_torch_autograd(oracle_mod):
    """Gradients from torch autograd of an independent plain fp64 loop."""
    import torch
    case, dout = _bwd_case(70)
    t = {k: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for k, v in case.items() if isinstance(v, np.ndarray)}
    batch, L, dim = case["u"].shape
    N = case["A"].shape[1]
    outs = []
    for b in range(batch):
        h = t["h0"][b]                                            # (dim, N)
        rows = []
        for s in range(L):
            dlt = torch.nn.functional.softplus(t["delta"][b, s] + t["delta_bias"])   # (dim,)
            h = torch.exp(dlt[:, None] * t["A"]) * h + (dlt * t["u"][b, s])[:, None] * t["B"][b, s][None, :]
            y = h @ t["C"][b, s] + t["D"] * t["u"][b, s]
            rows.append(y * torch.nn.functional.silu(t["z"][b, s]))
        outs.append(torch.stack(rows))
    loss = (torch.stack(outs) * torch.tensor(dout)).sum()
    loss.backward()
    g = oracle_mod.scan_bwd(case["u"], case["delta"], case["A"], case["B"], case["C"], dout,
                            D=case["D"], z=case["z"], delta_bias=case["delta_bias"], h0=case["h0"])
    for name, gname in _GRAD_OF.items():
        _close(g[gname], t[name].grad.numpy(), 1e-12)


# ------------------------------------------------------------ complex A
def _complex_case(rng, batch=2, L=10, dim=3, N=4, softplus=True, gate=True, dskip=True, h0=True):
    c = _rand_case(rng, batch, L, dim, N, softplus=softplus, gate=gate, dskip=dskip, h0=h0)
    c["A"] = c["A"] + 1j * rng.uniform(-4.0, 4.0, size=(dim, N))
    c["B"] = c["B"] + 1j * rng.standard_normal((batch, L, N))
    c["C"] = c["C"] + 1j * rng.standard_normal((batch, L, N))
    if h0:
        c["h0"] = c["h0"] + 1j * rng.standard_normal((batch, dim, N))
    return c


@pytest.mark.parametrize("softplus", [True, False])
def test_complex_with_zero_imaginary_parts_is_the_real_scan(oracle_mod, softplus):
    # with every imaginary part 0 the complex recurrence is the real one, and
    # the arithmetic is the same operation for operation: bit-identical
    rng = np.random.default_rng(80 + softplus)
    c = _rand_case(rng, softplus=softplus)
    cc = dict(c, A=c["A"] + 0j, B=c["B"] + 0j, C=c["C"] + 0j, h0=c["h0"] + 0j)
    out_r, st_r = oracle_mod.scan(**c)
    out_c, st_c = oracle_mod.scan_complex(**cc)
    assert np.array_equal(out_r, out_c)
    assert np.array_equal(st_r, st_c.real) and not np.any(st_c.imag)


def test_complex_brute_force_unrolled_sum(oracle_mod):
    # y_t = Re(sum_n sum_{s<=t} C_t (prod_{r=s+1..t} e^{Delta_r A}) Delta_s B_s x_s
    #          + C_t (prod_{r<=t} e^{Delta_r A}) h0) + D x_t, then the gate;
    # explicit products with cmath (no running state)
    import cmath
    rng = np.random.default_rng(91)
    c = _complex_case(rng, L=8)
    u, delta, A, B, C = c["u"], c["delta"], c["A"], c["B"], c["C"]
    batch, L, dim = u.shape
    N = A.shape[1]
    out = np.zeros_like(u)
    for b in range(batch):
        for d in range(dim):
            dl = [math.log1p(math.exp(delta[b, t, d] + c["delta_bias"][d])) for t in range(L)]
            for t in range(L):
                acc = 0j
                for n in range(N):
                    def prod(lo, hi):
                        p = 1 + 0j
                        for r in range(lo, hi + 1):
                            p *= cmath.exp(dl[r] * A[d, n])
                        return p
                    h = prod(0, t) * c["h0"][b, d, n]
                    for s in range(t + 1):
                        h += prod(s + 1, t) * dl[s] * B[b, s, n] * u[b, s, d]
                    acc += C[b, t, n] * h
                y = acc.real + c["D"][d] * u[b, t, d]
                out[b, t, d] = y * c["z"][b, t, d] * expit(c["z"][b, t, d])
    got, _ = oracle_mod.scan_complex(**c)
    np.testing.assert_allclose(got, out, rtol=1e-11, atol=1e-11)


def test_complex_lti_equals_convolution(oracle_mod):
    # constant Delta, B, C: y = x * K + D x with the complex kernel
    # K_k = Re(sum_n C_n e^{k Delta A_n} Delta B_n)  (NL-345 eq. (3), complex A)
    rng = np.random.default_rng(92)
    L, dim, N, dl = 40, 2, 5, 0.3
    A = -rng.uniform(0.1, 1.0, size=(dim, N)) + 1j * rng.uniform(-3, 3, size=(dim, N))
    Bv = rng.standard_normal(N) + 1j * rng.standard_normal(N)
    Cv = rng.standard_normal(N) + 1j * rng.standard_normal(N)
    u = rng.standard_normal((1, L, dim))
    D = rng.standard_normal(dim)
    out, _ = oracle_mod.scan_complex(u, np.full((1, L, dim), dl), A, np.broadcast_to(Bv, (1, L, N)),
                                     np.broadcast_to(Cv, (1, L, N)), D=D, delta_softplus=False)
    for d in range(dim):
        k = np.arange(L)
        K = np.real((Cv[None, :] * np.exp(np.outer(k, dl * A[d])) * dl * Bv[None, :]).sum(axis=1))
        ref = np.convolve(u[0, :, d], K)[:L] + D[d] * u[0, :, d]
        np.testing.assert_allclose(out[0, :, d], ref, rtol=1e-11, atol=1e-12)


def test_complex_pure_rotation_closed_form(oracle_mod):
    # A = i w (no decay), constant Delta, an impulse at t = 0, B = 1, h0 = 0:
    # h_t = Delta e^{i w Delta t}; C = 1 reads Delta cos(w Delta t), C = i reads
    # -Delta sin(w Delta t) (the sign of the phase)
    L, dl, w = 25, 0.2, 1.7
    u = np.zeros((1, L, 1))
    u[0, 0, 0] = 1.0
    A = np.array([[1j * w]])
    Bm = np.ones((1, L, 1), dtype=complex)
    t = np.arange(L)
    for Cval, ref in [(1.0, dl * np.cos(w * dl * t)), (1j, -dl * np.sin(w * dl * t))]:
        out, st = oracle_mod.scan_complex(u, np.full((1, L, 1), dl), A, Bm, np.full((1, L, 1), Cval),
                                          delta_softplus=False)
        np.testing.assert_allclose(out[0, :, 0], ref, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(st[0, 0, 0], dl * np.exp(1j * w * dl * (L - 1)), rtol=1e-12)


# ------------------------------------------------------------------ Mamba-2 SSD
# "Transformers are SSMs" review (nubint.ai), 提案手法: the SSM as a matrix
# transformation (a semiseparable matrix), its linear (recurrent) and
# quadratic (attention-like) forms computing the same map, and the block
# decomposition of that matrix behind the SSD algorithm.  The oracle's
# ssd_scan is the linear form; these pins compare it with the selective-scan
# oracle (scalar A per head is a diagonal A with equal entries), with the
# quadratic form written as a masked matrix product, and with the chunked
# block decomposition, each computed here in numpy.

def _ssd_case(rng, batch=2, L=13, H=4, P=3, G=2, N=5, softplus=True, bias=True, gate=True, dskip=True,
              h0=True):
    return dict(
        x=rng.standard_normal((batch, L, H, P)),
        dt=rng.standard_normal((batch, L, H)) * 0.7,
        A=-rng.uniform(0.2, 2.0, size=H),
        B=rng.standard_normal((batch, L, G, N)),
        C=rng.standard_normal((batch, L, G, N)),
        D=rng.standard_normal(H) if dskip else None,
        z=rng.standard_normal((batch, L, H, P)) if gate else None,
        dt_bias=rng.standard_normal(H) * 0.5 if bias else None,
        dt_softplus=softplus,
        h0=rng.standard_normal((batch, H, P, N)) if h0 else None)


def _ssd_delta(c):
    s = c["dt"] + (c["dt_bias"] if c["dt_bias"] is not None else 0.0)
    return np.logaddexp(0.0, s) if c["dt_softplus"] else s


def _ssd_epilogue(c, y):
    H = c["x"].shape[2]
    if c["D"] is not None:
        y = y + c["D"].reshape(1, 1, H, 1) * c["x"]
    if c["z"] is not None:
        y = y * c["z"] * expit(c["z"])
    return y


def _ssd_quadratic(c):
    """Quadratic (masked attention) form: per (b, h), with Delta's running sum
    S_t = sum_{r<=t} Delta_r, y = (Lmask o (C B^T)) diag(Delta) X + C_t
    e^{A S_t} h0, Lmask[t, s] = e^{A (S_t - S_s)} for s <= t, else 0."""
    x, A, B, C = c["x"], c["A"], c["B"], c["C"]
    batch, L, H, P = x.shape
    G = B.shape[2]
    dl = _ssd_delta(c)
    y = np.zeros_like(x)
    last = np.zeros((batch, H, P, B.shape[3]))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            S = np.cumsum(dl[b, :, h])
            mask = np.tril(np.exp(A[h] * (S[:, None] - S[None, :])))
            M = mask * (C[b, :, g] @ B[b, :, g].T) * dl[b, None, :, h]
            y[b, :, h] = M @ x[b, :, h]
            wlast = np.exp(A[h] * (S[-1] - S)) * dl[b, :, h]
            last[b, h] = (x[b, :, h] * wlast[:, None]).T @ B[b, :, g]
            if c["h0"] is not None:
                decay = np.exp(A[h] * S)
                y[b, :, h] += decay[:, None] * (C[b, :, g] @ c["h0"][b, h].T)
                last[b, h] += np.exp(A[h] * S[-1]) * c["h0"][b, h]
    return _ssd_epilogue(c, y), last


def _ssd_chunked(c, Q):
    """Block decomposition at chunk length Q: diagonal blocks by the quadratic
    form inside each chunk, off-diagonal blocks through the chunk-boundary
    states, which pass from chunk to chunk with the chunk's total decay."""
    x, A, B, C = c["x"], c["A"], c["B"], c["C"]
    batch, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    dl = _ssd_delta(c)
    y = np.zeros_like(x)
    last = np.zeros((batch, H, P, N))
    for b in range(batch):
        for h in range(H):
            g = h // (H // G)
            st = c["h0"][b, h].copy() if c["h0"] is not None else np.zeros((P, N))
            for t0 in range(0, L, Q):
                sl = slice(t0, min(L, t0 + Q))
                d, xx, Bc, Cc = dl[b, sl, h], x[b, sl, h], B[b, sl, g], C[b, sl, g]
                S = np.cumsum(d)
                mask = np.tril(np.exp(A[h] * (S[:, None] - S[None, :])))
                y[b, sl, h] = (mask * (Cc @ Bc.T) * d[None, :]) @ xx          # diagonal block
                y[b, sl, h] += np.exp(A[h] * S)[:, None] * (Cc @ st.T)         # from the carried state
                w = np.exp(A[h] * (S[-1] - S)) * d
                st = np.exp(A[h] * S[-1]) * st + (xx * w[:, None]).T @ Bc      # state at the chunk's end
            last[b, h] = st
    return _ssd_epilogue(c, y), last


def test_ssd_is_the_selective_scan_with_scalar_A_per_head(oracle_mod):
    rng = np.random.default_rng(40)
    c = _ssd_case(rng)
    out, last = oracle_mod.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                                    dt_bias=c["dt_bias"], dt_softplus=c["dt_softplus"], h0=c["h0"])
    batch, L, H, P = c["x"].shape
    G, N = c["B"].shape[2:]
    hpg = H // G
    for g in range(G):
        hs = slice(g * hpg, (g + 1) * hpg)
        ch = hpg * P
        rep = lambda a: np.repeat(a[hs], P)  # one value per channel (h, p) of the group
        o, s = oracle_mod.scan(c["x"][:, :, hs].reshape(batch, L, ch),
                               np.repeat(c["dt"][:, :, hs], P, axis=2), np.repeat(rep(c["A"])[:, None], N, 1),
                               c["B"][:, :, g], c["C"][:, :, g], D=rep(c["D"]),
                               z=c["z"][:, :, hs].reshape(batch, L, ch), delta_bias=rep(c["dt_bias"]),
                               delta_softplus=c["dt_softplus"], h0=c["h0"][:, hs].reshape(batch, ch, N))
        np.testing.assert_array_equal(out[:, :, hs].reshape(batch, L, ch), o)
        np.testing.assert_array_equal(last[:, hs].reshape(batch, ch, N), s)


@pytest.mark.parametrize("variant", ["full", "no_softplus", "no_gate_no_skip", "no_bias_no_h0"])
def test_ssd_equals_quadratic_form(oracle_mod, variant):
    rng = np.random.default_rng(41)
    kw = dict(full={}, no_softplus=dict(softplus=False), no_gate_no_skip=dict(gate=False, dskip=False),
              no_bias_no_h0=dict(bias=False, h0=False))[variant]
    c = _ssd_case(rng, **kw)
    if not c["dt_softplus"]:
        c["dt"] = np.abs(c["dt"])  # a positive step keeps the decays bounded
    out, last = oracle_mod.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                                    dt_bias=c["dt_bias"], dt_softplus=c["dt_softplus"], h0=c["h0"])
    ro, rl = _ssd_quadratic(c)
    np.testing.assert_allclose(out, ro, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(last, rl, rtol=1e-10, atol=1e-11)


@pytest.mark.parametrize("Q", [1, 3, 7, 64])
def test_ssd_equals_chunked_block_decomposition(oracle_mod, Q):
    rng = np.random.default_rng(42)
    c = _ssd_case(rng, L=23, H=4, P=2, G=1, N=6)
    out, last = oracle_mod.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], z=c["z"],
                                    dt_bias=c["dt_bias"], dt_softplus=c["dt_softplus"], h0=c["h0"])
    ro, rl = _ssd_chunked(c, Q)
    np.testing.assert_allclose(out, ro, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(last, rl, rtol=1e-10, atol=1e-11)


def test_ssd_delta_zero_keeps_state_exactly(oracle_mod):
    rng = np.random.default_rng(43)
    c = _ssd_case(rng, bias=False, softplus=False, gate=False)
    c["dt"][:] = 0.0
    out, last = oracle_mod.ssd_scan(c["x"], c["dt"], c["A"], c["B"], c["C"], D=c["D"], z=None,
                                    dt_bias=None, dt_softplus=False, h0=c["h0"])
    np.testing.assert_array_equal(last, c["h0"])
    H = c["x"].shape[2]
    G = c["B"].shape[2]
    for h in range(H):
        g = h // (H // G)
        ref = np.einsum("btn,bpn->btp", c["C"][:, :, g], c["h0"][:, h]) + c["D"][h] * c["x"][:, :, h]
        np.testing.assert_allclose(out[:, :, h], ref, rtol=1e-13, atol=1e-13)


def test_ssd_split_and_resume_equals_one_pass(oracle_mod):
    rng = np.random.default_rng(44)
    c = _ssd_case(rng, L=17)
    args = lambda sl, h0: (c["x"][:, sl], c["dt"][:, sl], c["A"], c["B"][:, sl], c["C"][:, sl])
    kw = lambda sl: dict(D=c["D"], z=c["z"][:, sl], dt_bias=c["dt_bias"], dt_softplus=True)
    out, last = oracle_mod.ssd_scan(*args(slice(None), None), h0=c["h0"], **kw(slice(None)))
    o1, s1 = oracle_mod.ssd_scan(*args(slice(0, 6), None), h0=c["h0"], **kw(slice(0, 6)))
    o2, s2 = oracle_mod.ssd_scan(*args(slice(6, None), None), h0=s1, **kw(slice(6, None)))
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=1), out)
    np.testing.assert_array_equal(s2, last)
