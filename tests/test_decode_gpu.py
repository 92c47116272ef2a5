"""GPU parity of ssm_selective_state_update (one-token decode) against the
fp64 oracle, including the full decode workload (batch 256, dim 5120, N 16,
1000 steps) compared on a grid of sampled channels at every step."""
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


def _oracle_step(h, st, A, D, io):
    return T.oracle.state_update(h, T.f64(st["x"], io), T.f64(st["dt"], io), A, T.f64(st["B"], io),
                                 T.f64(st["C"], io), D=D, z=T.f64(st["z"], io))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 4, 8, 13, 16, 24, 32, 64])
@pytest.mark.parametrize("dim", [77, 80])
def test_decode_steps_small(lib, io, N, dim):
    # dim 77: per-slice loads; dim 80 (rows of a multiple of 16 bytes): the
    # bulk-copy kernel for N = 4 (fp32), 8, 16, 32, 64, with a partial unit
    cfg = I.DecodeConfig("d", 3, dim, N, steps=20, io=io, seed=N + dim)
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    state = torch.from_numpy(h0).cuda()
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    h = h0.astype(np.float64)
    for k in range(cfg.steps):
        st = I.decode_step_inputs(cfg, k, bias)
        out = lib.selective_state_update(state, T.to_dev(st["x"], io), T.to_dev(st["dt"], io), Ad,
                                         T.to_dev(st["B"], io), T.to_dev(st["C"], io), D=Dd,
                                         z=T.to_dev(st["z"], io))
        ref, h = _oracle_step(h, st, A.astype(np.float64), D.astype(np.float64), io)
        T.check_out(T.from_dev(out), ref, io)
    T.check_state(T.from_dev(state), h, io)


def test_decode_without_gate_and_skip(lib):
    cfg = I.DecodeConfig("d", 2, 40, 16, steps=3, io="bf16", seed=1, has_z=False)
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    state = torch.from_numpy(h0).cuda()
    st = I.decode_step_inputs(cfg, 0, bias)
    out = lib.selective_state_update(state, T.to_dev(st["x"], "bf16"), T.to_dev(st["dt"], "bf16"),
                                     torch.from_numpy(A).cuda(), T.to_dev(st["B"], "bf16"),
                                     T.to_dev(st["C"], "bf16"))
    ref, h = T.oracle.state_update(h0, T.f64(st["x"], "bf16"), T.f64(st["dt"], "bf16"), A,
                                   T.f64(st["B"], "bf16"), T.f64(st["C"], "bf16"))
    T.check_out(T.from_dev(out), ref, "bf16")
    T.check_state(T.from_dev(state), h, "bf16")


def test_decode_steps_match_gpu_scan(lib):
    """Recurrent mode equals the scan: L decode steps (Delta given) equal one
    scan over the same L steps with softplus off and no bias."""
    io = "bf16"
    cfg = I.DecodeConfig("d", 2, 96, 16, steps=300, io=io, seed=3)
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    steps = [I.decode_step_inputs(cfg, k, bias) for k in range(cfg.steps)]
    stack = lambda key: np.stack([s[key] for s in steps], axis=1)
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    state = torch.from_numpy(h0).cuda()
    outs = []
    for s in steps:
        outs.append(lib.selective_state_update(state, T.to_dev(s["x"], io), T.to_dev(s["dt"], io), Ad,
                                               T.to_dev(s["B"], io), T.to_dev(s["C"], io), D=Dd,
                                               z=T.to_dev(s["z"], io)))
    dec = torch.stack(outs, dim=1)
    st2 = torch.from_numpy(h0).cuda()
    scan = lib.selective_scan_fwd(T.to_dev(stack("x"), io), T.to_dev(stack("dt"), io), Ad,
                                  T.to_dev(stack("B"), io), T.to_dev(stack("C"), io), D=Dd,
                                  z=T.to_dev(stack("z"), io), delta_softplus=False, last_state=st2)
    torch.cuda.synchronize()
    T.check_out(T.from_dev(dec), T.from_dev(scan), io)
    T.check_state(T.from_dev(state), T.from_dev(st2), io)


@pytest.mark.slow
def test_decode_workload_full_size(lib):
    """batch 256, dim 5120, N 16, 1000 fresh steps: every step's output and the
    state on 8 batch rows x 64 channels against the oracle run on exactly those
    channels; the final state on the same grid."""
    cfg = I.DECODE
    io = cfg.io
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    rng = np.random.default_rng(0)
    bsel = np.unique(np.concatenate([[0, cfg.batch - 1], rng.choice(cfg.batch, 6, replace=False)]))
    dsel = np.unique(np.concatenate([[0, 31, 32, cfg.dim - 1], rng.choice(cfg.dim, 60, replace=False)]))
    bt, dt_ = torch.as_tensor(bsel, device="cuda"), torch.as_tensor(dsel, device="cuda")
    state = torch.from_numpy(h0).cuda()
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    h = h0[bsel][:, dsel].astype(np.float64)
    As, Ds = A[dsel].astype(np.float64), D[dsel].astype(np.float64)
    worst = 0.0
    for k in range(cfg.steps):
        st = I.decode_step_inputs(cfg, k, bias)
        out = lib.selective_state_update(state, T.to_dev(st["x"], io), T.to_dev(st["dt"], io), Ad,
                                         T.to_dev(st["B"], io), T.to_dev(st["C"], io), D=Dd,
                                         z=T.to_dev(st["z"], io))
        sub = {"x": st["x"][bsel][:, dsel], "dt": st["dt"][bsel][:, dsel], "z": st["z"][bsel][:, dsel],
               "B": st["B"][bsel], "C": st["C"][bsel]}
        ref, h = _oracle_step(h, sub, As, Ds, io)
        worst = max(worst, T.check_out(T.from_dev(out[bt][:, dt_]), ref, io))
    T.check_state(T.from_dev(state[bt][:, dt_]), h, io)


@pytest.mark.parametrize("io", ["f32", "bf16"])
def test_decode_bulk_ring_wraps(lib, io):
    # 3072 units of 16 KB (6 per batch row, the last one 24 channels wide):
    # seven per CTA, so every buffer of the copy ring is reused and its
    # barrier changes phase
    cfg = I.DecodeConfig("d", 512, 1304, 16, steps=3, io=io, seed=5)
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    state = torch.from_numpy(h0).cuda()
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    h = h0.astype(np.float64)
    for k in range(cfg.steps):
        st = I.decode_step_inputs(cfg, k, bias)
        out = lib.selective_state_update(state, T.to_dev(st["x"], io), T.to_dev(st["dt"], io), Ad,
                                         T.to_dev(st["B"], io), T.to_dev(st["C"], io), D=Dd,
                                         z=T.to_dev(st["z"], io))
        ref, h = _oracle_step(h, st, A.astype(np.float64), D.astype(np.float64), io)
        T.check_out(T.from_dev(out), ref, io)
    T.check_state(T.from_dev(state), h, io)
    assert lib.device_status() == 0


def test_decode_bounded_wait_sets_device_status(lib):
    # every wait of the state copies runs out (the test hook asks each unit's
    # barrier for 16 bytes that never come): the kernel gives up after its
    # time limit, reports bit 0 and the context stays usable
    cfg = I.DecodeConfig("d", 2, 304, 16, steps=1, io="bf16", seed=6)
    A, D, bias = I.decode_params(cfg)
    h0 = I.decode_h0(cfg)
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    st = I.decode_step_inputs(cfg, 0, bias)
    args = [T.to_dev(st["x"], "bf16"), T.to_dev(st["dt"], "bf16"), Ad, T.to_dev(st["B"], "bf16"),
            T.to_dev(st["C"], "bf16")]
    assert lib.device_status() == 0
    lib.lib.ssm_test_inject_decode_wait_timeout(1)
    try:
        lib.selective_state_update(torch.from_numpy(h0).cuda(), *args, D=Dd, z=T.to_dev(st["z"], "bf16"))
        assert lib.device_status() & 1
    finally:
        lib.lib.ssm_test_inject_decode_wait_timeout(0)
    assert lib.device_status() == 0
    state = torch.from_numpy(h0).cuda()
    out = lib.selective_state_update(state, *args, D=Dd, z=T.to_dev(st["z"], "bf16"))
    ref, h = _oracle_step(h0.astype(np.float64), st, A.astype(np.float64), D.astype(np.float64), "bf16")
    T.check_out(T.from_dev(out), ref, "bf16")
    T.check_state(T.from_dev(state), h, "bf16")
    assert lib.device_status() == 0


def test_decode_sees_the_writes_of_the_kernel_before_it(lib):
    # The decode step is launched as a programmatic dependent of the stream's
    # previous kernel, so its launch overlaps that kernel's end.  Here each
    # step's state and x are written by a device kernel right before the
    # step (alternating between two different sources); a step that read
    # either before that kernel finished would see the previous step's
    # values and miss the oracle.
    cfg = I.DecodeConfig("d", 64, 2048, 16, steps=8, io="bf16", seed=21)
    A, D, bias = I.decode_params(cfg)
    Ad, Dd = torch.from_numpy(A).cuda(), torch.from_numpy(D).cuda()
    rng = np.random.default_rng(7)
    srcs = [rng.standard_normal((cfg.batch, cfg.dim, cfg.dstate)).astype(np.float32) for _ in range(2)]
    srcs_dev = [torch.from_numpy(s).cuda() for s in srcs]
    state = torch.empty_like(srcs_dev[0])
    x_dev = torch.empty((cfg.batch, cfg.dim), dtype=torch.bfloat16, device="cuda")
    for k in range(cfg.steps):
        st = I.decode_step_inputs(cfg, k, bias)
        x_src = T.to_dev(st["x"], "bf16")
        rest = {n: T.to_dev(st[n], "bf16") for n in ("dt", "B", "C", "z")}
        torch.cuda.synchronize()
        torch.mul(srcs_dev[k % 2], 1.0, out=state)  # kernels writing the step's inputs
        torch.mul(x_src, 1, out=x_dev)
        out = lib.selective_state_update(state, x_dev, rest["dt"], Ad, rest["B"], rest["C"], D=Dd, z=rest["z"])
        ref, h = _oracle_step(srcs[k % 2].astype(np.float64), st, A.astype(np.float64), D.astype(np.float64),
                              "bf16")
        T.check_out(T.from_dev(out), ref, "bf16", what=f"step {k}")
        T.check_state(T.from_dev(state), h, "bf16", what=f"step {k}")
    assert lib.device_status() == 0
