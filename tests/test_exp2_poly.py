"""The fast scan tier's FMA-pipe exp2 (exp2_poly2 in csrc/ssm_device.cuh):
Cody-Waite reduction x = r + f (r = round(x) by the 1.5 * 2^23 addition,
f in [-1/2, 1/2]), a degree-5 polynomial for 2^f, the exponent inserted with a
shift-add, x clamped to [-125, 127].

Bound: relative error <= 2^-22 against exp2 in fp64 -- the 2-ulp accuracy of
CUDA's exp2f and within a factor of ~1.4 of the SFU's ex2.approx (both are
checked on the GPU side by side).  The CPU test emulates the fp32 evaluation
step by step (each add/fma rounded to fp32) with the coefficients read from
the CUDA source; the GPU test runs the device function itself through the
library's test hook.
"""
import os
import re

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "selective_state_space_36_b200", "csrc", "ssm_device.cuh")
BOUND = 2.0 ** -22


def _coefs():
    text = open(SRC).read()
    m = re.search(r"#define SSM_EXP2_C \{([^}]*)\}", text)
    return [np.float32(float(v.strip().rstrip("f"))) for v in m.group(1).replace("\\", "").split(",")]


def _fma32(a, b, c):
    # exact product in fp64 (24 + 24 bits), one rounding of the sum to fp32
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def poly_exp2_f32(x):
    x = np.clip(np.asarray(x, np.float32), np.float32(-125.0), np.float32(127.0))
    k = np.float32(12582912.0)
    t = (x + k).astype(np.float32)
    f = (x - (t - k).astype(np.float32)).astype(np.float32)
    c = _coefs()
    p = np.full_like(f, c[4])
    for ci in (c[3], c[2], c[1], c[0], np.float32(1.0)):
        p = _fma32(p, f, np.full_like(f, ci))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def _grid():
    rng = np.random.default_rng(0)
    return np.concatenate([np.linspace(-125.0, 127.0, 400001, dtype=np.float32),
                           rng.uniform(-20.0, 0.0, 400000).astype(np.float32),   # the decays' range
                           rng.uniform(-1e-3, 1e-3, 100000).astype(np.float32),
                           np.arange(-125, 128, dtype=np.float32)])


def test_exp2_poly_cpu_emulation_within_bound():
    x = _grid()
    y = poly_exp2_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    err = np.max(np.abs(y / ref - 1.0))
    assert err <= BOUND, f"max relative error {err:.3e} > 2^-22"


def test_exp2_poly_special_values():
    ints = np.arange(-125, 128, dtype=np.float32)
    np.testing.assert_array_equal(poly_exp2_f32(ints), np.exp2(ints.astype(np.float64)).astype(np.float32))
    assert poly_exp2_f32(np.float32([0.0]))[0] == 1.0  # Delta = 0: decay exactly 1, the state is kept
    lo = poly_exp2_f32(np.float32([-126.0, -1000.0, -np.inf]))
    assert np.all(lo == np.float32(2.0 ** -125))      # clamped: negligible next to any input term
    hi = poly_exp2_f32(np.float32([128.0, 1e6]))
    assert np.all(hi == np.float32(2.0 ** 127))


@pytest.mark.gpu
def test_exp2_poly_on_the_gpu():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from selective_state_space_36_b200 import binding
    x = _grid()
    poly, sfu = binding.test_exp2_poly(torch.from_numpy(x).cuda())
    torch.cuda.synchronize()
    poly, sfu = poly.cpu().numpy().astype(np.float64), sfu.cpu().numpy().astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    e_poly = np.max(np.abs(poly / ref - 1.0))
    mask = x > -126  # ex2.approx.ftz flushes results below 2^-126
    e_sfu = np.max(np.abs(sfu[mask] / ref[mask] - 1.0))
    print(f"[exp2] FMA-pipe polynomial max rel err {e_poly:.3e}; SFU ex2.approx {e_sfu:.3e}")
    assert e_poly <= BOUND
    # the device evaluation is the emulated one (up to one fp32 ulp of rounding order)
    emu = poly_exp2_f32(x).astype(np.float64)
    assert np.max(np.abs(poly - emu) / ref) <= 2.0 ** -23
