"""The oracle's pins have teeth: each plausible slip, planted in a copy of the
oracle's C source and compiled on the CPU, must fail at least one pin.

The planted slips are the ones the pins are meant to exclude: reading y before
the state update, a dropped skip term, the bias outside softplus, B and C
swapped, A read transposed, a flipped sign in the decay, a wrong softplus, a
sigmoid in place of silu, a wrong ZOH factor, a dropped input, an off-by-one in
time, a missing state write-back, a decode step without Delta on B.
"""
import inspect

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    "readout_before_update": (
        "h[n] = abar * h[n] + bbar * x;\n                acc += j->C[tn + n] * h[n];",
        "acc += j->C[tn + n] * h[n];\n                h[n] = abar * h[n] + bbar * x;"),
    "dropped_skip": ("(j->Dskip ? j->Dskip[d] * x : 0.0)", "0.0"),
    "bias_outside_softplus": (
        "double s = j->delta[td] + (j->bias ? j->bias[d] : 0.0);\n"
        "            const double dlt = j->softplus ? oracle_softplus(s) : s;",
        "double s = j->delta[td];\n"
        "            const double dlt = (j->softplus ? oracle_softplus(s) : s) + (j->bias ? j->bias[d] : 0.0);"),
    "B_C_swapped": ("acc += j->C[tn + n] * h[n];", "acc += j->B[tn + n] * h[n];"),
    "A_transposed": ("const double an = j->A[d * N + n];", "const double an = j->A[n * Dm + d];"),
    "decay_sign": ("const double abar = exp(dlt * an);\n                double bbar;",
                   "const double abar = exp(-dlt * an);\n                double bbar;"),
    "softplus_without_max": ("return m + log1p(exp(-fabs(s)));", "return log1p(exp(-fabs(s)));"),
    "sigmoid_gate": ("return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    "zoh_factor": ("expm1(dlt * an) / an", "expm1(dlt * an) / (dlt * an)"),
    "dropped_input": ("h[n] = abar * h[n] + bbar * x;", "h[n] = abar * h[n] + bbar;"),
    "time_off_by_one": ("const double x = j->u[td];",
                        "const double x = j->u[(b * L + (t > 0 ? t - 1 : 0)) * Dm + d];"),
    "state_not_written": ("j->state[(b * Dm + d) * N + n] = h[n];", "(void)0;"),
    "decode_without_dt": ("h[n] = abar * h[n] + dlt * B[b * dstate + n] * xv;",
                          "h[n] = abar * h[n] + B[b * dstate + n] * xv;"),
    "h0_ignored": ("h[n] = j->state ? j->state[(b * Dm + d) * N + n] : 0.0;", "h[n] = 0.0;"),
    # complex A
    "complex_conjugate_phase": ("cexp(dlt * an)", "cexp(dlt * conj(an))"),
    "complex_readout_imaginary": ("double y = creal(acc) +", "double y = cimag(acc) +"),
    "complex_B_real_part_only": ("h[n] = abar * h[n] + (dlt * bn) * x;", "h[n] = abar * h[n] + (dlt * creal(bn)) * x;"),
    "complex_h0_imaginary_dropped": ("h[n] = state ? state[2 * (so + n)] + I * state[2 * (so + n) + 1] : 0.0;",
                                     "h[n] = state ? state[2 * (so + n)] : 0.0;"),
    # Mamba-2 SSD
    "ssd_group_index": ("const int64_t g = hd / hpg;", "const int64_t g = hd % groups;"),
    "ssd_input_without_delta": ("h[n] = abar * h[n] + dlt * B[bi + n] * xv;", "h[n] = abar * h[n] + B[bi + n] * xv;"),
    "ssd_decay_after_input": ("h[n] = abar * h[n] + dlt * B[bi + n] * xv;", "h[n] = abar * (h[n] + dlt * B[bi + n] * xv);"),
    "ssd_readout_with_B": ("acc += C[bi + n] * h[n];", "acc += B[bi + n] * h[n];"),
    "ssd_state_transposed": ("double *st = state ? state + ((b * H + hd) * P + p) * N : NULL;",
                             "double *st = state ? state + (b * H + hd) * P * N + p : NULL;"),
    "ssd_bias_ignored": ("const double s = dt[(b * L + t) * H + hd] + (dt_bias ? dt_bias[hd] : 0.0);",
                         "const double s = dt[(b * L + t) * H + hd];"),
    # backward
    "bwd_adjoint_not_decayed": ("lam[n] *= abar;", "(void)0;"),
    "bwd_dA_without_decay": ("dA[d * N + n] += lam[n] * hprev * abar * dl[t];",
                             "dA[d * N + n] += lam[n] * hprev * dl[t];"),
    "bwd_dC_with_previous_state": ("dC[tn + n] += dy * hs[(t + 1) * N + n];", "dC[tn + n] += dy * hprev;"),
    "bwd_silu_derivative": ("dz[td] = dout[td] * yv[t] * sg * (1.0 + z[td] * (1.0 - sg));",
                            "dz[td] = dout[td] * yv[t] * sg;"),
    "bwd_softplus_derivative": ("const double dd = delta_softplus ? ddl / (1.0 + exp(-sv)) : ddl;",
                                "const double dd = ddl;"),
}


def _pin_calls():
    """Every pin test in test_oracle_pins, expanded over its parameters."""
    calls = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = list(inspect.signature(fn).parameters)
        marks = getattr(fn, "pytestmark", [])
        grid = [{}]
        for m in marks:
            if m.name == "parametrize":
                argnames = [a.strip() for a in m.args[0].split(",")]
                grid = [dict(g, **dict(zip(argnames, v if len(argnames) > 1 else (v,))))
                        for g in grid for v in m.args[1]]
        for g in grid:
            calls.append((name, fn, g, params))
    return calls


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_planted_mistake_is_caught(mutant, tmp_path):
    src = oracle.source()
    old, new = MUTANTS[mutant]
    assert src.count(old) == 1, f"mutation anchor for {mutant} not found exactly once"
    variant = oracle.compile_variant(src.replace(old, new), str(tmp_path / f"lib_{mutant}.so"))
    caught = []
    for name, fn, kw, params in _pin_calls():
        try:
            with np.errstate(all="ignore"):
                fn(variant, **kw)
        except Exception:
            caught.append(name)
    assert caught, f"no pin catches the planted mistake {mutant!r}"


def test_unmodified_copy_passes_every_pin(tmp_path):
    """Control: the harness itself raises nothing on the real source, so every
    failure counted above comes from the planted slip."""
    variant = oracle.compile_variant(oracle.source(), str(tmp_path / "lib_control.so"))
    failed = []
    for name, fn, kw, params in _pin_calls():
        try:
            with np.errstate(all="ignore"):
                fn(variant, **kw)
        except Exception as e:  # pragma: no cover - reported below
            failed.append(f"{name}{kw}: {e!r}")
    assert not failed, failed
    assert len(_pin_calls()) >= 20
