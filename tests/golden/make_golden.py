"""Writes tests/golden/tiny_f32_oracle.json: sampled oracle outputs of the
tiny fp32 workload (batch 1, L 256, D 64, N 16, seed 0).

The pages print no worked numeric example of the selective scan, so the
golden values here are the oracle's own, frozen once its pins passed: a
regression anchor, so that any later change to the oracle's arithmetic shows
up.  Calls only the oracle and the seeded input generator.

Equations followed: NL-345, Mamba: Linear-Time Sequence Modeling with
Selective State Spaces, section 2 eq. (2) (recurrence, readout after the
update) with Abar = exp(Delta A) ("Discretization"); Bbar = Delta B (Euler);
Delta = softplus(raw + bias) (【論文要約】Mamba notes, S6 Algorithm 2);
out = (y + D u) silu(z).
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from selective_state_space_36_b200 import inputs as I  # noqa: E402

SAMPLES = [(0, 0, 0), (0, 0, 63), (0, 1, 5), (0, 17, 31), (0, 128, 2), (0, 200, 40),
           (0, 254, 62), (0, 255, 0), (0, 255, 63)]


def compute():
    x = I.scan_inputs(I.TINY_F32)
    f = lambda k: I.to_f64(x[k], "f32")
    out, last = oracle.scan(f("u"), f("delta"), f("A"), f("B"), f("C"), D=f("D"), z=f("z"),
                            delta_bias=f("delta_bias"), delta_softplus=True, nthreads=1)
    return {
        "workload": I.TINY_F32.name,
        "source": "oracle (fp64), frozen after its pins passed; pages print no numeric example",
        "out": [[b, t, d, float(out[b, t, d]).hex()] for b, t, d in SAMPLES],
        "last_state": [[0, d, n, float(last[0, d, n]).hex()] for d, n in [(0, 0), (31, 7), (63, 15)]],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_f32_oracle.json"), "w") as fh:
        json.dump(compute(), fh, indent=1)
