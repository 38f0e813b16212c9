"""Writes tiny_oracle.txt: oracle values for the tiny configuration
(X bf16 [4, 256], Wg/Wu bf16 [512, 256] ~ N(0, 1/K), seed 0) at 32 fixed
output positions, plus sums over all outputs.  Calls only the oracle and the
seeded input generator; re-run it only when the oracle's arithmetic changes
for a reason a page passage gives.

    python tests/golden/make_tiny_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from up_projection_b200 import synth  # noqa: E402


def main():
    X, Wg, Wu = synth.swiglu_inputs(4, 256, 512, "bf16", seed=0)
    out = oracle.swiglu_fwd(X, Wg, Wu, "bf16")
    r = np.random.Generator(np.random.PCG64(2024))
    im = r.integers(0, 4, size=32)
    inn = r.integers(0, 512, size=32)
    lines = ["# oracle values, tiny config, written by make_tiny_golden.py",
             f"sum_H {float(out['H'].sum())!r}", f"sum_abs_H {float(np.abs(out['H']).sum())!r}",
             f"sum_G {float(out['G'].sum())!r}", f"sum_U {float(out['U'].sum())!r}"]
    for m, n in zip(im, inn):
        lines.append(f"H {int(m)} {int(n)} {float(out['H'][m, n])!r}")
    with open(os.path.join(HERE, "tiny_oracle.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
