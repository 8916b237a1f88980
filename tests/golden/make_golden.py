"""Writes the stored expected values that come from the oracle (run from the repo root:
`python tests/golden/make_golden.py`). Calls only the oracle and the seeded generator."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from view_transformers_b200 import configs, synth  # noqa: E402


def perhead_budgets() -> str:
    w = configs.PERHEAD100
    scores = synth.head_scores(w)
    dens = oracle.water_fill(scores, w.heads * (1.0 - w.rho), 1.0)
    ks = [oracle.k_from_density(w.n_blocks, float(x)) for x in dens]
    lines = ["# Per-head block budgets k_h for the 100-frame workload (B = 608 blocks, 16 heads,",
             "# layer budget rho = 0.75 -> total density 4): LogNormal(0, 1) head scores from",
             "# Generator(PCG64(0)), capped water-filling (cap 1), k_h = clamp(floor(B d_h), 1, B).",
             "# Written by tests/golden/make_golden.py from the oracle.",
             "k " + " ".join(str(k) for k in ks),
             "density " + " ".join(repr(float(x)) for x in dens)]
    return "\n".join(lines) + "\n"


if __name__ == "__main__":
    with open(os.path.join(ROOT, "tests", "golden", "perhead100_budgets.txt"), "w") as f:
        f.write(perhead_budgets())
