"""Writes the stored expected values under tests/golden/ by calling only the oracle.

    python tests/golden/make_golden.py

tiny_route.json: the top-p routing CSR of the tiny workload (B1 H2 N512 d64,
block 64, i.i.d. N(0,1) bf16 inputs from seed 0, p = 0.9), computed by the fp64
oracle.  Definition: FVAttn review, §1 Key Terms "Top-p routing", with the
score fixed by this library (mean-pooled blocks, qbar.kbar/sqrt(d), softmax
over key blocks, ties to the lower index).  It guards the oracle against
unjustified changes; a change to it must name the passage that justifies it.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from workloads import TINY, generate  # noqa: E402


def main():
    Q, K, _ = generate(TINY)
    r = oracle.route(Q, K, TINY.p, TINY.bs)
    out = {
        "source": "FVAttn review, §1 Key Terms 'Top-p routing'; score as fixed by this library",
        "workload": TINY.describe(),
        "row_ptr": r.row_ptr.tolist(),
        "col_idx": r.col_idx.tolist(),
        "head_counts": r.head_counts.tolist(),
        "kept_mass": [round(float(x), 12) for x in r.diag[:, 0]],
    }
    with open(os.path.join(HERE, "tiny_route.json"), "w") as f:
        json.dump(out, f, indent=1)
        f.write("\n")


if __name__ == "__main__":
    main()
