"""Write tests/golden/qb_solve_65536x256_k8.txt: the oracle's balanced assignment of the
full-size QB workload (65536 x 256 scores, N(0,1) plus a per-expert skew N(0, 1.5^2),
seed 0, k = 8, SOLVE with at most 32 beta updates, midpoint thresholds).

The oracle takes a few minutes for this; the GPU test compares against the stored
result instead of re-running it. Only the oracle computes the values written here.

    python tests/golden/make_qb_solve_golden.py
"""
import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import workloads as W  # noqa: E402

OUT = os.path.join(ROOT, "tests", "golden", "qb_solve_65536x256_k8.txt")


def main():
    q = W.QB_CONFIG
    s = W.make_qb_scores(q["m"], q["n"], seed=0, skew_std=q["skew_std"])
    idx, beta, info, rc = oracle.balance_assign(s, q["k"], mode=oracle.QB_SOLVE, max_iters=32)
    assert rc == oracle.OK
    digest = hashlib.sha256(np.ascontiguousarray(idx, dtype="<i4").tobytes()).hexdigest()
    with open(OUT, "w") as fh:
        fh.write("# The oracle's balanced assignment of the full-size QB workload, written by\n"
                 "# tests/golden/make_qb_solve_golden.py (oracle only). Problem: \"MoE travelogue 6\"\n"
                 "# (kexue.fm/archives/11619), Linear programming eq. (3) with row sums k and column\n"
                 "# sums m k / n; the alternating QB iteration (at most 32 beta updates, midpoint\n"
                 "# thresholds), then the exact successive-shortest-path finish.\n"
                 f"# scores: workloads.make_qb_scores(m={q['m']}, n={q['n']}, seed=0, skew_std={q['skew_std']})\n")
        fh.write(f"m: {q['m']}\nn: {q['n']}\nk: {q['k']}\nmax_iters: 32\n")
        fh.write(f"info: {' '.join(str(int(v)) for v in info)}\n")
        fh.write(f"picks_sha256: {digest}\n")
        fh.write("beta_bits: " + " ".join(f"{int(b):08x}" for b in beta.view(np.uint32)) + "\n")
    print(OUT)


if __name__ == "__main__":
    main()
