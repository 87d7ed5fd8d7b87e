"""Choose the Zipf bias strength of the speculative-verify workload (B=128).

The workload wants Zipf(s=1.1)-skewed expert popularity imposed through the
per-expert selection bias: bias_e = -beta * ln(rank_e) over a seeded
permutation of ranks.  This script routes the workload's 128 tokens with the
oracle's router for a sweep of beta, fits the log-log slope of the sorted
per-expert token counts, and writes the sweep to ``zipf_calibration.txt``.
The chosen beta is copied by hand into ``synth.ZIPF_BETA``.

Run:  python tests/golden/calibrate_zipf.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from mxfp4_latent_moe_router_b200 import synth  # noqa: E402


def fitted_slope(ids: np.ndarray, E: int, max_rank: int = 64) -> float:
    counts = np.bincount(ids.ravel(), minlength=E)
    c = np.sort(counts)[::-1]
    c = c[:max_rank]
    c = c[c > 0]
    r = np.arange(1, len(c) + 1)
    return float(np.polyfit(np.log(r), np.log(c), 1)[0])


def main():
    shape = synth.SHAPES["b128"]
    w = synth.make_weights(shape)
    rank = np.empty(shape.num_experts)
    rank[np.argsort(-w["router_bias"], kind="stable")] = np.arange(1, shape.num_experts + 1)
    x = synth.make_x(shape)
    lines = ["# beta  fitted_slope(ranks 1..64)  distinct_experts  max_tokens_per_expert"]
    for beta in [0.02, 0.04, 0.06, 0.08, 0.10, 0.12, 0.13, 0.14, 0.15, 0.2, 0.3]:
        w["router_bias"] = (-beta * np.log(rank)).astype(np.float32)
        r = oracle.route(shape, w, x)
        counts = np.bincount(r["ids"].ravel(), minlength=shape.num_experts)
        lines.append("%.3f %.3f %d %d" % (beta, fitted_slope(r["ids"], shape.num_experts),
                                          int((counts > 0).sum()), int(counts.max())))
        print(lines[-1])
    with open(os.path.join(HERE, "zipf_calibration.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
