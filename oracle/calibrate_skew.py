"""Calibrate the skewed workload's logit offset (writes moe_inputs/skew_beta.json).

The skewed-routing workload adds to each routed expert's router logit an
offset o_i = -beta * s * ln(rank_i) with s = 1.1 (a Zipf(s)-shaped ranking over
a seeded permutation of the 256 routed experts).  beta is chosen so that, at
b = 0 on the workload's own tokens, the 8 most-loaded experts receive 30% of
all top-6 assignments (to within 0.5%).  The routing that decides it is the
oracle's (fp64); this script calls only oracle/ and the input generator.

Usage: python oracle/calibrate_skew.py
"""
import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import moe_inputs as mi  # noqa: E402
import oracle  # noqa: E402

TARGET_SHARE = 0.30
TOLERANCE = 0.005


def top8_share(z, w, beta):
    off = mi.zipf_offset(w, beta)
    r = oracle.route(z, np.zeros(w.n_routed, np.float32), w.k, w.n_routed, w.n_shared, off)
    c = np.sort(oracle.load_counts(r["topk_idx"], w.n_routed))[::-1]
    return c[:8].sum() / c.sum(), c


def main():
    w = mi.WORKLOADS["skew"]
    x = mi.host_x(w)
    wr = mi.host_wr(w)
    z = oracle.logits(x, wr)
    lo, hi = 0.0, 4.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        share, _ = top8_share(z, w, mid)
        if share < TARGET_SHARE:
            lo = mid
        else:
            hi = mid
    beta = 0.5 * (lo + hi)
    # keep 6 significant digits; re-check the stored value itself
    beta = float(f"{beta:.6g}")
    share, c = top8_share(z, w, beta)
    assert abs(share - TARGET_SHARE) <= TOLERANCE, share
    mean = w.k * w.T / w.n_routed
    out = {"beta": beta, "zipf_s": mi.ZIPF_S, "top8_share": round(float(share), 6),
           "max_over_mean_load": round(float(c[0] / mean), 4),
           "workload": "skew: T=16384, d=4096, seed 0, b=0",
           "written_by": "oracle/calibrate_skew.py"}
    with open(mi.SKEW_BETA_PATH, "w") as fh:
        json.dump(out, fh, indent=1)
        fh.write("\n")
    print(json.dumps(out))


if __name__ == "__main__":
    main()
