"""Calibrate the Zipf-ranked router bias of the skewed prefill workload.

TEST INFRASTRUCTURE (writes an input-recipe constant; uses only the oracle's
routing and the seeded input generator).

The workload asks for expert popularity shaped like Zipf(s=1.1) with the
hottest expert at about 10x the mean load.  A literal Zipf(1.1) inclusion
profile over 256 experts at top-8 is infeasible (the top expert would need to
appear in more than every token), so the rank shape is kept and its scale is
calibrated: b_e = -alpha * s * ln(r_e), and alpha is found by bisection on the
oracle's own top-k so that max_e count_e / (T k / E) = 10.

Usage:  python oracle/calibrate_zipf.py   (writes sparse_moe_layer_select_b200/zipf_alpha.json)
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from oracle import moe_oracle as O  # noqa: E402
from sparse_moe_layer_select_b200 import inputs as I  # noqa: E402

TARGET = 10.0


def load_stats(logits, bias, k, E):
    idx = O.select_topk(logits + bias[None, :].astype(np.float64), k)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    mean = idx.size / E
    return counts.max() / mean, counts.std() / mean, counts


def main():
    w = I.get("c3_xs2_prefill_zipf")
    x = I.generate_numpy((w.T, w.d_model), w.seed, I.TID_X, w.sigma_x)
    wr = I.generate_numpy((w.E, w.d_model), w.seed, I.TID_W_ROUTER, w.sigma_router)
    logits = O.router_logits(x, wr, None)
    lo, hi = 0.0, 4.0
    assert load_stats(logits, I.zipf_bias(w.E, w.zipf_s, hi), w.k, w.E)[0] > TARGET
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        r, _, _ = load_stats(logits, I.zipf_bias(w.E, w.zipf_s, mid), w.k, w.E)
        if r < TARGET:
            lo = mid
        else:
            hi = mid
    alpha = float(np.float32(hi))
    ratio, cv, counts = load_stats(logits, I.zipf_bias(w.E, w.zipf_s, alpha), w.k, w.E)
    out = {"alpha": alpha, "s": w.zipf_s, "target_max_over_mean": TARGET,
           "max_over_mean": float(ratio), "cv": float(cv),
           "min_count": int(counts.min()), "max_count": int(counts.max()),
           "experts_with_zero_rows": int((counts == 0).sum()),
           "written_by": "oracle/calibrate_zipf.py"}
    path = os.path.join(ROOT, "sparse_moe_layer_select_b200", "zipf_alpha.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
