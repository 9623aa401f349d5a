"""Calibrate the skew of the mid-size prefill workload on the oracle's routing.

TEST INFRASTRUCTURE.  The skewed workload (2048 tokens of the 30B-A3B layer)
routes a constant feature x[:, H-1] = 1 to eight "hot" experts with router
weight b.  This script bisects b on the oracle's fp64 routing until the hot
experts take 30 +- 1 % of all assignments, and writes b and the share to
tests/golden/skew_prefill_t2048.json.  Run: python -m oracle.calibrate_skew
"""
import json
import os
import sys

import numpy as np

import oracle
import synth

OUT = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "tests",
                   "golden", "skew_prefill_t2048.json")


def share(cfg, b):
    x, wr, hot, _, _ = synth.make_router_and_x(cfg, skew_b=b)
    idx, _, _, _ = oracle.route_parallel(cfg, x, wr, threads=os.cpu_count() or 4)
    return float(np.isin(idx, hot).mean()), hot


def main():
    cfg = synth.CONFIGS["prefill_skewed_bf16_t2048"]
    lo, hi = 0.0, 8.0
    target = 0.30
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        s, hot = share(cfg, mid)
        if abs(s - target) < 0.002:
            break
        if s < target:
            lo = mid
        else:
            hi = mid
    b = float(np.float32(mid))
    s, hot = share(cfg, b)
    assert abs(s - target) <= 0.01, s
    rec = {"what": "router weight b on the constant feature that routes ~30% of assignments "
                   "to the 8 hot experts of the skewed 2048-token workload",
           "written_by": "python -m oracle.calibrate_skew (fp64 oracle routing, bisection)",
           "workload": cfg.name, "b": b, "hot_share": s, "hot_experts": hot.tolist()}
    with open(OUT, "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps(rec))


if __name__ == "__main__":
    sys.exit(main())
