"""Writes zipf_scale.json: the bias scale c of the skewed-routing workload.

The 131,072-token workload routes with a Zipf-like expert popularity.  Its router bias gets
``-c * 1.1 * ln(rank_e)`` added (see ``moe_inputs``).  This script finds c by bisection so that
the oracle's routing of a 4096-token sample (CPU draws, seed 3, H = 2880, E = 32, top-4) has a
max/mean expert load of 4.0.  It calls only the oracle and the input generator.

    python tests/golden/make_zipf_scale.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import moe_inputs as mi  # noqa: E402
from oracle import moe_route_ref  # noqa: E402

TARGET = 4.0
N_SAMPLE = 4096


def load_ratio(c: float, x_bits, W_router_bits, H, E, k, seed) -> float:
    _, b = mi.draw_router(H, E, seed, "cpu", zipf=True, c=c)
    r = moe_route_ref(x_bits, W_router_bits, b.numpy(), k)
    count = r["count"]
    return float(count.max() / count.mean())


def main():
    w = mi.WORKLOADS["131k_skewed"]
    x = mi.draw_x(N_SAMPLE, w.H, w.seed, "cpu")
    W_router, _ = mi.draw_router(w.H, w.E, w.seed, "cpu")
    xb, Wb = mi.bf16_bits(x), mi.bf16_bits(W_router)
    lo, hi = 0.0, 2.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        if load_ratio(mid, xb, Wb, w.H, w.E, w.k, w.seed) < TARGET:
            lo = mid
        else:
            hi = mid
    c = hi
    ratio = load_ratio(c, xb, Wb, w.H, w.E, w.k, w.seed)
    out = dict(c=c, max_over_mean=ratio, target=TARGET, sample_tokens=N_SAMPLE, seed=w.seed,
               H=w.H, E=w.E, k=w.k, s=mi.ZIPF_S,
               generated_by="tests/golden/make_zipf_scale.py (oracle routing only)")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "zipf_scale.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
