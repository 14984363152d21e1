"""Calibrate the tiny fp32 layer's mask bias gamma with the oracle alone.

The tiny workload (d=128, E=8, K=2, I=256, T=64, seed 0, no renormalisation)
builds W_mask = N(0, 1/d) - gamma * mu, where mu is the tokens' mean vector.
The kept fraction of the seed batch is a step function of gamma.  This script
bisects (60 halvings on [-8, 8]) for both ends of the step on which the fp64
oracle keeps exactly half of the Top-K candidates, takes the middle of that
step (so that no candidate sits on the threshold), and writes the value to
tiny_gamma.json beside it.  Only the oracle and the input generator are used.

Run from the repository root:  python tests/golden/make_tiny_gamma.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from dynamic_expert_routing_router_b200 import inputs  # noqa: E402


def kept_fraction(gamma, T=64, seed=0):
    L = inputs.make_tiny(T=T, seed=seed, gamma=gamma)
    h = {k: inputs.host_array(v) for k, v in L.items()}
    r, z = oracle.logits(h["x"], h["W_gate"], h["W_mask"], "f32")
    rt = oracle.route(r, z, inputs.TINY.K, inputs.TINY.renorm)
    return float((rt["idx"] >= 0).mean())


def _edge(pred):
    """Smallest gamma in [-8, 8] with pred(kept_fraction(gamma)) true."""
    lo, hi = -8.0, 8.0  # kept fraction decreases with gamma on this batch
    for _ in range(60):
        mid = 0.5 * (lo + hi)
        if pred(kept_fraction(mid)):
            hi = mid
        else:
            lo = mid
    return hi


def main():
    g_lo = _edge(lambda f: f <= 0.5)   # first gamma keeping at most half
    g_hi = _edge(lambda f: f < 0.5)    # first gamma keeping less than half
    gamma = 0.5 * (g_lo + g_hi)
    out = {"gamma": gamma, "step": [g_lo, g_hi], "kept_fraction": kept_fraction(gamma),
           "recipe": "tiny fp32 layer, T=64, seed 0, target 0.5 of Top-K candidates kept",
           "written_by": "tests/golden/make_tiny_gamma.py (oracle only)"}
    with open(os.path.join(HERE, "tiny_gamma.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)


if __name__ == "__main__":
    main()
