"""Writes skew_router_bias.json: the additive router bias of the skewed-routing
workload (B = 256 sequences x K = 1, 512 rows; 4 seeded hot experts).

The workload asks for 4 hot experts that take about half of the top-6
assignments.  The reading taken: an fp32 bias beta is added to the hot
experts' router logits (0 elsewhere), and beta is bisected on the CPU oracle's
router (the only arithmetic this script calls) until the hot experts hold
50% +- 0.25% of the T * k slots of the workload's layer-0 input rows.  The
result is stored so the inputs need no oracle call: the workload table
carries the same value, and a CPU test checks both against a fresh bisection.

Run: python tests/golden/make_skew_router_bias.py
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
OUT = os.path.join(HERE, "skew_router_bias.json")


def bisect_beta(share: float = 0.5, tol: float = 0.01):
    """Smallest-magnitude bias on the hot experts giving them `share` of the
    top-k slots (within tol / 4), on the oracle's router.  Returns (beta as
    float32, the share it gives)."""
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    import oracle
    from moe_decoder_speculative_b200 import workloads as wl

    w = wl.workload(4)
    x = wl.make_hidden(w)
    layer = wl.make_layer(w, wl.layer_seeds(w)[0])
    hot = wl.hot_experts(w)

    def hot_share(beta):
        idx, _, _, _ = oracle.router(x, layer["w_router"], w.k, bias=wl.router_bias(w, beta))
        return float(np.isin(idx, hot).mean())

    lo, hi = 0.0, 8.0
    beta = hi
    for _ in range(40):
        beta = float(np.float32(0.5 * (lo + hi)))
        s = hot_share(beta)
        if abs(s - share) <= tol / 4:
            break
        if s < share:
            lo = beta
        else:
            hi = beta
    return beta, hot_share(beta)


def main():
    beta, share = bisect_beta()
    rec = {
        "_source": "skewed-routing workload: 4 hot experts take about 50% of the top-6 assignments; "
                   "an fp32 bias beta on the hot experts' router logits, bisected on the CPU oracle's router",
        "beta": beta,
        "hot_share": share,
    }
    with open(OUT, "w") as f:
        json.dump(rec, f, indent=2)
        f.write("\n")
    print(json.dumps(rec))


if __name__ == "__main__":
    main()
