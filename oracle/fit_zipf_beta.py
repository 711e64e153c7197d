"""Fit the bias amplitude beta of the Zipf-skewed prefill router and write it to
synth/zipf_beta.json.

The prefill workload skews expert popularity with a selection bias
b_e = beta * r_e ** -1.1 (r_e = the expert's rank in a seeded permutation), and
asks for a busiest expert of about 100 tokens out of 512 x top-8.  beta is found
by bisection with the oracle's router on the workload's own seeded tokens.
Run:  python oracle/fit_zipf_beta.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth   # noqa: E402

TARGET = 100


def max_load(wl, beta, x, wr):
    _, b = synth.router(wl, 0, beta=beta)
    idx, _, gap = oracle.route(x, wr.numpy(), b.numpy(), wl.k)
    return int(np.bincount(idx.reshape(-1), minlength=wl.E).max()), gap


def main():
    wl = synth.GLM_PREFILL
    wr, _ = synth.router(wl, 0, beta=0.0)
    x = synth.tokens(wl, wl.T).numpy()
    lo, hi = 0.0, 1.0
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        m, _ = max_load(wl, mid, x, wr)
        if m < TARGET:
            lo = mid
        else:
            hi = mid
    beta = hi
    m, gap = max_load(wl, beta, x, wr)
    out = os.path.join(ROOT, "synth", "zipf_beta.json")
    data = {}
    if os.path.exists(out):
        with open(out) as f:
            data = json.load(f)
    data[wl.name] = {"beta": beta, "max_tokens_per_expert": m,
                     "tokens_below_gap_1e-3": int((gap < 1e-3).sum()),
                     "how": "bisection on beta with the oracle router, raw draws"}
    with open(out, "w") as f:
        json.dump(data, f, indent=1)
    print(json.dumps(data[wl.name]))


if __name__ == "__main__":
    main()
