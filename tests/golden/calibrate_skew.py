"""Choose the skew constant c of the masked, Zipf-like workload.

The CMF code specialist page (Calibrate step) reports that on code the top 64
of 256 experts carry 73% of the routing mass, and (Defrag step) that about 160
of 256 experts are kept.  The skewed workload reproduces that shape: 160 active
experts, selection bias b_e = c * (-ln(rank_e + 1)) over a seeded ranking, and c
chosen so that the 64 highest-bias experts receive 73% of the (token, slot)
selections made by the ORACLE's router on the workload's own tokens.

Run:  python tests/golden/calibrate_skew.py   (writes skew_calibration.json)
Only ``oracle`` and the input generator ``synth`` are used.
"""
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402

TARGET, TOP = 0.73, 64


def share(orc, logits, top_set):
    hits = 0
    for t in range(logits.shape[0]):
        idx, _, _ = orc.select(logits[t])
        hits += int(np.isin(idx, top_set).sum())
    return hits / (logits.shape[0] * orc.prob.k)


def main():
    t0 = time.time()
    prob = synth.make_problem(5, bias=("skew", 0.0))
    ranks = synth.skew_ranks(prob.cfg, prob.mask)
    top_set = np.nonzero((ranks >= 0) & (ranks < TOP))[0]
    orc = oracle.Oracle(prob)
    logits = orc.logits(range(prob.T))
    print("logits for %d tokens in %.1fs" % (prob.T, time.time() - t0))

    def at(c):
        prob.b[:] = synth.skew_bias(prob.cfg, prob.mask, c)
        return share(orc, logits, top_set)

    lo, hi = 0.0, 1.0
    while at(hi) < TARGET:
        hi *= 2
    for _ in range(14):
        mid = 0.5 * (lo + hi)
        if at(mid) < TARGET:
            lo = mid
        else:
            hi = mid
    c = float("%.4g" % (0.5 * (lo + hi)))
    realised = at(c)
    out = dict(c=c, realised_top64_share=realised, target=TARGET, tokens=int(prob.T), k=int(prob.k),
               n_active=int(prob.mask.sum()), seed=int(prob.cfg["seed"]),
               how="bisection on c with the oracle router over every token of the workload")
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "skew_calibration.json")
    json.dump(out, open(path, "w"), indent=1)
    print(json.dumps(out), "in %.1fs" % (time.time() - t0))


if __name__ == "__main__":
    main()
