"""Writes the stored expected values under tests/golden/ by calling only the oracle.

forced_fallback.json -- the 1e8-score, 256-level workload (sorted descending,
k = 1e6, t = 0.1) with a deliberately weak bracket (s = 4096 samples, delta = 0.5)
and the first Philox seed >= 0 whose bracket misses the oracle's threshold, so the
certification pass must reject it and the full-sort fallback must run
("Fast LapSum: Exact Differentiable Top-k at Million Scale", abstract: a
certification pass with a full-sort fallback for the worst case).  Stores the
seed, the bracket ends and the membership counts of the oracle's restatement.

Run:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle                # noqa: E402
import workloads as W        # noqa: E402


def forced_fallback():
    w = W.WORKLOADS["levels1e8"]
    r = W.scores(w)[0]
    s, delta = 4096, 0.5
    b = oracle.solve(r, w.k, w.t, method=1)
    for seed in range(10_000):
        br = oracle.bracket(r, w.k, w.t, seed, s, delta)
        if not (float(br["a_L"]) <= b < float(br["a_R"])):
            cert = oracle.certify(r, w.k, w.t, br["a_L"], br["a_R"], band_cap=10**12)
            assert cert["verdict"] == 0
            return {"workload": w.name, "k": w.k, "t": w.t, "sample_size": s, "delta": delta,
                    "seed": seed, "jR": br["jR"], "jL": br["jL"],
                    "a_L": float(br["a_L"]), "a_R": float(br["a_R"]),
                    "c_L": cert["c_L"], "c_band": cert["c_band"], "c_R": cert["c_R"],
                    "G_aL": cert["G_aL"], "G_aR": cert["G_aR"], "b_oracle": b,
                    "source": "oracle (tests/golden/make_golden.py)"}
    raise RuntimeError("no failing seed found")


if __name__ == "__main__":
    out = forced_fallback()
    with open(os.path.join(HERE, "forced_fallback.json"), "w") as f:
        json.dump(out, f, indent=1)
    print(out)
