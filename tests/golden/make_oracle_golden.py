"""Writes tests/golden/oracle_small_case.json: the oracle's float64 outputs on
one small seeded case (a regression lock on the oracle's arithmetic). It calls
only the oracle; run it from the repository root:

    python -m tests.golden.make_oracle_golden
"""
import json
import os

import numpy as np

CASE = {"B": 1, "T": 9, "H": 2, "dk": 4, "dv": 3, "eta": 0.25, "seed": 2024, "apf": True}


def _inputs():
    rng = np.random.default_rng(CASE["seed"])
    B, T, H, dk, dv = (CASE[n] for n in ("B", "T", "H", "dk", "dv"))
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    v = rng.standard_normal((B, T, H, dv))
    beta = rng.uniform(0.1, 0.9, (B, T, H))
    r = rng.uniform(0.7, 1.0, (B, T, H))
    d0 = rng.uniform(0.5, 1.5, (B, H, dk))
    S0 = 0.5 * rng.standard_normal((B, H, dv, dk))
    return q, k, v, beta, r, d0, S0


def compute():
    import oracle
    q, k, v, beta, r, d0, S0 = _inputs()
    out, S, d = oracle.fwd(q, k, v, beta, r, d0, S0, eta=CASE["eta"], nthreads=1)
    return {"out": out.tolist(), "S": S.tolist(), "d": d.tolist()}


if __name__ == "__main__":
    res = compute()
    res["case"] = CASE
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_case.json"), "w") as fh:
        json.dump(res, fh, indent=1)
