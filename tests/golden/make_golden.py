"""Writes oracle_regression.json: outputs of the CPU oracle on small seeded
inputs, so that any later change to the oracle's arithmetic shows up as a
failing test and has to be justified.  The pages print no worked example;
these values are the oracle's own (this script calls only oracle/ and the
seeded input generators), not values from the pages.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from oracle import oracle  # noqa: E402
from speculative_decoding_05_b200 import workloads as WL  # noqa: E402

OUT = os.path.join(HERE, "oracle_regression.json")


def compute():
    res = {}
    # one step of the tiny workload: draft, prefix (off), full-block verify
    w = WL.get("tiny")
    inp = WL.make_inputs(w, device="cpu")
    h = {k: v.numpy() for k, v in inp.items()}
    d = oracle.draft(h["base"], h["U"], h["W"], h["prev_token"], h["u_draft"],
                     inv_temp=h["inv_temp"])
    L = np.full(w.B, w.K, np.int32)
    v = oracle.verify(h["target"], h["row_start"], L, h["base"], h["U"], h["W"], h["prev_token"],
                      d["tokens"], d["p_tok"], h["u_accept"], h["u_res"], inv_temp=h["inv_temp"])
    res["tiny_draft_tokens"] = d["tokens"].tolist()
    res["tiny_draft_p_tok"] = [float(x) for x in d["p_tok"].ravel()]
    res["tiny_verify_n_acc"] = v["n_acc"].tolist()
    res["tiny_verify_out_tokens"] = v["out_tokens"].tolist()
    # the prefix cut on a serving-sized batch, both cost readings and a budget
    w = WL.get("serving")
    inp = WL.make_inputs(WL.get("serving", V=1024, r=16), device="cpu")
    z, temps = inp["z"].numpy(), inp["temps"].numpy()
    xs, ys = inp["cost_tokens"].numpy(), inp["cost_ms"].numpy()
    for stair in (False, True):
        g = oracle.prefix_async(z, temps, xs, ys, staircase=stair)
        b = oracle.prefix_async(z, temps, xs, ys, staircase=stair, budget=w.B + 300)
        key = "stair" if stair else "linear"
        res[f"prefix_{key}_L"] = g["L"].tolist()
        res[f"prefix_{key}_objective"] = g["objective"]
        res[f"prefix_{key}_n_greedy"] = g["n_greedy"]
        res[f"prefix_{key}_budget_L"] = b["L"].tolist()
    # the temperature fit on a small calibration set
    c = WL.make_calibration(WL.Calibration("golden", N=3000, K=6, seed=8))
    f = oracle.sts_fit(c["z"].numpy(), c["n_acc"].numpy())
    res["sts_temps"] = [float(t) for t in f["temps"]]
    res["sts_ece"] = [f["ece_before"], f["ece_after"]]
    return res


if __name__ == "__main__":
    with open(OUT, "w") as fh:
        json.dump(compute(), fh, indent=1)
    print("wrote", OUT)
