"""Writes tiny_case.json: the oracle's results on a tiny seeded case, a regression pin of the oracle.

Calls only oracle/ (and numpy for the seeded inputs).  Rerun it only together with a change of the oracle's
arithmetic that the paper's text justifies, and say which passage in that change.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.join(HERE, "..", ".."))

import oracle  # noqa: E402

# tiny case: 2 heads, 32 tokens, d = 4, blocks of 4, 3 blocks per query, scale 0.5
BH, T, D, S, K, SCALE = 2, 32, 4, 4, 3, 0.5


def inputs():
    rng = np.random.default_rng(2024)
    return {name: np.round(rng.standard_normal((BH, T, D)), 3) for name in ("Q", "K", "V", "dO")}


def compute(x):
    Kbar = oracle.block_pool(x["K"], S)
    idx, _, _ = oracle.block_select(x["Q"], Kbar, S, K)
    Os, ls = oracle.attn_fwd(x["Q"], x["K"], x["V"], S, SCALE, idx)
    Of, lf = oracle.attn_fwd(x["Q"], x["K"], x["V"], S, SCALE)
    dQ, dK, dV = oracle.attn_bwd(x["Q"], x["K"], x["V"], x["dO"], S, SCALE, idx)
    loss = oracle.align_fwd(Of, Os)
    return {"Kbar": Kbar, "idx": idx, "O_sparse": Os, "lse_sparse": ls, "O_full": Of, "lse_full": lf,
            "dQ_sparse": dQ, "dK_sparse": dK, "dV_sparse": dV, "align_loss": np.array(loss)}


if __name__ == "__main__":
    oracle.build()
    x = inputs()
    out = compute(x)
    doc = {"case": dict(BH=BH, T=T, d=D, s=S, k=K, scale=SCALE),
           "inputs": {k: v.tolist() for k, v in x.items()},
           "outputs": {k: np.asarray(v).tolist() for k, v in out.items()}}
    with open(os.path.join(HERE, "tiny_case.json"), "w") as f:
        json.dump(doc, f)
    print("wrote tiny_case.json")
