"""Shared helpers for the parity tests (tolerances, conversions, oracle runs).

Every comparison made through check_close is also appended, as one JSON line,
to the file named by the environment variable SSA_PARITY_LOG when it is set
(the errors of a run, for the record, whether or not they pass)."""
from __future__ import annotations

import json
import os

import numpy as np

from block_top_sparse_b200 import inputs

# Tolerances against the fp64 oracle for outputs and gradients (bf16 or fp32
# results): max-abs 1e-2 beyond the final rounding of the stored element
# (half a bf16 ulp of the oracle value for bf16 outputs), and relative L2 5e-3.
MAX_ABS = 1e-2
REL_L2 = 5e-3
# Selection rows whose (k-1)-th and k-th candidate scores lie this close
# (relative) are exempt from bit-exact comparison.
TIE_REL = 1e-5


def bf16_half_ulp(x: np.ndarray) -> np.ndarray:
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def to_np(t) -> np.ndarray:
    import torch
    t = t.detach()
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.cpu().numpy().astype(np.float64)


def check_close(name: str, got: np.ndarray, ref: np.ndarray, bf16: bool) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (name, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "%s: non-finite values" % name
    diff = np.abs(got - ref)
    allow = MAX_ABS + (bf16_half_ulp(ref) if bf16 else 0.0)
    worst = float((diff - allow).max()) if diff.size else 0.0
    rel = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
    res = {"max_abs": float(diff.max()) if diff.size else 0.0, "rel_l2": rel}
    log_result(name, res)
    assert worst <= 0, "%s: max-abs excess %.3g (max diff %.3g)" % (name, worst, diff.max())
    assert rel <= REL_L2, "%s: rel-L2 %.3g > %.3g" % (name, rel, REL_L2)
    return res


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    got, ref = np.asarray(got, dtype=np.float64), np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))


def log_result(name: str, res: dict) -> None:
    path = os.environ.get("SSA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps(dict(name=name, **res)) + "\n")


def selection_report(got: np.ndarray, ref: np.ndarray, r1: np.ndarray, r2: np.ndarray) -> dict:
    """Rows of got that differ from ref, split into tie-exempt and real mismatches."""
    differ = np.any(got != ref, axis=-1)
    with np.errstate(invalid="ignore"):
        exempt = np.abs(r1 - r2) <= TIE_REL * np.maximum(np.abs(r1), np.abs(r2))
    exempt = np.where(np.isnan(r1) | np.isnan(r2), False, exempt)
    return {"rows": int(differ.size), "differ": int(differ.sum()), "exempt_rows": int(exempt.sum()),
            "mismatch": int((differ & ~exempt).sum()), "exempt_and_differ": int((differ & exempt).sum())}


def check_gpu_selection(ora, name: str, got: np.ndarray, Q: np.ndarray, Kbar: np.ndarray, s: int, k: int) -> dict:
    """Selection parity of got [BH, T, k] against the oracle on Q [BH, T, d], Kbar [BH, nb, d] (fp64):

    * every row is structurally valid (ascending, distinct, holds b(t), -1 padding at the end);
    * rows are bit-exact, except rows whose (k-1)-th and k-th oracle candidate scores lie within
      TIE_REL of each other;
    * on such an exempt row that differs, the chosen set is still a valid top-(k-1): the lowest
      oracle score among the chosen blocks is at least the highest among the blocks left out,
      less the same tolerance."""
    assert ora.check_selection(got, s), name + ": structurally invalid selection rows"
    ref, r1, r2 = ora.block_select(Q, Kbar, s, k)
    rep = selection_report(got, ref, r1, r2)
    assert rep["mismatch"] == 0, (name, rep)
    differ = np.argwhere(np.any(got != ref, axis=-1))
    if differ.size:
        sc = ora.block_scores(Q, Kbar, s, differ[:, 0], differ[:, 1])
        for i, (b, t) in enumerate(differ):
            bt = t // s
            chosen = [j for j in got[b, t] if 0 <= j < bt]
            left = [j for j in range(bt) if j not in chosen]
            assert len(chosen) == min(k - 1, bt), (name, b, t, chosen)
            if left:
                tol = TIE_REL * max(abs(r1[b, t]), abs(r2[b, t]))
                lo = min(sc[i, j] for j in chosen)
                hi = max(sc[i, j] for j in left)
                assert lo >= hi - tol, (name, int(b), int(t), lo, hi, tol)
    log_result(name + ".selection", rep)
    return rep


def workload_arrays(wl, **over):
    """Generate inputs; return (dict of numpy fp64 [BH,T,d] arrays, raw dict, effective workload)."""
    g = inputs.generate(wl, **over)
    w = g["wl"]
    f = {}
    for key in ("Q", "K", "V", "dO"):
        if key in g:
            f[key] = inputs.to_float64(g[key], w.dtype).reshape(w.B * w.H, w.T, w.d)
    return f, g, w


def to_device(arr: np.ndarray, dtype: str, device="cuda"):
    import torch
    if dtype == "bf16":
        t = torch.from_numpy(arr.view(np.int16).copy()).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))
    return t.to(device)
