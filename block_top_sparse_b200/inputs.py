"""Seeded synthetic inputs for the SSA block-sparse attention path.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle's
tests.  It holds random draws and workload structure only: no pooling, scoring,
selection, softmax or loss arithmetic of the method lives here.

Workloads follow the long-context settings of "SSA: Sparse Sparse Attention by
Aligning Full and Sparse Attention Outputs in Feature Space" (arXiv 2511.20102):
8k pre-training context, 32k continued training, 128k inference, receptive
fields k*s of 256 to 8192 tokens (paperlayer.ai summary, sections 3, 6 and
Appendix D).  No dataset item is reproduced; every tensor is drawn from numpy's
PCG64 generator.

bf16 tensors are produced by drawing fp32 values and rounding them to bf16 with
round-to-nearest-even on the host, so the GPU and the oracle read identical
values.  Arrays are returned as raw bit patterns (``uint16``) for bf16 and as
``float32`` for fp32, in [B, H, T, d] row-major layout.

Draw order for a given seed (documented so that any consumer can reproduce it):
  1. Q, K, V  ~ N(0, 1) * d**-0.25        (fp32, shape [B,H,T,d] each, in that order)
  2. structure draws (see ``_planted`` / ``_sink``)
  3. dO ~ N(0, 1)                           (only when requested)
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Optional, Tuple

import numpy as np

# Weight of the block-shared latent component in the keys of the planted
# workloads (within-block key correlation is PLANT_KEY_SHARE**2).
PLANT_KEY_SHARE = 0.5
# Correlation between a query and the latent direction of its planted blocks.
PLANT_QUERY_CORR = 0.6
# Number of planted preceding blocks per query.
PLANT_BLOCKS = 4
# Sink shift of block 0's keys along a per-head random unit direction, in units
# of the per-element standard deviation d**-0.25.
SINK_SHIFT_SIGMA = 2.0


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    T: int
    d: int
    s: int
    k: Tuple[int, ...]
    dtype: str            # "bf16" or "fp32"
    seed: int
    structure: str        # "plain", "planted" or "sink"
    backward: bool        # whether a dO is drawn and the backward runs
    note: str = field(default="", compare=False)

    @property
    def nb(self) -> int:
        return self.T // self.s


# The five workloads of the benchmark/parity contract.
WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 1, 2, 1024, 64, 64, (4,), "fp32", 0, "plain", True,
                     "tiny fwd+bwd, both streams + alignment; fp32"),
    "prefill": Workload("prefill", 1, 16, 8192, 128, 64, (16,), "bf16", 1, "planted", False,
                        "prefill fwd, receptive field 1024, planted blocks"),
    "train": Workload("train", 4, 16, 4096, 128, 64, (8,), "bf16", 2, "plain", True,
                      "training step fwd+bwd, both streams + alignment"),
    "long": Workload("long", 1, 32, 32768, 128, 128, (16,), "bf16", 3, "sink", True,
                     "32K-context fwd+bwd, receptive field 2048, sink block"),
    "sweep": Workload("sweep", 1, 8, 131072, 128, 128, (4, 8, 16, 32, 64), "bf16", 4, "planted", False,
                      "128K-context sparsity-budget sweep, fwd"),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_float64(x: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 values of a generated tensor (bf16 bits or fp32)."""
    if dtype == "bf16":
        return bf16_bits_to_f32(x).astype(np.float64)
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _encode(x32: np.ndarray, dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x32) if dtype == "bf16" else np.ascontiguousarray(x32, dtype=np.float32)


def _distinct_preceding(rng: np.random.Generator, m: np.ndarray, count: int) -> np.ndarray:
    """For each row n draw ``count`` distinct integers from [0, m[n]) (Floyd's method).

    Rows with m[n] <= count take every integer below m[n]; unused slots hold -1.
    """
    n = m.shape[0]
    out = np.full((n, count), -1, dtype=np.int64)
    big = m > count
    mb = m[big]
    sel = np.empty((mb.shape[0], count), dtype=np.int64)
    for q in range(count):
        hi = mb - count + q            # Floyd: draw r in [0, hi]
        r = rng.integers(0, hi + 1)
        dup = np.zeros(mb.shape[0], dtype=bool)
        for p in range(q):
            dup |= sel[:, p] == r
        sel[:, q] = np.where(dup, hi, r)
    out[big] = sel
    small = ~big
    if small.any():
        ms = m[small]
        ar = np.arange(count)[None, :]
        out[small] = np.where(ar < ms[:, None], ar, -1)
    return out


def _planted(rng: np.random.Generator, wl: Workload, Q: np.ndarray, K: np.ndarray) -> None:
    """Planted block structure (in place on fp32 Q, K).

    Every key block j of every head carries a latent direction z_j ~ N(0, I_d);
    the keys of block j become  sigma*(a*z_j + sqrt(1-a^2)*n_t)  with n_t the
    original unit-variance draw.  Each query t draws ``PLANT_BLOCKS`` distinct
    preceding blocks P(t) (all of them when fewer exist) and becomes
    sigma*(rho*w_t + sqrt(1-rho^2)*n'_t)  with  w_t = sum_{j in P(t)} z_j / sqrt(|P(t)|).
    Per-element standard deviation stays sigma = d**-0.25.
    """
    B, H, T, d, s = wl.B, wl.H, wl.T, wl.d, wl.s
    nb = T // s
    sigma = d ** -0.25
    a = PLANT_KEY_SHARE
    rho = PLANT_QUERY_CORR
    Z = rng.standard_normal((B, H, nb, d), dtype=np.float32)
    K *= np.float32(np.sqrt(1.0 - a * a))
    K += np.repeat(Z, s, axis=2) * np.float32(a * sigma)
    blk_of_t = np.arange(T) // s
    chunk = 1 << 15
    for b in range(B):
        for h in range(H):
            picks = _distinct_preceding(rng, blk_of_t.astype(np.int64), PLANT_BLOCKS)  # [T, 4]
            cnt = (picks >= 0).sum(axis=1)
            zb = Z[b, h]
            for t0 in range(0, T, chunk):
                p = picks[t0:t0 + chunk]
                c = cnt[t0:t0 + chunk]
                w = np.zeros((p.shape[0], d), dtype=np.float32)
                for q in range(PLANT_BLOCKS):
                    valid = p[:, q] >= 0
                    w[valid] += zb[p[valid, q]]
                has = c > 0
                w[has] /= np.sqrt(c[has]).astype(np.float32)[:, None]
                qq = Q[b, h, t0:t0 + chunk]
                qq[has] = qq[has] * np.float32(np.sqrt(1.0 - rho * rho)) + w[has] * np.float32(rho * sigma)


def _sink(rng: np.random.Generator, wl: Workload, K: np.ndarray) -> None:
    """Sink block: block 0's keys shifted by SINK_SHIFT_SIGMA*sigma along a per-head unit vector."""
    B, H, d, s = wl.B, wl.H, wl.d, wl.s
    sigma = d ** -0.25
    u = rng.standard_normal((B, H, d), dtype=np.float32)
    u /= np.linalg.norm(u, axis=-1, keepdims=True)
    K[:, :, 0:s, :] += np.float32(SINK_SHIFT_SIGMA * sigma) * u[:, :, None, :]


def generate(wl: Workload, *, T: Optional[int] = None, H: Optional[int] = None, B: Optional[int] = None,
             seed: Optional[int] = None, with_dO: Optional[bool] = None) -> Dict[str, np.ndarray]:
    """Draw Q, K, V (and dO) for a workload; sizes may be overridden for small parity cases.

    Returns a dict with 'Q', 'K', 'V' (and 'dO') encoded per ``wl.dtype`` and the
    effective Workload under key 'wl'.
    """
    from dataclasses import replace
    wl = replace(wl, T=T or wl.T, H=H or wl.H, B=B or wl.B, seed=wl.seed if seed is None else seed)
    if wl.T % wl.s:
        raise ValueError("T must be a multiple of s")
    rng = np.random.default_rng(wl.seed)
    shape = (wl.B, wl.H, wl.T, wl.d)
    sigma = np.float32(wl.d ** -0.25)
    Q = rng.standard_normal(shape, dtype=np.float32) * sigma
    K = rng.standard_normal(shape, dtype=np.float32) * sigma
    V = rng.standard_normal(shape, dtype=np.float32) * sigma
    if wl.structure == "planted":
        _planted(rng, wl, Q, K)
    elif wl.structure == "sink":
        _sink(rng, wl, K)
    elif wl.structure != "plain":
        raise ValueError(wl.structure)
    out = {"Q": _encode(Q, wl.dtype), "K": _encode(K, wl.dtype), "V": _encode(V, wl.dtype), "wl": wl}
    if wl.backward if with_dO is None else with_dO:
        dO = rng.standard_normal(shape, dtype=np.float32)
        out["dO"] = _encode(dO, wl.dtype)
    return out


def group_kv(g: Dict[str, np.ndarray], Hkv: int) -> Dict[str, np.ndarray]:
    """Grouped-query inputs from a draw of H heads: the key/value heads are the K, V of heads 0, G, 2G, ...
    (G = H / Hkv), so every query head keeps the per-element distribution of its workload."""
    H = g["Q"].shape[1]
    if Hkv < 1 or H % Hkv:
        raise ValueError("H must be a multiple of Hkv")
    G = H // Hkv
    out = dict(g)
    for key in ("K", "V"):
        out[key] = np.ascontiguousarray(g[key][:, ::G])
    return out


def random_tensor(shape, dtype: str, seed: int, std: float = 1.0) -> np.ndarray:
    """A plain N(0, std^2) tensor in the requested encoding (for edge-case tests)."""
    rng = np.random.default_rng(seed)
    return _encode(rng.standard_normal(shape, dtype=np.float32) * np.float32(std), dtype)
