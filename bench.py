#!/usr/bin/env python3
"""Benchmark of the SSA block-sparse attention hot path on B200.

One step = one pass of the whole path over one batch of the 32K-context
workload (B=1, H=32, T=32768, d=128, s=128, k=16, bf16, sink block):
  block pooling, causal top-k selection, inverse selection index, full causal
  attention forward, sparse attention forward, alignment loss forward,
  alignment backward (the main stream -- full on even steps, sparse on odd
  steps -- also receives its upstream gradient), full attention backward and
  sparse attention backward accumulating into one set of dQ, dK, dV.

The metric is the sparse attention's forward + backward throughput: `value` is
tokens/s of the sparse stream's calls (inverse index, forward, backward), timed
with CUDA events around those calls inside the timed region of whole steps; the
whole step's time and every call's time come from the same timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  N > 1 runs independent replicas, one per GPU
(the path has no exchange step); value = tokens of all ranks / max-over-ranks time.
``--impl reference`` times the fp64 CPU oracle on the host cores instead, on a
bounded sample of the same workload (see ``reference_arm``).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "sparse-attn fwd+bwd TFLOP/s & tokens/s at 32K ctx; % of bf16 tensor peak"
WORKLOAD = "long"
K_SEL = 16
E2E_GROUPS = 8  # head groups of the end-to-end pipeline (copy in / sparse path / copy out on three streams)
# DRAM bytes (read + write) per head of one attn_bwd_kernel launch of the full stream at the 32K
# workload: ncu dram__bytes_read.sum + dram__bytes_write.sum of the 8-head launch (509,917,696 +
# 413,089,536 B) divided by 8.  Set to None whenever the kernel changes until it is captured again.
FULL_BWD_DRAM_BYTES_PER_HEAD = 923007232 / 8


def flops(B, H, T, d, s, k):
    """Algorithmic FLOPs: sparse fwd 4*B*H*d*sum_t min(k*s, t+1); full fwd 4*B*H*d*T(T+1)/2; bwd = 2.5 x fwd."""
    t = np.arange(T, dtype=np.float64)
    sparse_fwd = 4.0 * B * H * d * np.minimum(k * s, t + 1).sum()
    full_fwd = 4.0 * B * H * d * T * (T + 1) / 2.0
    return sparse_fwd, 2.5 * sparse_fwd, full_fwd, 2.5 * full_fwd


def max_over_ranks(vals, device):
    """Element-wise maximum of per-rank timings over every rank of the default process group.

    The whole job finishes when its slowest replica does, so a job time is the max over ranks.
    With no process group (one GPU) the values come back unchanged.
    """
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in vals]
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def whole_job_tokens_per_s(tokens_per_rank, world, ms_per_step):
    """Throughput of the whole job: the tokens every replica processed in one step over the step time."""
    return tokens_per_rank * world / (ms_per_step / 1e3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc = index, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (getattr(self, "out", "") or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 7:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(rows[0][1]) if rows[0][1].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows)}


def oracle_sample(T_sample: int):
    """Run the oracle's sparse path on a prefix sample: head (0,0), first T_sample tokens.

    The sparse path is what the metric times: pooling, selection, sparse attention forward and backward.
    Returns (seconds, sample FLOPs of sparse fwd + bwd by the metric's count, description)."""
    import oracle
    from block_top_sparse_b200 import inputs
    wl = inputs.WORKLOADS[WORKLOAD]
    g = inputs.generate(wl, H=1, T=T_sample)
    f = {key: inputs.to_float64(g[key], "bf16").reshape(1, T_sample, wl.d) for key in ("Q", "K", "V", "dO")}
    s, k, scale = wl.s, K_SEL, wl.d ** -0.5
    t0 = time.perf_counter()
    Kbar = oracle.block_pool(f["K"], s)
    idx, _, _ = oracle.block_select(f["Q"], Kbar, s, k)
    oracle.attn_fwd(f["Q"], f["K"], f["V"], s, scale, idx)
    oracle.attn_bwd(f["Q"], f["K"], f["V"], f["dO"], s, scale, idx)
    dt = time.perf_counter() - t0
    sf, sb, _, _ = flops(1, 1, T_sample, wl.d, s, k)
    return dt, sf + sb, ("head (b=0,h=0), first %d of %d tokens: pool, select, sparse attention fwd + bwd; "
                         "extrapolated to the full workload by the sparse fwd+bwd FLOP count" % (T_sample, wl.T))


def reference_arm(args, rank):
    """The oracle as it stands on the host cores, on the metric's quantity (sparse attention fwd + bwd
    tokens/s), extrapolated from a prefix sample to the full workload by FLOPs."""
    if rank != 0:
        return
    import oracle
    from block_top_sparse_b200 import inputs
    oracle.build()
    wl = inputs.WORKLOADS[WORKLOAD]
    sf, sb, _, _ = flops(wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL)
    T_sample = args.ref_tokens
    for _ in range(args.warmup):
        oracle_sample(T_sample)
    times, fl, desc = [], None, None
    for _ in range(args.steps):
        dt, fl, desc = oracle_sample(T_sample)
        times.append(dt)
    est = sum(times) / len(times) * (sf + sb) / fl  # seconds for the full workload's sparse fwd + bwd
    tok_s = wl.B * wl.T / est
    line = {"metric": METRIC, "value": tok_s, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": est * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(wl),
            "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                             "sample": desc + "; time per sample %.2f s" % (sum(times) / len(times)),
                             "extrapolated": True},
            "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def exact_attended_flops(B, H, T, d, s, k):
    """Forward FLOPs by the attended-token count: query t sees (t mod s) + 1 keys of its own block and s keys
    of each of min(k-1, b(t)) earlier blocks."""
    t = np.arange(T, dtype=np.int64)
    n = (t % s) + 1 + s * np.minimum(k - 1, t // s)
    return 4.0 * B * H * d * float(n.sum())


def sweep(args):
    """Config 5: sparse forward tokens/s at T = 131072 for k in {4, 8, 16, 32, 64}, with the dropped mass
    delta_t = 1 - exp(lse_s - lse_f) (mean, p99, max) and max_t |o_f - o_s| / (2 delta_t max|v|), which the
    exact identity o_f = (1 - delta) o_s + delta u_drop bounds by 1.  One JSON line per k."""
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import build, inputs, ops
    build.build()
    wl = inputs.WORKLOADS["sweep"]
    g = inputs.generate(wl)
    dev = {key: torch.from_numpy(g[key].view(np.int16)).view(torch.bfloat16).cuda() for key in ("Q", "K", "V")}
    Q, K, V = dev["Q"], dev["K"], dev["V"]
    B, H, T, d, s = wl.B, wl.H, wl.T, wl.d, wl.s
    dims0 = L.make_dims(B, H, T, d, s, 1)
    Of, lf, _ = ops.attn_fwd(dims0, Q, K, V)
    vmax = torch.linalg.vector_norm(V.float(), dim=-1).amax(dim=-1, keepdim=True)
    for k in (4, 8, 16, 32, 64):
        dims = L.make_dims(B, H, T, d, s, k)
        idx = ops.block_select(dims, Q, ops.block_pool(dims, K))
        Os = torch.empty_like(Q)
        lse = torch.empty(B, H, T, dtype=torch.float32, device=Q.device)
        ws = ops._ws(dims, L.SSA_OP_SPARSE_FWD, Q.device)
        # the call builds its own inverse index: the timed forward includes it
        call = lambda: L.ssa_sparse_attn_fwd(dims, Q, K, V, idx, Os, lse, ws)
        for _ in range(args.warmup):
            call()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record()
        for _ in range(args.steps):
            call()
        b.record()
        torch.cuda.synchronize()
        ms = a.elapsed_time(b) / args.steps
        delta = ops.dropped_mass(dims, lse, lf).float()
        gap = torch.linalg.vector_norm(Of.float() - Os.float(), dim=-1)
        ratio = gap / (2 * delta.clamp(min=1e-30) * vmax)
        ratio = torch.where(delta > 1e-6, ratio, torch.zeros_like(ratio))  # rows with nothing dropped
        fl = flops(B, H, T, d, s, k)[0]
        print(json.dumps({"sweep": "sparse fwd, T=%d H=%d s=%d" % (T, H, s), "k": k, "receptive_field": k * s,
                          "sparse_fwd_ms": ms, "tokens_per_s": B * T / (ms / 1e3), "tflops": fl / (ms / 1e3) / 1e12,
                          "delta_mean": float(delta.mean()), "delta_p99": float(torch.quantile(delta.flatten()[::97], 0.99)),
                          "delta_max": float(delta.max()), "bound_ratio_max": float(ratio.max()),
                          "device_error": L.ssa_get_device_error()}), flush=True)
        del idx, Os, lse, ws
        torch.cuda.empty_cache()


def union(args):
    """Union of the selected blocks of a 128-query tile, per workload, from the GPU's own selections: the blocks a
    query-tile kernel with row masks would have to load, against the causal blocks it covers (full attention) and
    the blocks any one query attends (k).  One JSON line per workload."""
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import build, inputs, ops
    build.build()
    for name in ("prefill", "train", "long", "sweep"):
        wl = inputs.WORKLOADS[name]
        H = min(wl.H, 4)  # heads are independent: four are enough for the distribution
        g = inputs.generate(wl, H=H)
        Q = torch.from_numpy(g["Q"].view(np.int16)).view(torch.bfloat16).cuda()
        K = torch.from_numpy(g["K"].view(np.int16)).view(torch.bfloat16).cuda()
        for k in wl.k:
            dims = L.make_dims(wl.B, H, wl.T, wl.d, wl.s, k)
            idx = ops.block_select(dims, Q, ops.block_pool(dims, K)).cpu().numpy().reshape(wl.B * H, wl.T, k)
            sizes, causal = [], []
            for bh in range(wl.B * H):
                for t0 in range(0, wl.T, 128):
                    sel = idx[bh, t0:t0 + 128].ravel()
                    sizes.append(len(np.unique(sel[sel >= 0])))
                    causal.append((min(t0 + 128, wl.T) - 1) // wl.s + 1)
            sizes, causal = np.array(sizes), np.array(causal)
            keep = causal > k  # tiles whose queries have more blocks to choose from than k
            print(json.dumps({"union": name, "k": k, "s": wl.s, "tile": 128,
                              "mean_union_blocks": float(sizes.mean()), "p50": float(np.median(sizes)),
                              "max": int(sizes.max()),
                              "mean_union_over_causal": float((sizes[keep] / causal[keep]).mean()) if keep.any() else None,
                              "mean_union_over_k": float((sizes[keep] / k).mean()) if keep.any() else None}),
                  flush=True)
        del Q, K
        torch.cuda.empty_cache()


def _time(fn, steps, warmup):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def extras(args):
    """The rows beside the training path, one JSON line each: grouped-query sparse attention fwd+bwd at 32K
    (H = 32 query heads on Hkv = 8 key/value heads), sparse decoding over a 32K cache (64 sequences), and the
    rotary-position pass."""
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import build, inputs, ops
    build.build()
    hbm, _, peak_sust, _ = measured_peaks()
    wl = inputs.WORKLOADS[WORKLOAD]
    B, H, T, d, s, k = wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL
    # ---- grouped-query sparse attention: same FLOPs as 32 heads, 8 key/value heads
    Hkv = 8
    g = inputs.group_kv(inputs.generate(wl), Hkv)
    dev = {key: torch.from_numpy(g[key].view(np.int16)).view(torch.bfloat16).cuda() for key in ("Q", "K", "V", "dO")}
    dims = L.make_dims(B, H, T, d, s, k, Hkv=Hkv)
    st = ops.SSAStep(dims, main="sparse", grad_fp32=True)
    st.forward(dev["Q"], dev["K"], dev["V"])
    Q, K, V = dev["Q"], dev["K"], dev["V"]

    def sparse_call():
        L.ssa_sparse_index(dims, st.idx, st.index)
        L.ssa_sparse_attn_fwd(dims, Q, K, V, st.idx, st.Os, st.lse_s, st.ws[L.SSA_OP_SPARSE_FWD], O_lo=st.Os_lo,
                              index=st.index)
        L.ssa_sparse_attn_bwd(dims, Q, K, V, st.Os, st.lse_s, dev["dO"], st.idx, st.dQ, st.dK, st.dV,
                              L.SSA_BWD_GRAD_FP32, st.ws[L.SSA_OP_SPARSE_BWD], O_lo=st.Os_lo, index=st.index)
    ms = _time(sparse_call, args.steps, args.warmup)
    sf, sb, _, _ = flops(B, H, T, d, s, k)
    print(json.dumps({"extra": "gqa sparse attention fwd+bwd", "B": B, "H": H, "Hkv": Hkv, "T": T, "k": k,
                      "ms": ms, "tokens_per_s": B * T / (ms / 1e3), "tflops": (sf + sb) / (ms / 1e3) / 1e12,
                      "frac_of_peak": (sf + sb) / (ms / 1e3) / 1e12 / peak_sust,
                      "device_error": L.ssa_get_device_error()}), flush=True)
    del st, dev, Q, K, V
    torch.cuda.empty_cache()
    # ---- sparse decoding: 64 sequences, caches of 32768 tokens, new tokens at random lengths
    Bd = 64
    call, nbytes, wl = decode_workload(Bd, d, s, k)
    ms = _time(call, args.steps, args.warmup)
    print(json.dumps({"extra": "sparse decode", **wl, "ms": ms, "tokens_per_s": Bd / (ms / 1e3),
                      "gbs": nbytes / (ms / 1e3) / 1e9, "frac_of_hbm": nbytes / (ms / 1e3) / 1e9 / hbm,
                      "device_error": L.ssa_get_device_error()}), flush=True)
    del call
    torch.cuda.empty_cache()
    # ---- rotary positions on Q of the 32K workload (one read and one write)
    X = torch.randn((B, H, T, d), device="cuda").to(torch.bfloat16)
    rdims = L.make_dims(B, H, T, d, s, k)
    ms = _time(lambda: L.ssa_rope(rdims, X, H, 0, 500000.0, 4.0, 0), args.steps, args.warmup)
    print(json.dumps({"extra": "rope", "B": B, "H": H, "T": T, "ms": ms,
                      "gbs": 2 * X.numel() * 2 / (ms / 1e3) / 1e9,
                      "frac_of_hbm": 2 * X.numel() * 2 / (ms / 1e3) / 1e9 / hbm,
                      "device_error": L.ssa_get_device_error()}), flush=True)


def config_block(wl):
    return {"workload": "long-context fwd+bwd, both streams + alignment: B=%d H=%d T=%d d=%d s=%d k=%d, sink block"
                        % (wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL),
            "B": wl.B, "H": wl.H, "T": wl.T, "d": wl.d, "s": wl.s, "k": K_SEL, "global_batch": wl.B, "seq_len": wl.T,
            "parallelism": "replicas", "main_stream": "alternating full/sparse per step",
            "l2": "inputs larger than L2 (Q, K, V, dO 268 MB each)",
            "value_is": "sparse attention fwd+bwd tokens/s (inverse index + forward + backward calls, CUDA events "
                        "inside the timed region)",
            "gradients": "fp32 dQ, dK, dV (both streams summed in fp32); bf16 inputs and outputs"}


def ours(args, rank, world, local_rank):
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import build, inputs, ops

    build.build()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = inputs.WORKLOADS[WORKLOAD]
    g = inputs.generate(wl)
    host = {}
    for key in ("Q", "K", "V", "dO"):
        t = torch.from_numpy(g[key].view(np.int16)).view(torch.bfloat16)
        host[key] = t.pin_memory()
    d = {key: host[key].to(dev, non_blocking=False) for key in host}
    dims = L.make_dims(wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL, dtype="bf16")
    # fp32 gradients: the two streams' contributions to dQ, dK, dV are summed without rounding the first
    steps = [ops.SSAStep(dims, device=dev, main="full", grad_fp32=True),
             ops.SSAStep(dims, device=dev, main="sparse", grad_fp32=True)]
    G32 = L.SSA_BWD_GRAD_FP32
    # the two steps share no buffers: allocate once, reuse alternately
    stream = torch.cuda.current_stream(dev)

    names = ("pool", "select", "index", "full_fwd", "sparse_fwd", "align_fwd", "align_bwd", "full_bwd", "sparse_bwd")
    n_ev = max(args.steps, 1)
    ev = {name: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_ev)]
          for name in names}

    def run_step(i, timed=False):
        st = steps[i % 2]
        Q, K, V = d["Q"], d["K"], d["V"]
        dd = st.dims

        def rec(name, fn):
            if timed:
                ev[name][i][0].record(stream)
            fn()
            if timed:
                ev[name][i][1].record(stream)

        rec("pool", lambda: L.ssa_block_pool(dd, K, st.Kbar))
        rec("select", lambda: L.ssa_block_select(dd, Q, st.Kbar, st.idx))
        rec("index", lambda: L.ssa_sparse_index(dd, st.idx, st.index))
        rec("full_fwd", lambda: L.ssa_full_attn_fwd(dd, Q, K, V, st.Of, st.lse_f, st.ws[L.SSA_OP_FULL_FWD],
                                                    O_lo=st.Of_lo))
        rec("sparse_fwd", lambda: L.ssa_sparse_attn_fwd(dd, Q, K, V, st.idx, st.Os, st.lse_s,
                                                        st.ws[L.SSA_OP_SPARSE_FWD], O_lo=st.Os_lo, index=st.index))
        rec("align_fwd", lambda: L.ssa_align_loss_fwd(dd, st.Of, st.Os, 1.0, 1.0, 1.0, st.loss,
                                                      st.ws[L.SSA_OP_ALIGN_FWD]))
        st.main_grad_buffer().copy_(d["dO"], non_blocking=True)  # upstream gradient of the main stream
        acc = L.SSA_ACC_OF if st.main == "full" else L.SSA_ACC_OS
        rec("align_bwd", lambda: L.ssa_align_loss_bwd(dd, st.Of, st.Os, 1.0, 1.0, 1.0, st.dloss, st.dOf, st.dOs,
                                                      acc))
        rec("full_bwd", lambda: L.ssa_full_attn_bwd(dd, Q, K, V, st.Of, st.lse_f, st.dOf, st.dQ, st.dK, st.dV, G32,
                                                    st.ws[L.SSA_OP_FULL_BWD], O_lo=st.Of_lo))
        rec("sparse_bwd", lambda: L.ssa_sparse_attn_bwd(dd, Q, K, V, st.Os, st.lse_s, st.dOs, st.idx, st.dQ, st.dK,
                                                        st.dV, L.SSA_BWD_ACCUMULATE | G32,
                                                        st.ws[L.SSA_OP_SPARSE_BWD], O_lo=st.Os_lo, index=st.index))

    dist = None
    if world > 1:
        import torch.distributed as dist

    def barrier():
        if dist is not None:
            dist.barrier()

    for i in range(args.warmup):
        run_step(i)
    torch.cuda.synchronize(dev)
    if L.ssa_get_device_error() != L.SSA_OK:
        raise RuntimeError("device error during warm-up")

    # ---- timed region: K whole steps, inputs resident in HBM; every call bracketed by events ----
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(args.steps):
            run_step(i, timed=True)
        end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    ms = start.elapsed_time(end)
    clocks = clk.summary()
    op_ms_sum = {name: sum(a.elapsed_time(b) for a, b in ev[name][:args.steps]) for name in names}
    sparse_ms_sum = op_ms_sum["index"] + op_ms_sum["sparse_fwd"] + op_ms_sum["sparse_bwd"]

    # Pooling bandwidth from back-to-back launches (also reported from the in-step events above).
    # K (268 MB) exceeds L2, so every launch streams it from HBM.
    pa, pb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    pa.record(stream)
    for _ in range(10):
        L.ssa_block_pool(steps[0].dims, d["K"], steps[0].Kbar)
    pb.record(stream)
    torch.cuda.synchronize(dev)
    pool_b2b_ms = pa.elapsed_time(pb) / 10

    # ---- end to end, through the same calls with host buffers: each step copies Q, K, V, dO from pinned
    # host memory, runs the sparse path (pool, select, index, sparse forward, sparse backward) and copies
    # its results O, dQ, dK, dV back to pinned host memory.  Heads are independent through the whole path,
    # so the step runs over E2E_GROUPS groups of heads on three streams: a group's inputs are copied in on
    # one, its sparse path runs on the second, its results leave on the third, and the copies of one group
    # overlap the work and the copies of the others (events keep a group's inputs until its path has read
    # them and its results until they have left) ----
    BH = wl.B * wl.H
    ng = E2E_GROUPS if BH % E2E_GROUPS == 0 else 1
    hg = BH // ng
    gdims = L.make_dims(1, hg, wl.T, wl.d, wl.s, K_SEL, dtype="bf16")
    gst = ops.SSAStep(gdims, device=dev, main="sparse", grad_fp32=True)  # a group's scratch, reused in turn
    flat = lambda t: t.view(BH, wl.T, wl.d)  # noqa: E731
    dev_in = {key: flat(d[key]) for key in ("Q", "K", "V", "dO")}
    dev_out = {"O": flat(torch.empty_like(d["Q"]))}
    dev_out.update({key: flat(torch.empty(d["Q"].shape, dtype=torch.float32, device=dev)) for key in ("dQ", "dK", "dV")})
    host_in = {key: flat(host[key]) for key in dev_in}
    host_out = {"O": flat(torch.empty_like(host["Q"]).pin_memory())}
    host_out.update({key: flat(torch.empty(host["Q"].shape, dtype=torch.float32).pin_memory())
                     for key in ("dQ", "dK", "dV")})
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in, ev_comp, ev_out = ([torch.cuda.Event() for _ in range(ng)] for _ in range(3))

    def e2e_step():
        for g in range(ng):
            sl = slice(g * hg, (g + 1) * hg)
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_comp[g])  # the previous step's path has read this group's inputs
                for key in dev_in:
                    dev_in[key][sl].copy_(host_in[key][sl], non_blocking=True)
                ev_in[g].record(s_in)
            with torch.cuda.stream(s_comp):
                s_comp.wait_event(ev_in[g])
                s_comp.wait_event(ev_out[g])  # the previous step's results of this group have left
                Q, K, V, dO = (dev_in[key][sl] for key in ("Q", "K", "V", "dO"))
                O, dQ, dK, dV = (dev_out[key][sl] for key in ("O", "dQ", "dK", "dV"))
                L.ssa_block_pool(gdims, K, gst.Kbar)
                L.ssa_block_select(gdims, Q, gst.Kbar, gst.idx)
                L.ssa_sparse_index(gdims, gst.idx, gst.index)
                L.ssa_sparse_attn_fwd(gdims, Q, K, V, gst.idx, O, gst.lse_s, gst.ws[L.SSA_OP_SPARSE_FWD],
                                      O_lo=gst.Os_lo, index=gst.index)
                L.ssa_sparse_attn_bwd(gdims, Q, K, V, O, gst.lse_s, dO, gst.idx, dQ, dK, dV, G32,
                                      gst.ws[L.SSA_OP_SPARSE_BWD], O_lo=gst.Os_lo, index=gst.index)
                ev_comp[g].record(s_comp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[g])
                for key in dev_out:
                    host_out[key][sl].copy_(dev_out[key][sl], non_blocking=True)
                ev_out[g].record(s_out)

    e2e_step()  # untimed: first use of the streams and the group's buffers
    torch.cuda.synchronize(dev)
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e_start.record(stream)
    for s_ in (s_in, s_comp, s_out):
        s_.wait_event(e_start)
    for i in range(args.steps):
        e2e_step()
    for s_ in (s_in, s_comp, s_out):
        done = torch.cuda.Event()
        done.record(s_)
        stream.wait_event(done)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    e_ms = e_start.elapsed_time(e_end)
    # the pipelined path's sparse output must equal the timed steps' (the forward is deterministic per head): a
    # missing dependency between the streams would show here
    e2e_o_diff = (dev_out["O"].float() - flat(steps[1].Os).float()).abs().max().item()
    if L.ssa_get_device_error() != L.SSA_OK:
        raise RuntimeError("device error during timing")

    ms, e_ms, sparse_ms_sum = max_over_ranks([ms, e_ms, sparse_ms_sum], dev)
    if rank != 0:
        return

    hbm, peak_burst, peak_sust, peak_kind = measured_peaks()
    sf, sb, ff, fb = flops(wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL)
    ms_step = ms / args.steps
    sparse_ms = sparse_ms_sum / args.steps
    value = whole_job_tokens_per_s(wl.B * wl.T, world, sparse_ms)
    op_ms = {name: v / args.steps for name, v in op_ms_sum.items()}
    full_ms = op_ms["full_fwd"] + op_ms["full_bwd"]
    op_flops = {"full_fwd": ff, "full_bwd": fb, "sparse_fwd": sf, "sparse_bwd": sb}
    # Dominant call of the step: the full-attention backward.  DRAM bytes per launch of its kernel from
    # one ncu capture of this build on an 8-head case of the same workload (heads are independent units
    # of the grid, so the traffic scales by the head count to the benchmarked launch); None when no
    # capture of the current kernel exists.
    traffic = FULL_BWD_DRAM_BYTES_PER_HEAD * wl.H if FULL_BWD_DRAM_BYTES_PER_HEAD else None
    roof = {"kernel": "ssa_full_attn_bwd call (attn_bwd_kernel, prep, dQ conversion)", "bound": "tensor",
            "achieved": fb / (op_ms["full_bwd"] / 1e3) / 1e12, "peak": peak_sust,
            "unit": "TFLOP/s", "traffic": traffic, "traffic_unit": "DRAM bytes per launch (ncu)",
            "peak_basis": "%s bf16 dense, sustained (kernel timed inside a long step)" % peak_kind}
    roof["frac"] = roof["achieved"] / roof["peak"]
    sparse_tflops = (sf + sb) / (sparse_ms / 1e3) / 1e12
    sel_bytes = wl.B * wl.H * wl.T * (2 * wl.d + 4 * K_SEL)
    pool_bytes = wl.B * wl.H * wl.T * 2 * wl.d
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config_block(wl),
        "sparse_attn": {"fwd_bwd_ms": sparse_ms, "tflops": sparse_tflops,
                        "tflops_exact_attended": 3.5 * exact_attended_flops(wl.B, wl.H, wl.T, wl.d, wl.s, K_SEL)
                        / (sparse_ms / 1e3) / 1e12,
                        "frac_of_peak": sparse_tflops / peak_sust, "frac_of_burst_peak": sparse_tflops / peak_burst,
                        "tokens_per_s": wl.B * wl.T / (sparse_ms / 1e3), "flop_per_step": sf + sb,
                        "calls": "ssa_sparse_index + ssa_sparse_attn_fwd + ssa_sparse_attn_bwd (accumulating)"},
        "step_tokens_per_s": whole_job_tokens_per_s(wl.B * wl.T, world, ms_step),
        "full_attn": {"fwd_bwd_ms": full_ms, "tflops": (ff + fb) / (full_ms / 1e3) / 1e12,
                      "frac_of_peak": (ff + fb) / (full_ms / 1e3) / 1e12 / peak_sust},
        "op_ms": op_ms,
        "select_hbm": {"gbs": sel_bytes / (op_ms["select"] / 1e3) / 1e9,
                       "frac": sel_bytes / (op_ms["select"] / 1e3) / 1e9 / hbm,
                       "frac_of_nominal_8tbs": sel_bytes / (op_ms["select"] / 1e3) / 1e9 / 8000.0},
        "pool_hbm": {"gbs": pool_bytes / (op_ms["pool"] / 1e3) / 1e9,
                     "frac": pool_bytes / (op_ms["pool"] / 1e3) / 1e9 / hbm, "ms": op_ms["pool"],
                     "timing": "in-step CUDA events",
                     "back_to_back": {"ms": pool_b2b_ms, "gbs": pool_bytes / (pool_b2b_ms / 1e3) / 1e9,
                                      "frac": pool_bytes / (pool_b2b_ms / 1e3) / 1e9 / hbm}},
        "roofline": roof,
        "e2e": {"value": whole_job_tokens_per_s(wl.B * wl.T, world, e_ms / args.steps), "unit": "tokens/s",
                "h2d_bytes_per_step": sum(host[k].numel() * 2 for k in host),
                "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in host_out.values()),
                "path": "pool, select, index, sparse fwd, sparse bwd with Q, K, V, dO copied in and O, dQ, dK, dV "
                        "copied out every step, over %d head groups on three streams (copy in, sparse path, "
                        "copy out)" % ng,
                "o_max_abs_diff_vs_timed_steps": e2e_o_diff},
        "gpu_launches": args.steps * (ops.SSAStep.KERNELS_FWD + steps[0].kernels_bwd()),
        "clocks": clocks,
    }
    if not args.no_cpu_baseline:
        try:
            import oracle
            oracle.build()
            dt, fl, desc = oracle_sample(args.ref_tokens)
            line["cpu_baseline"] = {"value": wl.B * wl.T / (dt * (sf + sb) / fl), "unit": "tokens/s",
                                    "cores": oracle.num_threads(), "kind": "oracle",
                                    "sample": desc + "; %.2f s" % dt, "extrapolated": True}
        except Exception as e:  # the baseline never blocks the GPU number
            line["cpu_baseline"] = {"value": None, "unit": "tokens/s", "cores": None, "kind": "oracle",
                                    "sample": "failed: %s" % e}
    print(json.dumps(line), flush=True)


def decode_workload(Bd, d=128, s=128, k=16, Hd=32, Hk=8, Td=32768, seed=5):
    """Sparse decoding over key/value caches: Bd sequences with caches of Td tokens (Hk key/value heads, Hd
    query heads), the new token at a random length in [Td/2, Td).  Returns the decode call, the bytes it must
    read (the pooled keys of the complete blocks and the selected blocks' keys and values) and the workload's
    description."""
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import ops

    ddims = L.make_dims(Bd, Hd, Td, d, s, k, Hkv=Hk)
    rng = np.random.default_rng(seed)
    lens = torch.from_numpy(rng.integers(Td // 2, Td, size=Bd).astype(np.int32)).cuda()
    Kc = torch.randn((Bd, Hk, Td, d), device="cuda").mul_(d ** -0.25).to(torch.bfloat16)
    Vc = torch.randn((Bd, Hk, Td, d), device="cuda").mul_(d ** -0.25).to(torch.bfloat16)
    q = torch.randn((Bd, Hd, d), device="cuda").mul_(d ** -0.25).to(torch.bfloat16)
    Kbar = ops.block_pool(ddims, Kc)
    idx = torch.empty((Bd, Hk, k), dtype=torch.int32, device="cuda")
    o = torch.empty((Bd, Hd, d), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((Bd, Hd), dtype=torch.float32, device="cuda")
    ws = ops._ws(ddims, L.SSA_OP_DECODE, "cuda")
    Ls = lens.cpu().numpy().astype(np.int64)
    nbytes = float(sum(Hk * ((L_ // s) * d * 4 + min(k * s, L_ + 1) * d * 2 * 2) for L_ in Ls))

    def call():
        L.ssa_sparse_decode(ddims, lens, q, Kc, Vc, Kbar, idx, o, lse, ws)
    return call, nbytes, {"sequences": Bd, "H": Hd, "Hkv": Hk, "cache": Td, "k": k}


def single_op(args):
    """One library call at a chosen size, timed with CUDA events (for profiling runs)."""
    import torch
    from block_top_sparse_b200 import _lib as L
    from block_top_sparse_b200 import build, inputs, ops

    build.build()
    if args.op == "decode":  # args.sequences sequences over caches of 32768 tokens (8 key/value heads, G = 4)
        call, nbytes, wl = decode_workload(args.sequences)
        ms = _time(call, args.steps, args.warmup)
        print(json.dumps({"op": "decode", **wl, "ms": ms, "gbs": nbytes / (ms / 1e3) / 1e9,
                          "device_error": L.ssa_get_device_error()}), flush=True)
        return
    wl = inputs.WORKLOADS[args.workload]
    g = inputs.generate(wl, H=args.H or wl.H, T=args.T or wl.T, with_dO=True)
    w = g["wl"]
    k = args.k or w.k[0]
    dims = L.make_dims(w.B, w.H, w.T, w.d, w.s, k, dtype=w.dtype)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dev = {key: torch.from_numpy(g[key].view(np.int16) if w.dtype == "bf16" else g[key]).view(dt).cuda()
           for key in ("Q", "K", "V", "dO")}
    st = ops.SSAStep(dims, grad_fp32=True)
    st.forward(dev["Q"], dev["K"], dev["V"])
    st.dOf.copy_(dev["dO"])
    st.dOs.copy_(dev["dO"])
    Q, K, V = dev["Q"], dev["K"], dev["V"]
    calls = {
        "pool": lambda: L.ssa_block_pool(dims, K, st.Kbar),
        "select": lambda: L.ssa_block_select(dims, Q, st.Kbar, st.idx),
        "index": lambda: L.ssa_sparse_index(dims, st.idx, st.index),
        "full_fwd": lambda: L.ssa_full_attn_fwd(dims, Q, K, V, st.Of, st.lse_f, st.ws[L.SSA_OP_FULL_FWD],
                                                O_lo=st.Of_lo),
        "sparse_fwd": lambda: L.ssa_sparse_attn_fwd(dims, Q, K, V, st.idx, st.Os, st.lse_s,
                                                    st.ws[L.SSA_OP_SPARSE_FWD], O_lo=st.Os_lo, index=st.index),
        "full_bwd": lambda: L.ssa_full_attn_bwd(dims, Q, K, V, st.Of, st.lse_f, st.dOf, st.dQ, st.dK, st.dV,
                                                L.SSA_BWD_GRAD_FP32, st.ws[L.SSA_OP_FULL_BWD], O_lo=st.Of_lo),
        "sparse_bwd": lambda: L.ssa_sparse_attn_bwd(dims, Q, K, V, st.Os, st.lse_s, st.dOs, st.idx, st.dQ, st.dK,
                                                    st.dV, L.SSA_BWD_GRAD_FP32, st.ws[L.SSA_OP_SPARSE_BWD],
                                                    O_lo=st.Os_lo, index=st.index),
    }
    fn = calls[args.op]
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        fn()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    sf, sb, ff, fb = flops(w.B, w.H, w.T, w.d, w.s, k)
    fl = {"full_fwd": ff, "full_bwd": fb, "sparse_fwd": sf, "sparse_bwd": sb}.get(args.op)
    print(json.dumps({"op": args.op, "workload": w.name, "B": w.B, "H": w.H, "T": w.T, "k": k, "ms": ms,
                      "tflops": fl / (ms / 1e3) / 1e12 if fl else None,
                      "device_error": L.ssa_get_device_error()}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-tokens", type=int, default=16384, help="prefix length of the oracle sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true", help="the k sweep at T = 131072 (one JSON line per k)")
    ap.add_argument("--extras", action="store_true",
                    help="grouped-query sparse attention, sparse decoding and rotary positions (one line each)")
    ap.add_argument("--union", action="store_true",
                    help="size of the union of a 128-query tile's selected blocks, per workload (one line each)")
    ap.add_argument("--op", default=None,
                    choices=["pool", "select", "index", "full_fwd", "sparse_fwd", "full_bwd", "sparse_bwd", "decode"],
                    help="time one library call instead of the whole step (profiling)")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--T", type=int, default=0)
    ap.add_argument("--H", type=int, default=0)
    ap.add_argument("--k", type=int, default=0)
    ap.add_argument("--sequences", type=int, default=64, help="sequences of --op decode")
    args = ap.parse_args()
    if args.sweep:
        sweep(args)
        return
    if args.union:
        union(args)
        return
    if args.extras:
        extras(args)
        return
    if args.op:
        single_op(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
