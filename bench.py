"""Benchmark of the Sol-Attn forward on B200.

One step = one full forward (block pooling, moments + thresholds, fused
routing / exact / approximation kernel) over the Wan-2.1-14B-like
self-attention shape: B=1, H=40, L=75,600 (21x45x80 latent grid), d=128,
64-token blocks (ragged 16-token tail), C=64, beta=1.0, synthetic seeded
Fourier-feature inputs.  The same shape in the kernel's own select-all
(dense) mode gives the speedup.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
Under torchrun (N > 1) every rank runs its own batch element of the same
shape (weak scaling, no data-path collective); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sol_attn fwd ms & executed TFLOPS (% BF16 peak); speedup vs own dense mode"
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def load_traffic():
    """dram bytes per fused-kernel launch from the committed ncu summary, if that
    summary was taken on the current kernel source (else None)."""
    import hashlib
    summ = os.path.join(ROOT, "profiles", "fused_kernel_traffic.txt")
    src = os.path.join(ROOT, "block_sparse_attention_moments_b200", "csrc", "fused.cuh")
    if not os.path.exists(summ):
        return None
    fields = {}
    with open(summ) as f:
        for line in f:
            if ":" in line and not line.startswith("#"):
                key, val = line.split(":", 1)
                fields[key.strip()] = val.strip()
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()
    if fields.get("fused_cuh_sha256") != h or "dram_bytes_per_launch_full" not in fields:
        return None
    return float(fields["dram_bytes_per_launch_full"])


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join("/tmp", f"sol_attn_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.dev)], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) == 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup(n_gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    pg = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
        pg = dist
    torch.cuda.set_device(local)
    return rank, world, local, pg


def _reduce_device(pg):
    """NCCL reduces CUDA tensors; gloo (CPU tests of this path) reduces host tensors."""
    return "cuda" if pg.get_backend() == "nccl" else "cpu"


def max_over_ranks(x: float, pg) -> float:
    """Timing of a multi-GPU step: the slowest rank's (host-side reduction, not a data-path collective)."""
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], device=_reduce_device(pg), dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, pg) -> float:
    if pg is None:
        return x
    import torch
    t = torch.tensor([x], device=_reduce_device(pg), dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.SUM)
    return float(t.item())


WORKLOAD_TEXT = {
    "tiny": "tiny check B=1 H=1 L=1024 (4x16x16) d=64",
    "small": "small B=1 H=2 L=4096 (4x32x32) d=128",
    "image": "image-generation shape B=2 H=24 L=16384 (1x128x128) d=128",
    "wan": "Wan-2.1-14B-like self-attention B=1 H=40 L=75600 (21x45x80) d=128",
    "hunyuan": "HunyuanVideo-13B-like self-attention B=1 H=24 L=118800 (33x45x80) d=128",
}


def rank_inputs(wl, rank: int):
    """bf16 bits of this rank's batch element: heads b*H .. b*H+H-1 of a batch of world size."""
    import dataclasses

    from synth import fourier_inputs
    big = dataclasses.replace(wl, B=rank + 1)
    heads = list(range(rank * wl.H, (rank + 1) * wl.H))
    q, k, v = fourier_inputs(big, heads=heads)
    return q[rank:rank + 1], k[rank:rank + 1], v[rank:rank + 1]


def cpu_baseline(wl, beta: float, budget_rows: int):
    """The fp64 oracle, as it stands, on a bounded sample: one head, `budget_rows`
    query blocks spread over the sequence (plus that head's pooling and moments)."""
    import numpy as np

    from oracle import sol_attn_head
    from synth import bf16_bits_to_f64, fourier_inputs
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count() or 1
    q, k, v = fourier_inputs(wl, heads=[0])
    q, k, v = (bf16_bits_to_f64(x[0, 0]) for x in (q, k, v))
    rows = sorted(set(np.linspace(0, wl.N - 1, budget_rows).astype(int).tolist()))
    t0 = time.perf_counter()
    r = sol_attn_head(q, k, v, beta, rows=rows)
    dt = time.perf_counter() - t0
    d, N = wl.d, wl.N
    approx = not math.isinf(beta)
    flops = sum(4.0 * 64 * 64 * d * int(r["counts"][i]) + (4.0 * 64 * d * N if approx else 0) + 2.0 * d * N
                for i in rows)
    return {"value": flops / dt / 1e12, "unit": "TFLOPS", "cores": int(cores), "kind": "oracle",
            "sample": f"1 of {wl.B * wl.H} heads, {len(rows)} of {N} query blocks (fp64 numpy, incl. that head's "
                      f"pooling and moments), {dt:.1f} s", "seconds": dt, "flops": flops}


def run_reference(args):
    """Reference arm: the fp64 CPU oracle timed on the host cores (rank 0 only)."""
    from synth import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        cpu_baseline(wl, args.beta, 4)
    vals, secs, flops = [], 0.0, 0.0
    cb = None
    for _ in range(args.steps):
        cb = cpu_baseline(wl, args.beta, args.ref_rows)
        secs += cb["seconds"]
        flops += cb["flops"]
    value = flops / secs / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} H={wl.H} L={wl.L} d={wl.d} block=64 C={wl.chunk} beta={args.beta}",
                   "sample_per_step": cb["sample"] if cb else None},
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cb["cores"] if cb else None, "kind": "oracle",
                         "sample": cb["sample"] if cb else None},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_role_profile(args):
    """Per-role cycle accounting of the fused kernel (profiling build; not a bench line)."""
    os.environ["SOL_ATTN_PROFILE"] = "1"
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    qb, kb, vb = rank_inputs(wl, 0)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    for beta, flags, tag in ((args.beta, 0, "sparse"), (-math.inf, sa.FLAG_SELECT_ALL, "dense")):
        for _ in range(args.warmup):
            sa.forward(q, k, v, beta, wl.chunk, flags=flags)
        sa.profile_read(reset=True)
        sa.forward(q, k, v, beta, wl.chunk, flags=flags)
        prof = sa.profile_read(reset=True)
        tiles = max(prof["softmax.tiles"], 1)
        per_cta = {k2: v2 / nsm for k2, v2 in prof.items()}
        print(json.dumps({"workload": wl.name, "mode": tag, "ctas": nsm, "tiles_per_cta": tiles / nsm,
                          "cycles_per_cta": {k2: round(v2) for k2, v2 in per_cta.items()},
                          # per tile of the owning warpgroup (each warpgroup takes every other tile)
                          "softmax_cycles_per_own_tile": {k2: round(prof[k2] / tiles, 1) for k2 in
                                                          ("softmax.wait_desc", "softmax.wait_s", "softmax.pass",
                                                           "softmax.wait_handoff", "softmax.meet",
                                                           "softmax.wait_o", "softmax.epilogue",
                                                           "softmax.wait_exchange", "softmax.tmem_load",
                                                           "softmax.exp_block")},
                          "issuer_cycles_per_tile": {k2: round(prof[k2] / tiles, 1) for k2 in
                                                     ("s.issue", "s.wait_buffer", "s.wait_k", "s.wait_desc",
                                                      "pv.issue", "pv.wait_p", "pv.wait_v", "pv.wait_desc")},
                          "other_roles_cycles_per_tile": {k2: round(prof[k2] / tiles, 1) for k2 in
                                                          ("sched.walk", "sched.descriptor", "sched.wait_ring",
                                                           "route.item", "route.wait_item_empty", "k.wait_stage",
                                                           "v.wait_stage")},
                          "rescales": prof["softmax.rescales"]}), flush=True)


def run_ablation(args):
    """Approximation ablation (not a bench line): for each beta, the output of the
    full method, of its first-order extension and of the exact-only variant (no
    approximation of unselected blocks, same selection) against the select-all
    output of the same kernel, as relative l2 error and mean per-row cosine
    similarity.  "Sol-Attn: ...",
    experiments: ablation of the proxy-score approximation."""
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    qb, kb, vb = rank_inputs(wl, 0)
    if args.ablation_keys == "near-block-constant":
        from synth import near_block_constant_keys
        kb = near_block_constant_keys(kb, 0.1, seed=73)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    dense = sa.forward(q, k, v, -math.inf, wl.chunk, flags=sa.FLAG_SELECT_ALL).float()

    def compare(o):
        o = o.float()
        rel = (torch.linalg.vector_norm(o - dense) / torch.linalg.vector_norm(dense)).item()
        cos = torch.nn.functional.cosine_similarity(o.reshape(-1, o.shape[-1]), dense.reshape(-1, o.shape[-1]),
                                                    dim=-1).mean().item()
        return rel, cos

    for beta in args.ablation_betas:
        o_full = sa.forward(q, k, v, beta, wl.chunk)
        counts = sa.stats(wl.B, wl.H, wl.L)
        density = counts.double().mean().item() / counts.shape[-1]
        o_exact = sa.forward(q, k, v, beta, wl.chunk, flags=sa.FLAG_EXACT_ONLY)
        o_first = sa.forward(q, k, v, beta, wl.chunk, flags=sa.FLAG_FIRST_ORDER)
        rf, cf = compare(o_full)
        re, ce = compare(o_exact)
        r1, c1 = compare(o_first)
        print(json.dumps({"mode": "ablation", "workload": wl.name, "keys": args.ablation_keys, "beta": beta,
                          "density": density,
                          "approx": {"rel_l2_vs_dense": rf, "cosine_vs_dense": cf},
                          "first_order": {"rel_l2_vs_dense": r1, "cosine_vs_dense": c1},
                          "exact_only": {"rel_l2_vs_dense": re, "cosine_vs_dense": ce}}), flush=True)


def run_density(args):
    """Per-row density report (not a bench line): for each beta, the distribution
    of |S_i| / N over all query blocks of the workload from sol_attn_stats, as a
    10-bin histogram with mean, quartiles and extremes.  "Sol-Attn: ...",
    experiments: per-row sparsity of the adaptive threshold (Fig. 7)."""
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    qb, kb, vb = rank_inputs(wl, 0)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    for beta in args.ablation_betas:
        sa.forward(q, k, v, beta, wl.chunk)
        counts = sa.stats(wl.B, wl.H, wl.L)
        dens = (counts.double() / counts.shape[-1]).flatten().cpu().numpy()
        hist, edges = np.histogram(dens, bins=10, range=(0.0, 1.0))
        print(json.dumps({"mode": "density", "workload": wl.name, "beta": beta, "rows": int(dens.size),
                          "mean": float(dens.mean()), "min": float(dens.min()), "max": float(dens.max()),
                          "quartiles": [float(x) for x in np.quantile(dens, [0.25, 0.5, 0.75])],
                          "histogram": {"edges": [round(float(e), 2) for e in edges], "counts": hist.tolist()}}),
              flush=True)


def run_chunk_sweep(args):
    """Chunk-size sweep (not a bench line): the forward at several C, each against
    the workload's own C: max |difference| of the outputs (C changes only the
    order of the online-softmax updates, so only rounding) and the time per call.
    "Sol-Attn: ...", experiments: setup (C affects efficiency, not the output)."""
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    qb, kb, vb = rank_inputs(wl, 0)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    ref = sa.forward(q, k, v, args.beta, wl.chunk).float()
    for C in args.chunks:
        for _ in range(2):
            o = sa.forward(q, k, v, args.beta, C)
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for _ in range(3):
            o = sa.forward(q, k, v, args.beta, C)
        t1.record()
        torch.cuda.synchronize()
        diff = (o.float() - ref).abs().max().item()
        print(json.dumps({"mode": "chunk_sweep", "workload": wl.name, "beta": args.beta, "chunk": C,
                          "ms_per_call": t0.elapsed_time(t1) / 3, "max_abs_diff_vs_default_chunk": diff}),
              flush=True)


def run_speedup_sweep(args):
    """Speedup over the kernel's own select-all (dense) mode across sequence
    lengths and sparsity levels (not a bench line): per length L, bf16
    Fourier-feature inputs on a (L/4096) x 64 x 64 token grid, `--sweep-heads`
    heads, d = 128, C = 64; per beta the measured density (sol_attn_stats), the
    time per forward and the speedup.  L2 is flushed (256 MB write) before every
    timed call.  "Sol-Attn: ...", experiments: kernel-level speedup over dense
    attention across 16K-128K tokens and sparsity levels (Fig. 5a)."""
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import custom_fourier
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda")
    H, d, C = args.sweep_heads, 128, 64

    def time_call(fn, reps=3):
        for _ in range(2):
            fn()
        total = 0.0
        for _ in range(reps):
            flush.zero_()
            t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t0.record()
            fn()
            t1.record()
            torch.cuda.synchronize()
            total += t0.elapsed_time(t1)
        return total / reps

    for L in args.sweep_lengths:
        qb, kb, vb = custom_fourier(1, H, (max(1, L // 4096), 64, 64), d, 3.0, seed=2000 + L // 1024)
        q, k, v = dev(qb), dev(kb), dev(vb)
        Lr = q.shape[2]
        N = -(-Lr // sa.BLOCK)
        dense_ms = time_call(lambda: sa.forward(q, k, v, -math.inf, C, flags=sa.FLAG_SELECT_ALL))
        for beta in args.sweep_betas:
            ms = time_call(lambda: sa.forward(q, k, v, beta, C))
            counts = sa.stats(1, H, Lr)
            pairs = int(counts.to(torch.int64).sum().item())
            density = pairs / (H * N * N)
            tflops = sa.executed_flops(pairs, 1, H, Lr, d, approx=True) / (ms * 1e-3) / 1e12
            print(json.dumps({"mode": "speedup_sweep", "L": Lr, "heads": H, "beta": beta,
                              "density": round(density, 4), "sparsity": round(1.0 - density, 4),
                              "ms_per_call": ms, "dense_ms_per_call": dense_ms,
                              "speedup_vs_dense": dense_ms / ms, "executed_tflops": tflops}), flush=True)
        del q, k, v


def run_routing_cost(args):
    """Routing-cost report (not a bench line): the method's routing against a
    materialised top-k router, on the workload's shape.  "Sol-Attn: ...",
    experiments: routing latency against top-k / top-p routers that materialise
    and traverse the proxy map (Fig. 5b/5c).

    method  exposed: the moment kernels (key mean and covariance, then mu_i,
            sigma_i and tau_i for every query block; CUDA events).  The routing
            dot products and threshold tests run inside the fused kernel beside
            its tiles; their routing-warp busy cycles (profiling build), summed
            over the SMs and divided by SMs x SM clock, are reported apart.
    top-k   the whole proxy map of every head written to HBM, then each row's
            k largest blocks selected (k = the row-average |S_i| of the method
            at this beta, so both keep the same number of blocks); CUDA events.
    Workspace bytes of each are reported beside the times."""
    os.environ["SOL_ATTN_PROFILE"] = "1"
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    wl = WORKLOADS[args.workload]
    qb, kb, vb = rank_inputs(wl, 0)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    B, H, L, d, N = 1, wl.H, wl.L, wl.d, wl.N
    nsm = torch.cuda.get_device_properties(0).multi_processor_count
    out = torch.empty_like(q)

    def timed(fn, reps=5):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    sa.stage_pool(q, k, v)
    thr_ms = timed(lambda: sa.stage_threshold(B, H, L, d, args.beta))
    # one full forward in the profiling build for the in-kernel routing cycles
    sa.forward(q, k, v, args.beta, wl.chunk)
    sa.profile_read(reset=True)
    sa.forward(q, k, v, args.beta, wl.chunk)
    prof = sa.profile_read(reset=True)
    counts = sa.stats(B, H, L)
    kk = int(round(counts.double().mean().item()))
    clk_hz = 1e6 * float(os.environ.get("SOL_ATTN_SM_MHZ", "1965"))
    route_ms = prof["route.item"] / nsm / clk_hz * 1e3
    sa.stage_pool(q, k, v)
    topk_ms = timed(lambda: sa.topk_route(B, H, L, d, kk))
    method_bytes = B * H * N * 4 + B * H * (d + d * d) * 8          # thresholds + key moments
    topk_bytes = B * H * N * N * 4                                     # the materialised map
    # The top-k router runs as its own kernels before attention can start; of
    # the method's routing only the moment kernels do, the dot products and
    # threshold tests run inside the fused kernel beside its tiles.
    print(json.dumps({"mode": "routing_cost", "workload": wl.name, "beta": args.beta, "blocks_kept_per_row": kk,
                      "method": {"exposed_ms": thr_ms, "workspace_bytes": method_bytes,
                                 "in_kernel_routing_warp_ms_equivalent": route_ms},
                      "topk_materialised": {"exposed_ms": topk_ms, "workspace_bytes": topk_bytes},
                      "exposed_time_ratio_topk_over_method": topk_ms / thr_ms,
                      "workspace_ratio_topk_over_method": topk_bytes / method_bytes,
                      "sm_clock_mhz_assumed": clk_hz / 1e6}), flush=True)


def run_all_configs(args):
    """Per-configuration report (not a bench line): for each video shape and
    beta of the workload list, and the select-all mode, the forward time (the
    three stages, CUDA events, inputs larger than L2), executed TFLOPS by the
    method's accounting, the fused kernel's fraction of the measured bf16 burst
    peak and the speedup over the same shape's select-all mode."""
    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS
    peaks, _ = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    for name in args.configs:
        wl = WORKLOADS[name]
        qb, kb, vb = rank_inputs(wl, 0)
        dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
        q, k, v = dev(qb), dev(kb), dev(vb)
        out = torch.empty_like(q)
        B, H, L, d, N = 1, wl.H, wl.L, wl.d, wl.N

        def one(beta, flags, reps):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
            tot = [0.0, 0.0, 0.0]
            for r in range(reps + 3):
                ev[0].record()
                sa.stage_pool(q, k, v)
                ev[1].record()
                sa.stage_threshold(B, H, L, d, beta, flags=flags)
                ev[2].record()
                sa.stage_fused(q, k, v, out, wl.chunk, flags=flags)
                ev[3].record()
                torch.cuda.synchronize()
                if r >= 3:
                    for i in range(3):
                        tot[i] += ev[i].elapsed_time(ev[i + 1]) / reps
            counts = sa.stats(B, H, L)
            pairs = int(counts.to(torch.int64).sum().item())
            return tot, pairs

        dense_t, dense_pairs = one(-math.inf, sa.FLAG_SELECT_ALL, 2)
        dense_ms = sum(dense_t)
        rows = [("select-all", dense_t, dense_pairs, -math.inf)]
        for beta in wl.betas:
            if math.isinf(beta):
                continue
            t, pairs = one(beta, 0, args.steps)
            rows.append((beta, t, pairs, beta))
        for label, t, pairs, beta in rows:
            ms = sum(t)
            approx = not math.isinf(beta)
            fl = sa.executed_flops(pairs, B, H, L, d, approx=approx)
            print(json.dumps({"mode": "config", "workload": wl.name, "beta": label, "density": pairs / (B * H * N * N),
                              "ms_per_forward": ms, "stage_ms": {"pool": t[0], "threshold": t[1], "fused": t[2]},
                              "executed_tflops": fl / (ms * 1e-3) / 1e12,
                              "fused_frac_of_burst_peak": fl / (t[2] * 1e-3) / 1e12 / peak,
                              "speedup_vs_select_all": dense_ms / ms}), flush=True)
        del q, k, v, out
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="wan")
    ap.add_argument("--beta", type=float, default=1.0)
    ap.add_argument("--ref-rows", type=int, default=48, help="query blocks per reference step")
    ap.add_argument("--cpu-rows", type=int, default=768, help="query blocks in the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the select-all (dense) comparison run")
    ap.add_argument("--ablation", action="store_true",
                    help="approximation ablation: full method and exact-only against select-all (not a bench line)")
    ap.add_argument("--ablation-betas", type=float, nargs="+", default=[0.75, 1.0, 1.5],
                    help="betas of --ablation and --density")
    ap.add_argument("--ablation-keys", default="fourier", choices=["fourier", "near-block-constant"],
                    help="keys of --ablation: the workload's, or each block's first key + 0.1 N(0,1)")
    ap.add_argument("--chunk-sweep", action="store_true",
                    help="outputs and times at several chunk sizes C (not a bench line)")
    ap.add_argument("--chunks", type=int, nargs="+", default=[1, 16, 64, 256, 1024])
    ap.add_argument("--density", action="store_true",
                    help="per-row density histogram from sol_attn_stats (not a bench line)")
    ap.add_argument("--speedup-sweep", action="store_true",
                    help="speedup over the select-all mode across lengths and sparsity (not a bench line)")
    ap.add_argument("--sweep-lengths", type=int, nargs="+", default=[16384, 32768, 65536, 131072])
    ap.add_argument("--sweep-betas", type=float, nargs="+", default=[0.84, 1.28, 1.64],
                    help="about 80%%, 90%% and 95%% sparsity on Gaussian proxy logits")
    ap.add_argument("--sweep-heads", type=int, default=8)
    ap.add_argument("--all-configs", action="store_true",
                    help="time, TFLOPS, fraction of peak and speedup for every video shape and beta (not a bench line)")
    ap.add_argument("--configs", nargs="+", default=["wan", "hunyuan"])
    ap.add_argument("--routing-cost", action="store_true",
                    help="method's routing against a materialised top-k router (not a bench line)")
    ap.add_argument("--role-profile", action="store_true",
                    help="run the profiling build (libsol_attn_profile.so) and print per-role cycle accounting")
    args = ap.parse_args()
    if args.role_profile:
        return run_role_profile(args)
    if args.routing_cost:
        return run_routing_cost(args)
    if args.all_configs:
        return run_all_configs(args)
    if args.ablation:
        return run_ablation(args)
    if args.density:
        return run_density(args)
    if args.speedup_sweep:
        return run_speedup_sweep(args)
    if args.chunk_sweep:
        return run_chunk_sweep(args)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    import numpy as np
    import torch

    import block_sparse_attention_moments_b200 as sa
    from synth import WORKLOADS

    rank, world, local, pg = dist_setup(args.gpus)
    wl = WORKLOADS[args.workload]
    B, H, L, d, C = 1, wl.H, wl.L, wl.d, wl.chunk
    N = wl.N
    qb, kb, vb = rank_inputs(wl, rank)
    dev = lambda x: torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    q, k, v = dev(qb), dev(kb), dev(vb)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream()
    in_bytes = 3 * B * H * L * d * 2
    # inputs that fit in L2 are evicted by a 256 MB write before every timed step
    # (outside the stage events, which then give the step time)
    flush = torch.empty(64 << 20, dtype=torch.float32, device="cuda") if in_bytes <= (126 << 20) else None

    def step(beta, flags, ev=None):
        if flush is not None:
            flush.zero_()
        if ev is None:
            sa.stage_pool(q, k, v, stream=stream)
            sa.stage_threshold(B, H, L, d, beta, flags=flags, stream=stream)
            sa.stage_fused(q, k, v, out, C, flags=flags, stream=stream)
            return
        ev[0].record(stream)
        sa.stage_pool(q, k, v, stream=stream)
        ev[1].record(stream)
        sa.stage_threshold(B, H, L, d, beta, flags=flags, stream=stream)
        ev[2].record(stream)
        sa.stage_fused(q, k, v, out, C, flags=flags, stream=stream)
        ev[3].record(stream)

    def timed(beta, flags, sampler=None):
        for _ in range(args.warmup):
            step(beta, flags)
        torch.cuda.synchronize()
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
        if pg is not None:
            pg.barrier()
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for s in range(args.steps):
            step(beta, flags, evs[s])
        end.record(stream)
        torch.cuda.synchronize()
        clocks = sampler.stop() if sampler else None
        if pg is not None:
            pg.barrier()
        total_ms = start.elapsed_time(end)
        per = [sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps for i in range(3)]
        if flush is not None:   # the flushes sit between the steps: time the stages only
            total_ms = sum(e[0].elapsed_time(e[3]) for e in evs)
        counts = sa.stats(B, H, L, stream=stream)
        torch.cuda.synchronize()
        pairs = int(counts.to(torch.int64).sum().item())
        return total_ms, per, pairs, clocks

    # sparse run (the headline) and the same kernel in select-all (dense) mode
    sampler = ClockSampler(local)
    total_ms, per_ms, pairs, clocks = timed(args.beta, 0, sampler)
    if args.no_dense:
        dense_ms, dense_pairs = float("nan"), B * H * N * N
    else:
        dense_ms, dense_per, dense_pairs, _ = timed(-math.inf, sa.FLAG_SELECT_ALL)
    flops_step = sa.executed_flops(pairs, B, H, L, d, approx=True)
    fused_flops = flops_step  # the fused kernel executes all exact, proxy and routing FLOPs
    step_ms = max_over_ranks(total_ms / args.steps, pg)
    fused_ms = max_over_ranks(per_ms[2], pg)
    all_flops = sum_over_ranks(flops_step, pg)
    dense_step_ms = max_over_ranks(dense_ms / args.steps, pg)
    value = all_flops / (step_ms * 1e-3) / 1e12

    # end to end through the host-buffer entry point (pinned host memory)
    e2e = None
    if not args.no_e2e:
        hq = torch.from_numpy(qb.view(np.int16)).pin_memory()
        hk = torch.from_numpy(kb.view(np.int16)).pin_memory()
        hv = torch.from_numpy(vb.view(np.int16)).pin_memory()
        ho = torch.empty_like(hq).pin_memory()
        for _ in range(2):
            sa.forward_host(hq, hk, hv, args.beta, C, out=ho)
        if pg is not None:
            pg.barrier()
        ksteps = max(2, min(args.steps, 5))
        t0 = time.perf_counter()
        for _ in range(ksteps):
            sa.forward_host(hq, hk, hv, args.beta, C, out=ho)
        e2e_s = max_over_ranks((time.perf_counter() - t0) / ksteps, pg)
        nbytes = q.numel() * 2
        e2e = {"value": all_flops / e2e_s / 1e12, "unit": "TFLOPS", "h2d_bytes_per_step": 3 * nbytes,
               "d2h_bytes_per_step": nbytes, "ms_per_step": e2e_s * 1e3}

    peaks, peak_src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    achieved = fused_flops / (fused_ms * 1e-3) / 1e12
    if rank != 0:
        if pg is not None:
            pg.destroy_process_group()
        return
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cb = cpu_baseline(wl, args.beta, args.cpu_rows)
        cpu = {k2: cb[k2] for k2 in ("value", "unit", "cores", "kind", "sample")}
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "TFLOPS",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: {WORKLOAD_TEXT.get(wl.name, wl.name)} per GPU, block=64 C={C} "
                               f"beta={args.beta}, bf16 Fourier-feature Q/K, Gaussian V",
                   "per_gpu_batch": 1, "global_batch": world, "seq_len": L, "parallelism": f"dp{world} (weak)",
                   "l2": (f"inputs ({in_bytes / 1e9:.2f} GB/step) larger than L2 (126 MB)" if flush is None else
                          f"inputs ({in_bytes / 1e6:.1f} MB/step) fit in L2: a 256 MB write flushes it before "
                          f"each step, outside the timed stages")},
        "ms_per_call": step_ms,
        "pct_bf16_peak": 100.0 * value / world / peak,
        "stage_ms": {"pool": per_ms[0], "threshold": per_ms[1], "fused": per_ms[2]},
        "density": pairs / (B * H * N * N),
        "dense_ms_per_call": None if args.no_dense else dense_step_ms,
        "dense_tflops": None if args.no_dense else
        sa.executed_flops(dense_pairs, B, H, L, d, approx=False) / (dense_step_ms * 1e-3) / 1e12,
        "speedup_vs_dense": None if args.no_dense else dense_step_ms / step_ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     # the committed capture covers the default workload's sparse call only
                     "traffic": load_traffic() if (wl.name == "wan" and args.beta == 1.0) else None,
                     "peak_source": f"{peak_src} bf16 burst (MEASURED_PEAKS.json)" if peak_src == "measured"
                     else "fallback 1.59 PFLOP/s", "frac_of_sustained": achieved / peak_sus,
                     "kernel": "sol_attn_fused_kernel", "algorithmic_flops_per_launch": fused_flops},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps * sa.kernels_per_forward(),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
