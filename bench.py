#!/usr/bin/env python3
"""Benchmark: sparse prefill attention layer (selection + sparse attention) on B200.

One step = one pass of the whole hot path over one attention layer of the
Llama-3.1-8B shape at L = 131072 (B = 1, 32 q heads, 8 kv heads, d = 128,
causal, bf16): ``sparse_prefill_plan`` (anchor selection, theta = 5, sink 128,
local 256) followed by ``sparse_prefill_attn``.  Inputs come from the seeded
synthetic generator of ``workloads`` (sink bias + planted needles) and are
resident in HBM before the timed region; at 1.5 GB they are larger than L2.

Metric: kept-FLOP throughput (4 * d * sum_i |K_i| per layer) in TFLOP/s over
the whole step; ``ms_per_step`` is ms per layer.  Extra keys: the attention
kernel's roofline fraction, the SALE mode and the same kernel run dense, an
end-to-end number through host buffers, clocks sampled during the timed
region, and the CPU oracle timed on a bounded sample.

Multi-GPU (``torchrun --nproc-per-node N``): every rank processes its own
layer (independent problems, weak scaling, no collective on the data path);
the timed region is bracketed by barriers and the max over ranks is reported.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only).
``--sweep`` runs the density sweep, ``--decode`` the decode steps that reuse
a plan, ``--fp8`` the E4M3 attention and ``--key-mass`` the key mass from the
prefill LSE; each prints its own JSON lines instead of the headline step.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import C2_LLAMA_128K, CONFIGS, Workload, generate  # noqa: E402

METRIC = "sparse prefill attn ms/layer @128K & kept-FLOP TFLOP/s vs bf16 peak"
UNIT = "TFLOP/s (kept FLOPs, plan+attn)"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sus=float(d["bf16_tflops_sustained"]), src="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def _kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in ("attn.cuh", "attn_pair.cuh", "common.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "block_sparse_long_sm_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def _recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu
    record, only if the kernel source is the one the counters were taken on."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
    except Exception:
        return None
    if rec.get("source_sha256") != _kernel_source_hash() or rec.get("workload") != workload:
        return None
    return rec.get("bytes_per_launch")


def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def oracle_sample(w: Workload, inp, theta: float, n_rows: int = 256):
    """CPU oracle on a bounded sample: anchor selection for the query blocks that
    hold the last ``n_rows`` rows of q head 0, then fp64 sparse attention for
    those rows (the longest rows of the layer)."""
    from oracle import attention as oatt
    from oracle import selection as osel
    from workloads import bf16_bits_to_f32
    qh = bf16_bits_to_f32(inp.q[0, 0]).astype(np.float64)
    kh = bf16_bits_to_f32(inp.k[0, 0]).astype(np.float64)
    vh = bf16_bits_to_f32(inp.v[0, 0]).astype(np.float64)
    L = w.seq_len
    rows = list(range(max(0, L - n_rows), L))
    blocks = sorted({i // 128 for i in rows})
    t0 = time.perf_counter()
    sel = {qb: osel.anchor_block(qh, kh, qb, bq=128, sink=w.sink, local=w.local,
                                 theta=theta).kept for qb in blocks}
    oatt.attend_rows(qh, kh, vh, rows, lambda i: i // 128, lambda b: sel[b], bq=128,
                     sink=w.sink, local=w.local)
    dt = time.perf_counter() - t0
    pairs = 0
    for i in rows:
        qb = i // 128
        ls = max(0, (qb + 1) * 128 - w.local)
        pairs += min(w.sink, ls) + (i + 1 - ls) + len(sel[qb])
    flops = 4 * 128 * pairs
    cores = len(os.sched_getaffinity(0))
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max((i.get("num_threads", 1) for i in info), default=cores)
    except Exception:
        pass
    return dict(value=flops / dt / 1e12, unit=UNIT, cores=cores, kind="oracle",
                sample=f"q head 0, last {len(rows)} rows of {w.name} (their query blocks' "
                       f"anchor selection + fp64 sparse attention); {dt:.1f} s",
                seconds=dt, flops=flops)


def run_reference(args, w: Workload):
    world, rank, _ = _dist()
    if rank != 0:
        return
    inp = generate(w, kv_groups=[0])
    vals = []
    for _ in range(args.warmup):
        oracle_sample(w, inp, args.theta, n_rows=16)
    for _ in range(args.steps):
        vals.append(oracle_sample(w, inp, args.theta, n_rows=16))
    v = statistics.median(x["value"] for x in vals)
    cb = dict(vals[-1])
    cb["value"] = v
    for key in ("seconds", "flops"):
        cb.pop(key, None)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": statistics.median(x["seconds"] for x in vals) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w, args),
            "cpu_baseline": cb, "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0,
                                        "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def _config(w: Workload, args, world: int = 1):
    return {"workload": w.name, "batch": w.batch, "heads_q": w.heads_q, "heads_kv": w.heads_kv,
            "seq_len": w.seq_len, "head_dim": 128, "causal": True, "mode": args.mode,
            "theta": args.theta, "sink": w.sink, "local": w.local, "block_q": 128,
            "l2": f"inputs ({2 * 128 * w.seq_len * w.batch * (w.heads_q + 2 * w.heads_kv) / 1e9:.2f} GB) "
                  + ("larger than L2 (126 MB); no flush" if w.seq_len * w.batch * (w.heads_q + 2 * w.heads_kv) * 256 > 126e6
                     else "smaller than L2"),
            "parallelism": (f"one layer split by kv head over {world} GPUs"
                            if getattr(args, "split", False) and world > 1
                            else "independent layer per GPU")}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--mode", default="anchor", choices=["anchor", "sale", "dense"])
    ap.add_argument("--theta", type=float, default=5.0)
    ap.add_argument("--config", default=C2_LLAMA_128K.name, choices=sorted(CONFIGS))
    ap.add_argument("--no-extras", action="store_true", help="skip SALE/dense/e2e/cpu legs")
    ap.add_argument("--sweep", action="store_true",
                    help="density sweep instead of the headline step: one JSON line per "
                         "(layer, theta), theta from +inf to 2, with the same kernel run dense")
    ap.add_argument("--decode", action="store_true",
                    help="decode-shaped reuse of the plan instead of the headline step: one "
                         "decoding query per q head per step at positions L-1, L, ...")
    ap.add_argument("--fp8", action="store_true",
                    help="E4M3 quantisation + FP8 attention over the plan instead of the "
                         "headline step")
    ap.add_argument("--split", action="store_true",
                    help="under torchrun, split one layer by kv head across the ranks (strong "
                         "scaling) instead of running one layer per rank (weak scaling)")
    ap.add_argument("--key-mass", action="store_true",
                    help="key mass from the prefill LSE over the plan instead of the headline step")
    args = ap.parse_args()
    w = CONFIGS[args.config]
    if args.sweep:
        sweep()
        return
    if args.decode:
        decode_bench(args, w)
        return
    if args.fp8 or args.key_mass:
        variant_bench(args, w)
        return
    if args.impl == "reference":
        run_reference(args, w)
        return

    import torch
    import torch.distributed as dist

    import block_sparse_long_sm_b200 as spa

    world, rank, local = _dist()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    inp = generate(w)
    q_h = torch.from_numpy(inp.q.view(np.int16)).view(torch.bfloat16).pin_memory()
    k_h = torch.from_numpy(inp.k.view(np.int16)).view(torch.bfloat16).pin_memory()
    v_h = torch.from_numpy(inp.v.view(np.int16)).view(torch.bfloat16).pin_memory()
    q = q_h.to(dev)
    k = k_h.to(dev)
    v = v_h.to(dev)
    B, Hq, Hkv, L = w.batch, w.heads_q, w.heads_kv, w.seq_len
    o = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device=dev)
    p = spa.make_params(B, Hq, Hkv, L, mode=args.mode, sink=w.sink, local=w.local,
                        theta=args.theta, tau=w.tau, block_k=w.block_k if args.mode == "sale" else None)
    # --split: this rank's kv heads of the one layer (all of it on one GPU)
    split = args.split and world > 1
    if split:
        from block_sparse_long_sm_b200.shard import rank_sub_layer
        sub = rank_sub_layer(p, world, rank)
        p = sub.params
        qa, ka, va, oa, _ = sub.pointers(q, k, v, o)
    else:
        qa, ka, va, oa = q, k, v, o
    ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)

    def step():
        spa.check(spa.sparse_prefill_plan(p, qa, ka, ws, stream=stream), "plan")
        spa.check(spa.sparse_prefill_attn(p, qa, ka, va, ws, oa, None, stream=stream), "attn")

    for _ in range(max(3, args.warmup)):
        step()
    st, stats = spa.sparse_prefill_stats(p, ws, stream=stream)
    spa.check(st, "stats")
    flops_step = spa.kept_flops(stats)

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            ev[i][0].record(stream)
            spa.check(spa.sparse_prefill_plan(p, qa, ka, ws, stream=stream), "plan")
            ev[i][1].record(stream)
            spa.check(spa.sparse_prefill_attn(p, qa, ka, va, ws, oa, None, stream=stream), "attn")
            ev[i][2].record(stream)
        t_end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms = t_start.elapsed_time(t_end)
    plan_ms = [a.elapsed_time(b) for a, b, _ in ev]
    attn_ms = [b.elapsed_time(c) for _, b, c in ev]
    if world > 1:
        t = torch.tensor([total_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_step = total_ms / args.steps
    layer_flops = flops_step * world            # weak: every rank runs a whole layer
    if split:
        # strong: the ranks' kept FLOPs add up to the one layer's
        t = torch.tensor([float(flops_step)], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        layer_flops = float(t.item())
    value = layer_flops * args.steps / (total_ms / 1e3) / 1e12
    peaks = _peaks()
    attn_avg = sum(attn_ms) / len(attn_ms)
    achieved = flops_step / (attn_avg / 1e3) / 1e12
    extras = {}
    # kernels per plan: anchor = pooling + fused scan/compaction (the bench uses
    # step 1); SALE = two K-mean passes, two quantisations, scan, compaction
    n_launch_plan = {"anchor": 2, "sale": 6, "dense": 0}[args.mode]
    launches = (n_launch_plan + 1) * args.steps

    if rank == 0 and not args.no_extras:
        extras = bench_extras(spa, torch, w, args, q, k, v, o, q_h, k_h, v_h, stream, dev, stats)
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": _config(w, args, world),
            "plan_ms": statistics.median(plan_ms), "attn_ms": statistics.median(attn_ms),
            "kept_fraction": stats.kept_pairs / stats.dense_pairs,
            "kept_flops_per_layer": flops_step,
            "roofline": {"bound": "tensor",
                         "kernel": "sparse_attn_pair_kernel" if (w.heads_q // w.heads_kv) % 2 == 0
                                   else "sparse_attn_kernel",
                         "achieved": achieved, "peak": peaks["bf16_sus"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_sus"],
                         "traffic": _recorded_traffic(
                             w.name, "sparse_attn_pair_kernel" if (w.heads_q // w.heads_kv) % 2 == 0
                             else "sparse_attn_kernel"),
                         "peak_source": f"{peaks['src']} bf16 dense, sustained (kernel timed inside a long loop)"},
            "clocks": clk.summary(),
            "gpu_launches": launches,
        }
        line.update(extras)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def sweep():
    """Kept fraction vs time and vs tensor peak over theta (the density sweep
    of the 128K Llama layer, its B = 4, L = 16384 variant and the 64K Qwen
    layer with half its kv heads diffuse).  One JSON line per point; theta =
    +inf is compared with DENSE mode (same kernel, every causal key)."""
    import torch
    import block_sparse_long_sm_b200 as spa
    from workloads import C3_QWEN_64K, C4_B4_16K, C4_SWEEP_128K, THETA_DENSITY_SWEEP
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    peaks = _peaks()

    def timed(fn, reps=3, warm=2):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    # theta = -inf keeps only the sink and local keys: the attention time of
    # that point is what the sink and local tiles cost inside every step
    plan = [(C4_SWEEP_128K, THETA_DENSITY_SWEEP + (-math.inf,)), (C4_B4_16K, THETA_DENSITY_SWEEP),
            (C3_QWEN_64K, (5.0,))]
    for w, thetas in plan:
        inp = generate(w)
        to = lambda u: torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).to(dev).view(torch.bfloat16)
        q, k, v = to(inp.q), to(inp.k), to(inp.v)
        del inp
        B, Hq, Hkv, L = w.batch, w.heads_q, w.heads_kv, w.seq_len
        o = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device=dev)
        pd = spa.make_params(B, Hq, Hkv, L, mode="dense", sink=w.sink, local=w.local)
        wsd = torch.empty(spa.sparse_prefill_workspace_bytes(pd), dtype=torch.uint8, device=dev)
        spa.check(spa.sparse_prefill_plan(pd, q, k, wsd, stream=stream))
        dense_ms = timed(lambda: spa.check(spa.sparse_prefill_attn(pd, q, k, v, wsd, o, None,
                                                                   stream=stream)))
        st, sd = spa.sparse_prefill_stats(pd, wsd, stream=stream)
        spa.check(st, "stats")
        del wsd
        for theta in thetas:
            p = spa.make_params(B, Hq, Hkv, L, mode="anchor", sink=w.sink, local=w.local,
                                theta=theta)
            ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)
            plan_ms = timed(lambda: spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream)))
            attn_ms = timed(lambda: spa.check(spa.sparse_prefill_attn(p, q, k, v, ws, o, None,
                                                                      stream=stream)))
            st, s = spa.sparse_prefill_stats(p, ws, stream=stream)
            spa.check(st, "stats")
            flops = spa.kept_flops(s)
            alg_bytes = 2 * B * Hq * L * 128 + 2 * B * Hkv * L * 128 + 4 * s.kept_candidates
            print(json.dumps({
                "sweep": "density", "workload": w.name, "theta": theta,
                "kept_fraction": s.kept_pairs / s.dense_pairs,
                "kept_candidates_fraction": s.kept_candidates / max(1, s.candidates),
                "plan_ms": plan_ms, "attn_ms": attn_ms, "step_ms": plan_ms + attn_ms,
                "attn_tflops": flops / (attn_ms / 1e3) / 1e12,
                "attn_frac": flops / (attn_ms / 1e3) / 1e12 / peaks["bf16_sus"],
                "selection_gbs": alg_bytes / (plan_ms / 1e3) / 1e9,
                "selection_frac": alg_bytes / (plan_ms / 1e3) / 1e9 / peaks["hbm"],
                "dense_attn_ms": dense_ms, "speedup_vs_dense": dense_ms / (plan_ms + attn_ms),
                "peak_source": peaks["src"]}), flush=True)
            del ws
        del q, k, v, o
        torch.cuda.empty_cache()


def decode_bench(args, w: Workload):
    """Decode steps that reuse one plan: after sparse_prefill_plan (untimed) and
    sparse_decode_prepare, step t runs sparse_decode_attn for one query per
    q head at position L - 1 + t against a K/V cache of L + steps + 64 rows.
    Every step reads about 0.5 GB of K/V at the 128K layer (more than L2), so
    no flush is needed.  The roofline counts 512 bytes per key of each kv
    head's key set (sink + union of its q heads' selections + window) plus q
    and O, over the time of the whole call (both kernels)."""
    import torch
    import block_sparse_long_sm_b200 as spa
    world, rank, local = _dist()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    inp = generate(w)
    B, Hq, Hkv, L = w.batch, w.heads_q, w.heads_kv, w.seq_len
    n_steps = max(3, args.warmup) + args.steps
    cap = L + n_steps + 64
    to = lambda u: torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).to(dev).view(torch.bfloat16)
    q, k = to(inp.q), to(inp.k)
    k_cache = torch.empty((B, Hkv, cap, 128), dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty((B, Hkv, cap, 128), dtype=torch.bfloat16, device=dev)
    k_cache[:, :, :L] = k
    v_cache[:, :, :L] = to(inp.v)
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    k_cache[:, :, L:] = torch.randn((B, Hkv, cap - L, 128), generator=g, device=dev).to(torch.bfloat16)
    v_cache[:, :, L:] = torch.randn((B, Hkv, cap - L, 128), generator=g, device=dev).to(torch.bfloat16)
    del inp
    p = spa.make_params(B, Hq, Hkv, L, mode=args.mode, sink=w.sink, local=w.local,
                        theta=args.theta, tau=w.tau,
                        block_k=w.block_k if args.mode == "sale" else None)
    ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)
    spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream), "plan")
    del q, k
    sc = torch.empty(spa.sparse_decode_scratch_bytes(p, cap), dtype=torch.uint8, device=dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    spa.check(spa.sparse_decode_prepare(p, cap, ws, sc, stream=stream), "prepare")
    b.record(stream)
    torch.cuda.synchronize()
    prepare_ms = a.elapsed_time(b)
    qd = torch.randn((B, Hq, 128), generator=g, device=dev).to(torch.bfloat16)
    od = torch.empty((B, Hq, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)

    def call(pos):
        spa.check(spa.sparse_decode_attn(p, qd, k_cache, v_cache, cap, pos, ws, sc, od, lse,
                                         stream=stream), "decode")

    warm = max(3, args.warmup)
    for t in range(warm):
        call(L - 1 + t)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            ev[i][0].record(stream)
            call(L - 1 + warm + i)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    ms = [x.elapsed_time(y) for x, y in ev]
    st, _ = spa.sparse_prefill_stats(p, ws, stream=stream)
    spa.check(st, "stats")

    # key-set sizes per (b, kv head, subgroup of up to 8 q heads): the union
    # of the last prompt block's selections, read from the plan's lists
    from block_sparse_long_sm_b200.binding import WorkspaceView
    view = WorkspaceView(p, ws)
    counts_h = view.counts.cpu().numpy()
    group = Hq // Hkv
    gh = next(d for d in range(8, 0, -1) if group % d == 0)
    qb = (L - 1) // 128
    union_sizes = []
    for b in range(B):
        for g in range(Hkv):
            for hs in range(group // gh):
                sel = [np.zeros(0, np.int64)]
                for j in range(gh):
                    h = g * group + hs * gh + j
                    if args.mode != "dense":   # only this block's list leaves the GPU
                        n = int(counts_h[view.block_index(b, h, qb)])
                        off = view.list_offset(b, h, qb)
                        sel.append(view.lists[off:off + n].cpu().numpy().astype(np.int64))
                union_sizes.append(len(np.unique(np.concatenate(sel))))
    counts = np.array(union_sizes, dtype=np.int64)
    ls = max(0, (qb + 1) * 128 - w.local)
    uk = w.block_k if args.mode == "sale" else 1
    bytes_steps = []
    for i in range(args.steps):
        pos = L - 1 + warm + i
        if args.mode == "dense":
            keys = len(counts) * (pos + 1)
        else:
            s1 = min(w.sink, pos + 1)
            keys = int(np.sum(s1 + counts * uk + (pos + 1 - max(ls, s1))))
        bytes_steps.append(512 * keys + 2 * 2 * 128 * B * Hq)
    peaks = _peaks()
    ms_med = statistics.median(ms)
    alg = statistics.median(bytes_steps)
    gbs = alg / (ms_med / 1e3) / 1e9
    line = {
        "metric": "decode step reusing the prefill plan (one query per q head)",
        "value": 1e3 / ms_med * B, "unit": "decoded tokens/s", "n_gpus": 1,
        "steps": args.steps, "warmup": warm, "ms_per_step": ms_med, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(_config(w, args), kv_capacity=cap, prepare_ms=prepare_ms,
                       l2="K/V read per step larger than L2 (126 MB); no flush"),
        "roofline": {"bound": "hbm", "kernel": "decode_attn_kernel (+ decode_combine_kernel)",
                     "achieved": gbs, "peak": peaks["hbm"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm"], "traffic": None,
                     "algorithmic_bytes": alg,
                     "peak_source": f"{peaks['src']} HBM copy bandwidth"},
        "clocks": clk.summary(),
        "gpu_launches": 2 * args.steps,
        "cpu_baseline": oracle_decode_sample(w, args.theta),
    }
    print(json.dumps(line), flush=True)


def _oracle_cores():
    cores = len(os.sched_getaffinity(0))
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max((i.get("num_threads", 1) for i in info), default=cores)
    except Exception:
        pass
    return cores


def oracle_decode_sample(w: Workload, theta: float, heads: int = 4):
    """fp64 oracle of one decode step for the first `heads` q heads of kv head
    0 at pos = L - 1 (their last-block anchor selection, then attention over
    the decode key set), scaled to all q heads: decoded tokens/s."""
    from oracle import decode as odec
    from oracle import selection as osel
    from workloads import bf16_bits_to_f32
    inp = generate(w, kv_groups=[0])
    L = w.seq_len
    kh = bf16_bits_to_f32(inp.k[0, 0]).astype(np.float64)
    vh = bf16_bits_to_f32(inp.v[0, 0]).astype(np.float64)
    qb = (L - 1) // 128
    t0 = time.perf_counter()
    for h in range(heads):
        qh = bf16_bits_to_f32(inp.q[0, h]).astype(np.float64)
        sel = osel.anchor_block(qh, kh, qb, bq=128, sink=w.sink, local=w.local, theta=theta).kept
        keys = odec.decode_keys(L - 1, L, sel, bq=128, sink=w.sink, local=w.local)
        odec.decode_attend(qh[L - 1], kh, vh, keys)
    dt = time.perf_counter() - t0
    per_step = dt * w.heads_q * w.batch / heads
    return dict(value=w.batch / per_step, unit="decoded tokens/s", cores=_oracle_cores(),
                kind="oracle",
                sample=f"{heads} q heads of {w.name} at pos L-1 (selection of the last block + "
                       f"fp64 decode attention), scaled to {w.heads_q} heads; {dt:.2f} s")


def oracle_rows_sample(w: Workload, theta: float, what: str, n_rows: int = 64):
    """fp64 oracle on the last `n_rows` rows of q head 0: FP8 (quantisation
    + attention of the dequantised operands) or the key mass (LSE of each
    row, then exp(s - LSE) over its kept set); TFLOP/s on 4 d (FP8) or 2 d
    (key mass) per kept pair."""
    from oracle import attention as oatt
    from oracle import decode as odec
    from oracle import fp8 as ofp8
    from oracle import selection as osel
    from workloads import bf16_bits_to_f32
    inp = generate(w, kv_groups=[0])
    L = w.seq_len
    q32 = bf16_bits_to_f32(inp.q[0, 0])
    k32 = bf16_bits_to_f32(inp.k[0, 0])
    v32 = bf16_bits_to_f32(inp.v[0, 0])
    rows = list(range(L - n_rows, L))
    blocks = sorted({i // 128 for i in rows})
    t0 = time.perf_counter()
    qh, kh, vh = (x.astype(np.float64) for x in (q32, k32, v32))
    sel = {qb: osel.anchor_block(qh, kh, qb, bq=128, sink=w.sink, local=w.local,
                                 theta=theta).kept for qb in blocks}
    keys_of = odec.prefill_keys_of_row(L, lambda b: sel[b], bq=128, sink=w.sink, local=w.local)
    if what == "fp8":
        q_hat, k_hat, v_hat = ofp8.dequantized_head(q32, k32, v32)
        for i in rows:
            oatt.attend_row(q_hat[i], k_hat, v_hat, keys_of(i), 1 / math.sqrt(128))
        per_pair = 4 * 128
    else:
        _, lse = oatt.attend_rows(qh, kh, vh, rows, lambda i: i // 128, lambda b: sel[b], bq=128,
                                  sink=w.sink, local=w.local)
        odec.key_mass(qh[rows[0]:], kh, lse, range(len(rows)),
                      lambda n: keys_of(rows[n]))
        per_pair = 2 * 128
    dt = time.perf_counter() - t0
    pairs = sum(len(keys_of(i)) for i in rows)
    return dict(value=per_pair * pairs / dt / 1e12, unit="TFLOP/s", cores=_oracle_cores(),
                kind="oracle",
                sample=f"q head 0, last {n_rows} rows of {w.name} ({what}); {dt:.2f} s")


def variant_bench(args, w: Workload):
    """FP8 attention (--fp8) or the key mass from the prefill LSE (--key-mass)
    over the same plan as the headline step (anchor, theta, 128K layer).  The
    plan (and, for the key mass, the bf16 attention that yields the LSE) runs
    once, untimed; each timed step is sparse_fp8_quantize +
    sparse_prefill_attn_fp8, or sparse_key_mass.  Inputs are larger than L2.
    Roofline of the dominant kernel: FP8 attention on kept FLOPs (4 d per kept
    pair) against the measured bf16 peak times 2 (the nominal fp8:bf16 ratio);
    the key mass on 2 d per kept pair (its QK^T) against the bf16 peak."""
    import torch
    import block_sparse_long_sm_b200 as spa
    world, rank, local = _dist()
    if rank != 0:
        return
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    inp = generate(w)
    to = lambda u: torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).to(dev).view(torch.bfloat16)
    q, k, v = to(inp.q), to(inp.k), to(inp.v)
    del inp
    B, Hq, Hkv, L = w.batch, w.heads_q, w.heads_kv, w.seq_len
    p = spa.make_params(B, Hq, Hkv, L, mode=args.mode, sink=w.sink, local=w.local,
                        theta=args.theta, tau=w.tau,
                        block_k=w.block_k if args.mode == "sale" else None)
    ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)
    spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream), "plan")
    st, stats = spa.sparse_prefill_stats(p, ws, stream=stream)
    spa.check(st, "stats")
    o = torch.empty((B, Hq, L, 128), dtype=torch.bfloat16, device=dev)
    peaks = _peaks()
    if args.fp8:
        q8 = torch.empty((B, Hq, L, 128), dtype=torch.uint8, device=dev)
        k8 = torch.empty((B, Hkv, L, 128), dtype=torch.uint8, device=dev)
        v8 = torch.empty((B, Hkv, L, 128), dtype=torch.uint8, device=dev)
        scales = torch.empty(spa.sparse_fp8_scales_floats(p), dtype=torch.float32, device=dev)
        scratch = torch.empty(spa.sparse_fp8_scratch_bytes(p), dtype=torch.uint8, device=dev)
        quant = lambda: spa.check(spa.sparse_fp8_quantize(p, q, k, v, q8, k8, v8, scales, scratch,
                                                          stream=stream), "fp8 quantize")
        attn = lambda: spa.check(spa.sparse_prefill_attn_fp8(p, q8, k8, v8, scales, ws, o, None,
                                                              stream=stream), "fp8 attn")
        flops = spa.kept_flops(stats)
        peak, kernel, n_launch = 2.0 * peaks["bf16_sus"], "sparse_attn_fp8_kernel", 6
        metric = "FP8 sparse prefill attn (quantise + attn) kept-FLOP TFLOP/s"
    else:
        lse = torch.empty((B, Hq, L), dtype=torch.float32, device=dev)
        spa.check(spa.sparse_prefill_attn(p, q, k, v, ws, o, lse, stream=stream), "attn")
        mass = torch.empty((B, Hkv, L), dtype=torch.float32, device=dev)
        quant = None
        attn = lambda: spa.check(spa.sparse_key_mass(p, q, k, lse, 0, ws, mass, stream=stream),
                                 "key mass")
        flops = 2 * 128 * int(stats.kept_pairs)
        peak, kernel, n_launch = peaks["bf16_sus"], "key_mass_kernel", 1
        metric = "key mass from the prefill LSE, QK^T TFLOP/s on kept pairs"
    warm = max(3, args.warmup)
    for _ in range(warm):
        if quant:
            quant()
        attn()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            ev[i][0].record(stream)
            if quant:
                quant()
            ev[i][1].record(stream)
            attn()
            ev[i][2].record(stream)
        torch.cuda.synchronize()
    step_ms = statistics.median(a.elapsed_time(c) for a, _, c in ev)
    kern_ms = statistics.median(b.elapsed_time(c) for _, b, c in ev)
    achieved = flops / (kern_ms / 1e3) / 1e12
    line = {
        "metric": metric, "value": flops / (step_ms / 1e3) / 1e12, "unit": "TFLOP/s",
        "n_gpus": 1, "steps": args.steps, "warmup": warm, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if args.fp8 else "bf16", "data": "synthetic",
        "config": _config(w, args), "kernel_ms": kern_ms,
        "kept_fraction": stats.kept_pairs / stats.dense_pairs,
        "roofline": {"bound": "tensor", "kernel": kernel, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": None,
                     "peak_source": f"{peaks['src']} bf16 dense, sustained"
                                    + (" x 2 (nominal fp8:bf16)" if args.fp8 else "")},
        "clocks": clk.summary(),
        "gpu_launches": n_launch * args.steps,
        "cpu_baseline": oracle_rows_sample(w, args.theta, "fp8" if args.fp8 else "key_mass"),
    }
    print(json.dumps(line), flush=True)


# SALE thresholds that really skip key blocks on the synthetic 128K layer
# (about 45 % of the candidate blocks kept at 0.1, about 10 % at 0.3)
SALE_PRUNING_TAUS = (0.1, 0.3)


def _operating_point(spa, torch, timed, p, ws, q, k, v, o, stream, peaks, dense_ms, label):
    """Plan and attention of one selection setting on the resident layer:
    kept fraction, times, kept-FLOP roofline of the attention, selection
    bytes against HBM, and the speedup over the same kernel run dense."""
    spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream))
    spa.check(spa.sparse_prefill_attn(p, q, k, v, ws, o, None, stream=stream))
    plan_ms = timed(lambda: spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream)))
    attn_ms = timed(lambda: spa.check(spa.sparse_prefill_attn(p, q, k, v, ws, o, None,
                                                              stream=stream)))
    st, s = spa.sparse_prefill_stats(p, ws, stream=stream)
    spa.check(st, "stats")
    flops = spa.kept_flops(s)
    B, Hq, Hkv, L = p.batch, p.heads_q, p.heads_kv, p.seq_len
    unit = p.block_k if p.mode == spa.SPA_MODE_SALE else 1
    alg_bytes = 2 * B * Hq * L * 128 + 2 * B * Hkv * L * 128 + 4 * s.kept_candidates // unit
    tfl = flops / (attn_ms / 1e3) / 1e12
    return dict(label, kept_fraction=s.kept_pairs / s.dense_pairs,
                kept_candidates_fraction=s.kept_candidates / max(1, s.candidates),
                plan_ms=plan_ms, attn_ms=attn_ms, step_ms=plan_ms + attn_ms,
                attn_tflops=tfl, attn_frac=tfl / peaks["bf16_sus"],
                selection_gbs=alg_bytes / (plan_ms / 1e3) / 1e9,
                selection_frac=alg_bytes / (plan_ms / 1e3) / 1e9 / peaks["hbm"],
                speedup_vs_dense=dense_ms / (plan_ms + attn_ms))


def bench_extras(spa, torch, w, args, q, k, v, o, q_h, k_h, v_h, stream, dev, stats):
    """Selection roofline, SALE mode, dense mode, end-to-end and the CPU baseline."""
    peaks = _peaks()
    out = {}
    B, Hq, Hkv, L = w.batch, w.heads_q, w.heads_kv, w.seq_len

    def timed(fn, reps=3):
        ts = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    # dense mode: same attention kernel over every causal key
    pd = spa.make_params(B, Hq, Hkv, L, mode="dense", sink=w.sink, local=w.local)
    wsd = torch.empty(spa.sparse_prefill_workspace_bytes(pd), dtype=torch.uint8, device=dev)
    spa.check(spa.sparse_prefill_plan(pd, q, k, wsd, stream=stream))
    dense_ms = timed(lambda: spa.check(spa.sparse_prefill_attn(pd, q, k, v, wsd, o, None, stream=stream)))
    st, sd = spa.sparse_prefill_stats(pd, wsd, stream=stream)
    dflops = spa.kept_flops(sd)
    out["dense"] = {"attn_ms": dense_ms, "tflops": dflops / (dense_ms / 1e3) / 1e12,
                    "frac": dflops / (dense_ms / 1e3) / 1e12 / peaks["bf16_sus"]}
    del wsd

    # selection roofline (anchor plan): algorithmic bytes = read Q + read K once + write lists
    p = spa.make_params(B, Hq, Hkv, L, mode="anchor", sink=w.sink, local=w.local, theta=args.theta)
    ws = torch.empty(spa.sparse_prefill_workspace_bytes(p), dtype=torch.uint8, device=dev)
    spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream))
    st, s = spa.sparse_prefill_stats(p, ws, stream=stream)
    plan_ms = timed(lambda: spa.check(spa.sparse_prefill_plan(p, q, k, ws, stream=stream)))
    alg_bytes = 2 * B * Hq * L * 128 + 2 * B * Hkv * L * 128 + 4 * s.kept_candidates
    gbs = alg_bytes / (plan_ms / 1e3) / 1e9
    out["selection"] = {"mode": "anchor", "ms": plan_ms, "algorithmic_bytes": alg_bytes,
                        "achieved_gbs": gbs, "peak_gbs": peaks["hbm"],
                        "frac": gbs / peaks["hbm"], "kept_candidates": s.kept_candidates,
                        "candidates": s.candidates}
    del ws

    # the sparse operating points of the same layer: theta swept over {3, 7}
    # besides the headline's value, and SALE at a tau that skips key blocks
    points = []
    for theta in (3.0, 7.0):
        pt = spa.make_params(B, Hq, Hkv, L, mode="anchor", sink=w.sink, local=w.local, theta=theta)
        wst = torch.empty(spa.sparse_prefill_workspace_bytes(pt), dtype=torch.uint8, device=dev)
        points.append(_operating_point(spa, torch, timed, pt, wst, q, k, v, o, stream, peaks,
                                       dense_ms, dict(mode="anchor", theta=theta)))
        del wst
    for tau in SALE_PRUNING_TAUS:
        pt = spa.make_params(B, Hq, Hkv, L, mode="sale", sink=w.sink, local=w.local, tau=tau,
                             block_k=w.block_k)
        wst = torch.empty(spa.sparse_prefill_workspace_bytes(pt), dtype=torch.uint8, device=dev)
        points.append(_operating_point(spa, torch, timed, pt, wst, q, k, v, o, stream, peaks,
                                       dense_ms, dict(mode="sale", tau=tau, block_k=w.block_k)))
        del wst
    out["operating_points"] = points

    # SALE mode
    ps = spa.make_params(B, Hq, Hkv, L, mode="sale", sink=w.sink, local=w.local, tau=w.tau,
                         block_k=w.block_k)
    wss = torch.empty(spa.sparse_prefill_workspace_bytes(ps), dtype=torch.uint8, device=dev)
    spa.check(spa.sparse_prefill_plan(ps, q, k, wss, stream=stream))
    sale_plan = timed(lambda: spa.check(spa.sparse_prefill_plan(ps, q, k, wss, stream=stream)))
    sale_attn = timed(lambda: spa.check(spa.sparse_prefill_attn(ps, q, k, v, wss, o, None, stream=stream)))
    st, ss = spa.sparse_prefill_stats(ps, wss, stream=stream)
    sflops = spa.kept_flops(ss)
    out["sale"] = {"tau": w.tau, "block_k": w.block_k, "plan_ms": sale_plan, "attn_ms": sale_attn,
                   "kept_fraction": ss.kept_pairs / ss.dense_pairs,
                   "kept_tflops": sflops / ((sale_plan + sale_attn) / 1e3) / 1e12}
    del wss

    # end to end through host buffers: H2D of Q/K/V, plan + attn, D2H of O
    o_h = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
    pe = spa.make_params(B, Hq, Hkv, L, mode=args.mode, sink=w.sink, local=w.local,
                         theta=args.theta, tau=w.tau,
                         block_k=w.block_k if args.mode == "sale" else None)
    wse = torch.empty(spa.sparse_prefill_workspace_bytes(pe), dtype=torch.uint8, device=dev)

    def e2e():
        q.copy_(q_h, non_blocking=True)
        k.copy_(k_h, non_blocking=True)
        v.copy_(v_h, non_blocking=True)
        spa.check(spa.sparse_prefill_plan(pe, q, k, wse, stream=stream))
        spa.check(spa.sparse_prefill_attn(pe, q, k, v, wse, o, None, stream=stream))
        o_h.copy_(o, non_blocking=True)
    e2e()
    e_ms = timed(e2e, reps=3)
    st, se = spa.sparse_prefill_stats(pe, wse, stream=stream)
    out["e2e"] = {"value": spa.kept_flops(se) / (e_ms / 1e3) / 1e12, "unit": UNIT,
                  "ms_per_step": e_ms,
                  "h2d_bytes_per_step": 2 * (q.numel() + k.numel() + v.numel()),
                  "d2h_bytes_per_step": 2 * o.numel()}
    del wse

    # CPU oracle on a bounded sample (same metric and unit)
    if int(os.environ.get("WORLD_SIZE", "1")) == 1:
        inp = generate(w, kv_groups=[0])
        cb = oracle_sample(w, inp, args.theta, n_rows=256)
        cb.pop("seconds", None)
        cb.pop("flops", None)
        out["cpu_baseline"] = cb
    return out


if __name__ == "__main__":
    main()
