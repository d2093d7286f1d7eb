#!/usr/bin/env python
"""Benchmark of the Dust estimator hot path for one transformer linear layer on B200.

One step = the whole path over one batch of seeded synthetic input resident in HBM:
  dust_noisy_linear_fwd (noise + per-draw loss change) -> dust_credit (centring + discounted
  credit scan) -> dust_weight_grad (output-error estimate g + weight estimate G_W),
and, on N > 1 GPUs, one NCCL all-reduce of G_W (each rank holds its own batch; weak scaling).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C] [--impl ours|reference]
Multi-GPU: launched by torchrun, one rank per GPU (RANK / LOCAL_RANK / WORLD_SIZE from the env).
Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle instead (rank 0
only), on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "Dust estimator tokens*draws/s per layer"
UNIT = "tokens*draws/s"
L2_FLUSH_BYTES = 256 << 20

# ALU roofline of the noise kernels: issue slots of all SMs at the maximum SM clock divided by
# the algorithm's minimal per-normal operation count (one Philox4x32-10 block = 10 rounds x
# (2 wide multiplies + 2 three-input XORs) per 4 normals; 3 ops per uniform; Box-Muller 10 ops
# per pair: log, scale, rsqrt, multiply, angle FMA, range scale, sin, cos, 2 products; plus the
# consumer FMAs: 2 per normal in the forward, 1 in the draw reduction).
LANES_PER_SM = 128
OPS_PER_NORMAL = {"fwd_bf16_noise_loss": 20.0, "ghat_reduce_draws": 19.0,
                  "fwd_bf16_noise_loss_grouped": 20.0, "ghat_reduce_draws_grouped": 19.0,
                  # LM head: generator 18 (Philox 10, uniform 3, Box-Muller 5), sigma a (1),
                  # exp(sigma a) - 1 as a degree-5 series (5), the weighted sum (1)
                  "lmhead_ce_noise": 25.0}
# DRAM bytes (read + write) per launch of a dominant kernel, from one ncu capture of the
# current build of that kernel on that workload (profiles/ holds the capture summaries);
# absent entries are reported as null.
MEASURED_TRAFFIC = {
    ("fwd_bf16_noise_loss", "gpt2s-mlp-win-768x3072"): (68.49e6 + 2.45e6,
                                                       "profiles/ncu_full_fwd_persistent_gpt2s_mlp_win_768x3072.md"),
    ("lmhead_ce_noise", "head-4096-slab1024"): (33.85e6 + 75.21e6,
                                                "profiles/ncu_full_lmhead_head-4096-slab1024.md"),
}
HEAD_METRIC = "Dust LM-head estimator tokens*draws/s"
ATTN_METRIC = "Dust attention-reward estimator tokens*draws/s"


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d["bf16_tflops_sustained"],
                    sm_max_mhz=d.get("sm_max_mhz", 1965.0), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                sm_max_mhz=1965.0, source="fallback")


def describe(wl) -> str:
    shapes = sorted({(l.d_in, l.d_out) for l in wl.layers})
    s = ", ".join(f"{a}->{b}" for a, b in shapes)
    return (f"{wl.name} (cfg {wl.cfg_id}): {wl.n_seq}x{wl.seq_len} tokens"
            f"{' packed' if wl.packed else ''}, {len(wl.layers)} layer(s) {s}, K={wl.K}, "
            f"sigma={wl.sigma}, gamma={wl.gamma}, {wl.dtype}")


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(data, n_tokens: int, max_seconds: float):
    """Run the oracle's whole estimator on the first n_tokens of each layer until max_seconds
    of work; returns (token*draws processed per layer, seconds, threads, description)."""
    import oracle
    wl = data.wl
    done = 0
    t0 = time.perf_counter()
    layers_run = 0
    while True:
        L = data.layers[layers_run % len(data.layers)]
        n = min(n_tokens, wl.N)
        cu = np.asarray(data.cu_seqlens, dtype=np.int64)
        cu = np.unique(np.clip(cu, 0, n)).astype(np.int32)
        oracle.dust_layer(L.x_f64[:n], L.W_f64, L.u_f64[:n], wl.K, wl.sigma, wl.gamma, cu,
                          wl.seed, L.shape.layer_id)
        done += n * wl.K
        layers_run += 1
        el = time.perf_counter() - t0
        if el >= max_seconds or layers_run >= 64:
            break
    desc = (f"oracle (fp64 C, OpenMP) whole estimator on the first {min(n_tokens, wl.N)} tokens "
            f"of {layers_run} layer pass(es) of the workload (credit segments truncated to the "
            f"sample)")
    return done, el, oracle.get_threads(), desc


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    data = workloads.generate(args.workload, n_layers=1)
    wl = data.wl
    n_tok = args.ref_tokens
    times = []
    for k in range(args.warmup + args.steps):
        done, el, cores, desc = oracle_sample(data, n_tok, 0.0)
        if k >= args.warmup:
            times.append(el)
    tot = sum(times)
    value = done * len(times) / tot
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(wl), "sample_tokens": min(n_tok, wl.N)},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------------------ GPU arm
class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="clocks_", suffix=".csv")
        self.proc = None
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(gpu_index), "-lms", "200"], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for ln in f:
                p = [x.strip() for x in ln.split(",")]
                if len(p) < 9:
                    continue
                try:
                    sm.append(float(p[1]))
                    smax.append(float(p[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, p[5:9]):
                    if v.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "samples": len(sm),
                "reasons": sorted(reasons)}


def kernel_work(name, wl, shapes):
    """Algorithmic work of one launch over the given layer shapes: (bound, amount, what)."""
    N, K = wl.N, wl.K
    if name in OPS_PER_NORMAL:
        return "alu", sum(N * s.d_out * K for s in shapes), "normals"
    if name.startswith("gw_bf16_tcgen05"):
        return "tensor", sum(2.0 * N * s.d_in * s.d_out for s in shapes), "flops"
    if name.startswith("credit_scan"):
        return "hbm", 8.0 * K * N * len(shapes), "bytes"
    return None, None, None


def generator_ceiling(dust, torch, dev, reps: int = 10) -> float:
    """Gnormal/s of the generator-only probe (generate and add, nothing else) over a grid of
    8 x 256 threads per SM, 1024 normals each: what the noise kernels' generator can reach."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    n, nq = sms * 8 * 256, 256
    out = torch.empty(n, dtype=torch.float32, device=dev)
    key = dust.NoiseKey(0x5EED0000, 0)
    for _ in range(3):
        dust.dust_debug_normal_sum(key, n, nq, out)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        dust.dust_debug_normal_sum(key, n, nq, out)
    b.record()
    torch.cuda.synchronize(dev)
    return 4.0 * n * nq * reps / (a.elapsed_time(b) / 1e3) / 1e9


def run_gpu(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import zeroth_order_transformer_b200 as dust

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    data = workloads.generate(args.workload)
    wl = data.wl
    peaks = measured_peaks()

    def dev_t(store, dtype):
        if dtype == "f32":
            return torch.from_numpy(np.ascontiguousarray(store)).to(dev)
        return torch.from_numpy(np.ascontiguousarray(store).view(np.int16)).view(torch.bfloat16).to(dev)

    layers = []
    for L in data.layers:
        x, W, u = (dev_t(a, wl.dtype) for a in (L.x_store, L.W_store, L.u_store))
        layers.append((L.shape, x, W, u))
    cu = torch.from_numpy(data.cu_seqlens).to(dev)
    tdt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    max_in = max(s.d_in for s, *_ in layers)
    max_out = max(s.d_out for s, *_ in layers)
    ws_bytes = max(dust.dust_workspace_size(op, 1 if wl.dtype == "bf16" else 0, wl.N, s.d_in,
                                            s.d_out, wl.K)
                   for op in range(3) for s, *_ in layers)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
    dloss = torch.empty((wl.K, wl.N), dtype=torch.float32, device=dev)
    r = torch.empty((wl.K, wl.N), dtype=torch.float32, device=dev)
    GWs = [torch.empty((s.d_out, s.d_in), dtype=torch.float32, device=dev) for s, *_ in layers]
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    gamma = wl.gamma

    stacks = {}

    def step(inputs=None):
        inputs = inputs or layers
        if len(inputs) > 1:
            # a block stack: the grouped calls, one launch per step for all layers
            st = stacks.get(id(inputs))
            if st is None:
                st = dust.DustStack([(x, W, u, s.layer_id) for s, x, W, u in inputs], wl.K)
                stacks[id(inputs)] = st
            st.estimate(cu, wl.sigma, gamma, wl.seed, 0, rank * wl.N)
            out = st.G_W
        else:
            s, x, W, u = inputs[0]
            key = dust.NoiseKey(wl.seed, s.layer_id, 0, rank * wl.N)
            dust.dust_noisy_linear_fwd(x, W, u, wl.K, wl.sigma, key, dloss, ws)
            dust.dust_credit(dloss, cu, gamma, r, ws)
            dust.dust_weight_grad(r, x, s.d_out, wl.K, wl.sigma, key, GWs[0], False, None, ws)
            out = GWs
        if world > 1:
            for G in out:
                dist.all_reduce(G)
        return out

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    # ---- timed region
    dust.dust_profile_enable(1 << 16)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    for k in range(args.steps):
        flush.zero_()
        starts[k].record(stream)
        step()
        stops[k].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    clocks = sampler.stop() if sampler else None
    prof = dust.dust_profile_read()
    dust.dust_profile_disable()
    step_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    total_ms = sum(step_ms)
    if world > 1:
        t = torch.tensor([total_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    ms_per_step = total_ms / args.steps
    units = wl.N * wl.K * len(layers) * world
    # tokens*draws per layer processed per second: N K n_layers n_gpus / step time
    value = units / (ms_per_step / 1e3)

    # ---- per-kernel statistics (rank 0's launches)
    per = {}
    for name, ms in prof:
        d = per.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += ms
    kern_total = sum(v[1] for v in per.values())
    kernels = {n: {"launches": c, "ms_total": round(t, 4), "ms_avg": round(t / c, 5),
                   "share": round(t / kern_total, 4) if kern_total else None}
               for n, (c, t) in sorted(per.items(), key=lambda kv: -kv[1][1])}
    s0 = layers[0][0]
    shapes = [s for s, *_ in layers]
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    for n, info in kernels.items():
        bound, amount, what = kernel_work(n, wl, shapes if n.endswith("_grouped") else [s0])
        if amount is None or (len(layers) > 1 and not n.endswith("_grouped")):
            continue
        per_s = amount / (info["ms_avg"] / 1e3)
        if what == "normals":
            info["gnormals_per_s"] = round(per_s / 1e9, 2)
        elif what == "flops":
            info["tflops"] = round(per_s / 1e12, 2)
        else:
            info["gbs"] = round(per_s / 1e9, 2)
    # dominant kernel: the largest total time among kernels with a defined algorithmic work
    def work_of(n):
        return kernel_work(n, wl, shapes if n.endswith("_grouped") else [s0])

    dominant = next((n for n in kernels if work_of(n)[1] is not None), None)
    roofline = None
    if dominant:
        bound, amount, what = work_of(dominant)
        avg_s = kernels[dominant]["ms_avg"] / 1e3
        if bound == "alu":
            peak = sms * LANES_PER_SM * peaks["sm_max_mhz"] * 1e6 / OPS_PER_NORMAL[dominant] / 1e9
            ach = amount / avg_s / 1e9
            roofline = {"kernel": dominant, "bound": "alu", "achieved": round(ach, 2),
                        "peak": round(peak, 2), "unit": "Gnormal/s", "frac": round(ach / peak, 4),
                        "traffic": None,
                        "peak_basis": f"{sms} SMs x {LANES_PER_SM} lanes x "
                                      f"{peaks['sm_max_mhz']:.0f} MHz / "
                                      f"{OPS_PER_NORMAL[dominant]:.0f} ops per normal"}
        elif bound == "tensor":
            ach = amount / avg_s / 1e12
            roofline = {"kernel": dominant, "bound": "tensor", "achieved": round(ach, 2),
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": round(ach / peaks["bf16_tflops"], 4), "traffic": None}
        elif bound == "hbm":
            ach = amount / avg_s / 1e9
            roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(ach, 2),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None}
        if roofline is not None:
            roofline["peak_source"] = peaks["source"]
            tr = MEASURED_TRAFFIC.get((dominant, wl.name))
            if tr is not None:
                roofline["traffic"] = tr[0]
                roofline["traffic_source"] = tr[1]
            if bound == "alu":
                gc = generator_ceiling(dust, torch, dev)
                roofline["generator_ceiling"] = round(gc, 2)
                roofline["frac_of_generator_ceiling"] = round(roofline["achieved"] / gc, 4)

    # ---- end to end through the public API, host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        host_in = []
        h2d = 0
        for s, x, W, u in layers:
            hx, hW, hu = (t.cpu().pin_memory() for t in (x, W, u))
            host_in.append((s, hx, hW, hu))
            h2d += sum(t.numel() * t.element_size() for t in (hx, hW, hu))
        dev_in = [(s, torch.empty_like(x), torch.empty_like(W), torch.empty_like(u))
                  for s, x, W, u in layers]
        host_out = [torch.empty(G.shape, dtype=G.dtype, pin_memory=True) for G in GWs]
        d2h = sum(G.numel() * G.element_size() for G in GWs)

        if len(layers) == 1:
            # one layer: the public host-input call, upload pipelined with the compute
            s1 = layers[0][0]
            host_layer = dust.DustLayer(wl.N, s1.d_in, s1.d_out, wl.K, tdt, dev)
            red = (lambda G: dist.all_reduce(G)) if world > 1 else None

            def e2e_step():
                _, hx, hW, hu = host_in[0]
                host_layer.estimate_from_host(
                    hx, hW, hu, data.cu_seqlens, wl.sigma, gamma,
                    dust.NoiseKey(wl.seed, s1.layer_id, 0, rank * wl.N), host_out[0],
                    chunks=4, reduce=red)
        else:
            def e2e_step():
                for (s, hx, hW, hu), (_, dx, dW, du) in zip(host_in, dev_in):
                    dx.copy_(hx, non_blocking=True)
                    dW.copy_(hW, non_blocking=True)
                    du.copy_(hu, non_blocking=True)
                out = step(dev_in)
                for G, hG in zip(out, host_out):
                    hG.copy_(G, non_blocking=True)

        for _ in range(max(1, args.warmup // 2)):
            flush.zero_()
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        es = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        ee = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for k in range(args.steps):
            flush.zero_()
            es[k].record(stream)
            e2e_step()
            ee[k].record(stream)
        torch.cuda.synchronize(dev)
        e_ms = sum(a.elapsed_time(b) for a, b in zip(es, ee))
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t.item())
        e2e = {"value": units / (e_ms / args.steps / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms / args.steps}

    # ---- optional: the optimizer step fused into the weight estimate (single-layer workloads)
    opt_line = None
    if args.optimizer != "none" and len(layers) == 1:
        s1, x1, W1, u1 = layers[0]
        Wm = torch.zeros((s1.d_out, s1.d_in), dtype=torch.float32, device=dev)
        mm = torch.zeros_like(Wm)
        vv = torch.zeros_like(Wm) if args.optimizer == "adam" else None
        Wb = torch.empty((s1.d_out, s1.d_in), dtype=torch.bfloat16, device=dev)
        key = dust.NoiseKey(wl.seed, s1.layer_id, 0, rank * wl.N)

        def opt_params(t):
            return dust.sgd_momentum(1e-2, 0.9) if args.optimizer == "sgd" else dust.adam(1e-3, t)

        for t in range(1, 3):
            dust.dust_weight_grad_step(r, x1, s1.d_out, wl.K, wl.sigma, key, opt_params(t), Wm,
                                       mm, vv, W_bf16=Wb, workspace=ws)
        torch.cuda.synchronize(dev)
        ea = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        eb = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        reps = max(5, args.steps)
        ea[0].record(stream)
        for t in range(reps):
            dust.dust_weight_grad(r, x1, s1.d_out, wl.K, wl.sigma, key, GWs[0], False, None, ws)
        eb[0].record(stream)
        ea[1].record(stream)
        for t in range(reps):
            dust.dust_weight_grad_step(r, x1, s1.d_out, wl.K, wl.sigma, key, opt_params(t + 3),
                                       Wm, mm, vv, W_bf16=Wb, workspace=ws)
        eb[1].record(stream)
        torch.cuda.synchronize(dev)
        t_plain = ea[0].elapsed_time(eb[0]) / reps
        t_step = ea[1].elapsed_time(eb[1]) / reps
        opt_line = {"kind": args.optimizer, "weight_grad_ms": round(t_plain, 5),
                    "weight_grad_with_step_ms": round(t_step, 5),
                    "step_overhead_ms": round(t_step - t_plain, 5)}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, el, cores, desc = oracle_sample(data, args.cpu_tokens, args.cpu_seconds)
        cpu = {"value": done / el, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc, "seconds": round(el, 2)}

    n_launch_per_step = sum(c for c in (v["launches"] for v in kernels.values())) / args.steps
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "operands": "bf16 x, W, u; u32 Philox words",
        "data": "synthetic (seeded; shapes of the Dust page's transformer layers)",
        "config": {"workload": describe(wl), "tokens_per_gpu": wl.N, "d_in": s0.d_in,
                   "d_out": s0.d_out, "K": wl.K, "layers": len(layers),
                   "parallelism": f"dp{world}: one batch per GPU, NCCL all-reduce of G_W",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": int(round(n_launch_per_step * args.steps)),
        "clocks": clocks,
        "kernels": kernels,
    }
    if opt_line is not None:
        line["optimizer"] = opt_line
    print(json.dumps(line), flush=True)


def kernel_table(prof, work, peaks, sms):
    """Per-kernel launches, times, shares and achieved rates from the profile records, and the
    roofline object of the dominant kernel (the largest total time with a defined work)."""
    per = {}
    for name, t in prof:
        d = per.setdefault(name, [0, 0.0])
        d[0] += 1
        d[1] += t
    tot = sum(v[1] for v in per.values())
    kernels = {n: {"launches": c, "ms_total": round(t, 4), "ms_avg": round(t / c, 5),
                   "share": round(t / tot, 4)}
               for n, (c, t) in sorted(per.items(), key=lambda kv: -kv[1][1])}
    roofline = None
    for n, info in kernels.items():
        bound, amount, what = work(n)
        if amount is None:
            continue
        rate = amount / (info["ms_avg"] / 1e3)
        info[{"normals": "gnormals_per_s", "flops": "tflops", "bytes": "gbs"}[what]] = round(
            rate / (1e12 if what == "flops" else 1e9), 2)
        if roofline is not None:
            continue
        if bound == "alu":
            ops = OPS_PER_NORMAL.get(n, 19.0)
            peak = sms * LANES_PER_SM * peaks["sm_max_mhz"] * 1e6 / ops / 1e9
            roofline = {"kernel": n, "bound": "alu", "achieved": round(rate / 1e9, 2),
                        "peak": round(peak, 2), "unit": "Gnormal/s",
                        "frac": round(rate / 1e9 / peak, 4), "traffic": None,
                        "peak_basis": f"{sms} SMs x {LANES_PER_SM} lanes x "
                                      f"{peaks['sm_max_mhz']:.0f} MHz / {ops:.0f} ops per normal"}
        elif bound == "hbm":
            roofline = {"kernel": n, "bound": "hbm", "achieved": round(rate / 1e9, 2),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(rate / 1e9 / peaks["hbm_gbs"], 4), "traffic": None}
        elif bound == "tensor":
            roofline = {"kernel": n, "bound": "tensor", "achieved": round(rate / 1e12, 2),
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": round(rate / 1e12 / peaks["bf16_tflops"], 4), "traffic": None}
        roofline["peak_source"] = peaks["source"]
    return kernels, roofline


def attn_kernel_work(name, aw):
    """Algorithmic work of one launch of the attention-reward step's kernels."""
    N, K = aw.N, aw.K
    if name == "attn_reward":
        return "hbm", 2.0 * K * N * aw.d + 4.0 * N * aw.d + 4.0 * K * N, "bytes"
    if name.startswith("discounted_credit_scan"):
        return "hbm", 8.0 * K * N, "bytes"
    if name == "ghat_reduce_draws":
        return "alu", N * aw.d * K, "normals"
    if name.startswith("gw_bf16_tcgen05"):
        return "tensor", 2.0 * N * aw.d_model * aw.d, "flops"
    return None, None, None


def run_attn(args) -> None:
    """The estimate of an attention projection from the attention-internal reward:
    dust_attn_reward (c = -<ghat, delta_o>) -> dust_discounted_credit -> dust_weight_grad of
    the perturbed projection.  One GPU; one JSON line."""
    import torch

    import zeroth_order_transformer_b200 as dust
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    aw = workloads.ATTN_WORKLOADS[args.attn]
    data = workloads.generate_attn(aw)
    peaks = measured_peaks()
    G = torch.from_numpy(data.ghat).to(dev)
    dO = torch.from_numpy(data.dO_store.view(np.int16)).view(torch.bfloat16).to(dev)
    x = torch.from_numpy(data.x_store.view(np.int16)).view(torch.bfloat16).to(dev)
    cu = torch.from_numpy(data.cu_seqlens).to(dev)
    ws = torch.empty(max(dust.dust_workspace_size(dust.DUST_OP_CREDIT, 0, aw.N, 0, 0, aw.K),
                         dust.dust_workspace_size(dust.DUST_OP_WEIGHT_GRAD, 1, aw.N, aw.d_model,
                                                  aw.d, aw.K)), dtype=torch.uint8, device=dev)
    c = torch.empty((aw.K, aw.N), dtype=torch.float32, device=dev)
    r = torch.empty_like(c)
    GW = torch.empty((aw.d, aw.d_model), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    key = dust.NoiseKey(aw.seed, 2)

    def step(GG=G, DD=dO, XX=x):
        dust.dust_attn_reward(GG, DD, c)
        dust.dust_discounted_credit(c, cu, aw.gamma, r, ws)
        dust.dust_weight_grad(r, XX, aw.d, aw.K, aw.sigma, key, GW, False, None, ws)
        return GW

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    dust.dust_profile_enable(1 << 16)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    prof = dust.dust_profile_read()
    dust.dust_profile_disable()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    units = aw.N * aw.K
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kernels, roofline = kernel_table(prof, lambda n: attn_kernel_work(n, aw), peaks, sms)
    if roofline is not None and roofline["bound"] == "alu":
        gc = generator_ceiling(dust, torch, dev)
        roofline["generator_ceiling"] = round(gc, 2)
        roofline["frac_of_generator_ceiling"] = round(roofline["achieved"] / gc, 4)
    e2e = None
    if not args.no_e2e:
        hG, hD, hx = (t.cpu().pin_memory() for t in (G, dO, x))
        dG, dD, dx = torch.empty_like(G), torch.empty_like(dO), torch.empty_like(x)
        hW = torch.empty(GW.shape, dtype=GW.dtype, pin_memory=True)

        def e2e_step():
            dG.copy_(hG, non_blocking=True)
            dD.copy_(hD, non_blocking=True)
            dx.copy_(hx, non_blocking=True)
            hW.copy_(step(dG, dD, dx), non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ee:
            flush.zero_()
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = sum(a.elapsed_time(b) for a, b in ee) / args.steps
        e2e = {"value": units / (e_ms / 1e3), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hG, hD, hx)),
               "d2h_bytes_per_step": hW.numel() * hW.element_size()}
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        n_tok = 256
        G64 = data.ghat[:n_tok].astype(np.float64)
        D64 = workloads.bf16_bits_to_f64(data.dO_store[:, :n_tok])
        X64 = workloads.bf16_bits_to_f64(data.x_store[:n_tok])
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            cc = oracle.attn_reward(G64, D64)
            rr = oracle.discounted_credit(cc, np.array([0, n_tok], dtype=np.int32), aw.gamma)
            g = oracle.output_error(rr, aw.K, aw.sigma, aw.seed, aw.d, 2)
            oracle.weight_grad(g, X64)
            done += n_tok * aw.K
        el = time.perf_counter() - t0
        cpu = {"value": done / el, "unit": UNIT, "cores": oracle.get_threads(), "kind": "oracle",
               "seconds": round(el, 2),
               "sample": f"oracle (fp64 C, OpenMP) reward-based estimate on the first {n_tok} "
                         f"tokens (credit truncated to the sample), repeated for about "
                         f"{args.cpu_seconds:.0f} s"}
    line = {
        "metric": ATTN_METRIC, "value": units / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "operands": "bf16 delta_o and x, f32 ghat",
        "data": "synthetic (seeded; GPT-2-small attention shape)",
        "config": {"workload": f"{aw.name}: {aw.n_seq}x{aw.seq_len} tokens, projection "
                               f"{aw.d_model}->{aw.d}, K={aw.K}, sigma={aw.sigma}, "
                               f"gamma={aw.gamma}",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": sum(v["launches"] for v in kernels.values()), "clocks": clocks,
        "kernels": kernels,
    }
    print(json.dumps(line), flush=True)


def spsa_kernel_work(name, wl, P):
    """Algorithmic work of one launch of the SPSA probe step's kernels (one layer)."""
    N, s = wl.N, wl.layers[0]
    if name == "spsa_probe_gemm":
        return "tensor", 2.0 * N * s.d_in * s.d_out * P, "flops"
    if name == "spsa_residual_gemm":
        return "tensor", 2.0 * N * s.d_in * s.d_out, "flops"
    if name in ("spsa_directions", "spsa_estimate"):
        return "alu", s.d_out * s.d_in * P, "normals"
    return None, None, None


def run_spsa(args) -> None:
    """The SPSA / MeZO contrast estimator on a workload's first layer: dust_spsa_probe (the two
    perturbed forwards of P probes) -> dust_spsa_estimate (the weight estimate).  One GPU."""
    import torch

    import zeroth_order_transformer_b200 as dust
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    data = workloads.generate(args.workload, n_layers=1)
    wl = data.wl
    L = data.layers[0]
    s0 = L.shape
    P = args.spsa_probes
    peaks = measured_peaks()

    def dev_t(store):
        return torch.from_numpy(np.ascontiguousarray(store).view(np.int16)).view(
            torch.bfloat16).to(dev)

    x, W, u = dev_t(L.x_store), dev_t(L.W_store), dev_t(L.u_store)
    ws = torch.empty(dust.dust_workspace_size(dust.DUST_OP_SPSA_PROBE, 1, wl.N, s0.d_in, s0.d_out,
                                              P), dtype=torch.uint8, device=dev)
    p = torch.empty(P, dtype=torch.float32, device=dev)
    G = torch.empty((s0.d_out, s0.d_in), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    key = dust.NoiseKey(wl.seed, s0.layer_id)

    def step(xx=x, WW=W, uu=u):
        dust.dust_spsa_probe(xx, WW, uu, P, 1e-3, key, p, workspace=ws)
        dust.dust_spsa_estimate(p, P, s0.d_out, s0.d_in, key, G)
        return G

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    dust.dust_profile_enable(1 << 16)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    prof = dust.dust_profile_read()
    dust.dust_profile_disable()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kernels, roofline = kernel_table(prof, lambda n: spsa_kernel_work(n, wl, P), peaks, sms)
    units = wl.N * P
    e2e = None
    if not args.no_e2e:
        hx, hW, hu = (t.cpu().pin_memory() for t in (x, W, u))
        dx, dW, du = torch.empty_like(x), torch.empty_like(W), torch.empty_like(u)
        hG = torch.empty(G.shape, dtype=G.dtype, pin_memory=True)

        def e2e_step():
            dx.copy_(hx, non_blocking=True)
            dW.copy_(hW, non_blocking=True)
            du.copy_(hu, non_blocking=True)
            hG.copy_(step(dx, dW, du), non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ee:
            flush.zero_()
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = sum(a.elapsed_time(b) for a, b in ee) / args.steps
        e2e = {"value": units / (e_ms / 1e3), "unit": "tokens*probes/s", "ms_per_step": e_ms,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hx, hW, hu)),
               "d2h_bytes_per_step": hG.numel() * hG.element_size()}
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        n_tok = 64
        done, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            pp, _, _ = oracle.spsa_probe(L.x_f64[:n_tok], L.W_f64, L.u_f64[:n_tok], 1, 1e-3,
                                         wl.seed, s0.layer_id, done // n_tok % P)
            done += n_tok
        el = time.perf_counter() - t0
        cpu = {"value": done / el, "unit": "tokens*probes/s", "cores": oracle.get_threads(),
               "kind": "oracle", "seconds": round(el, 2),
               "sample": f"oracle (fp64 C) two perturbed forwards of one probe on {n_tok} tokens, "
                         f"repeated for about {args.cpu_seconds:.0f} s (the estimate step not "
                         f"included)"}
    line = {
        "metric": "SPSA/MeZO contrast estimator tokens*probes/s", "value": units / (ms / 1e3),
        "unit": "tokens*probes/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32", "operands": "bf16 x, W, u and directions", "data": "synthetic (seeded)",
        "config": {"workload": f"{describe(wl)}; first layer; P={P} probes, eps=1e-3",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": sum(v["launches"] for v in kernels.values()), "clocks": clocks,
        "kernels": kernels,
    }
    print(json.dumps(line), flush=True)


def head_kernel_work(name, hw):
    """Algorithmic work of one launch of the LM-head step's kernels."""
    N, K = hw.N, hw.K
    zb = 2 if hw.dtype == "bf16" else 4
    if name in ("lmhead_ce_noise", "ghat_reduce_draws"):
        return "alu", N * hw.S * K, "normals"
    if name == "lmhead_ce_stats":
        return "hbm", N * hw.V * zb + N * 16, "bytes"
    if name.startswith("gw_bf16_tcgen05"):
        return "tensor", 2.0 * N * hw.d_model * hw.S, "flops"
    if name.startswith("credit_scan"):
        return "hbm", 8.0 * K * N, "bytes"
    return None, None, None


def run_head(args) -> None:
    """The LM-head estimator on cached logits: dust_noisy_logits_ce (cross-entropy change with
    noise on the vocabulary slab) -> dust_credit -> dust_weight_grad on the slab's channels
    (g and the slab's rows of the head weight estimate).  One GPU; one JSON line."""
    import torch

    import zeroth_order_transformer_b200 as dust
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    hw = workloads.HEAD_WORKLOADS[args.head]
    data = workloads.generate_head(hw)
    peaks = measured_peaks()

    def dev_t(store):
        if hw.dtype == "f32":
            return torch.from_numpy(np.ascontiguousarray(store)).to(dev)
        return torch.from_numpy(np.ascontiguousarray(store).view(np.int16)).view(
            torch.bfloat16).to(dev)

    z, h = dev_t(data.z_store), dev_t(data.h_store)
    y = torch.from_numpy(data.y).to(dev)
    cu = torch.from_numpy(data.cu_seqlens).to(dev)
    dt = 1 if hw.dtype == "bf16" else 0
    ws_bytes = max(dust.dust_workspace_size(dust.DUST_OP_LOGITS_CE, dt, hw.N, hw.V, hw.S, hw.K),
                   dust.dust_workspace_size(dust.DUST_OP_CREDIT, 0, hw.N, 0, 0, hw.K),
                   dust.dust_workspace_size(dust.DUST_OP_WEIGHT_GRAD, dt, hw.N, hw.d_model,
                                            hw.S, hw.K))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dloss = torch.empty((hw.K, hw.N), dtype=torch.float32, device=dev)
    r = torch.empty_like(dloss)
    GW = torch.empty((hw.S, hw.d_model), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    key = dust.NoiseKey(hw.seed, 48)
    slab_key = key._replace(channel_offset=hw.v0)

    def step(zz=z, yy=y, hh=h):
        dust.dust_noisy_logits_ce(zz, yy, hw.v0, hw.S, hw.K, hw.sigma, key, dloss, ws)
        dust.dust_credit(dloss, cu, hw.gamma, r, ws)
        dust.dust_weight_grad(r, hh, hw.S, hw.K, hw.sigma, slab_key, GW, False, None, ws)
        return GW

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    dust.dust_profile_enable(1 << 16)
    sampler = ClockSampler(int(os.environ.get("LOCAL_RANK", "0")))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    clocks = sampler.stop()
    prof = dust.dust_profile_read()
    dust.dust_profile_disable()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    units = hw.N * hw.K
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    kernels, roofline = kernel_table(prof, lambda n: head_kernel_work(n, hw), peaks, sms)
    if roofline is not None and (roofline["kernel"], hw.name) in MEASURED_TRAFFIC:
        roofline["traffic"], roofline["traffic_source"] = MEASURED_TRAFFIC[(roofline["kernel"], hw.name)]
    if roofline is not None and roofline["bound"] == "alu":
        gc = generator_ceiling(dust, torch, dev)
        roofline["generator_ceiling"] = round(gc, 2)
        roofline["frac_of_generator_ceiling"] = round(roofline["achieved"] / gc, 4)
    # end to end: logits, targets and hidden states from pinned host memory, G_W back
    e2e = None
    if not args.no_e2e:
        hz, hy, hh = (t.cpu().pin_memory() for t in (z, y, h))
        dz, dy, dh = torch.empty_like(z), torch.empty_like(y), torch.empty_like(h)
        hG = torch.empty(GW.shape, dtype=GW.dtype, pin_memory=True)

        def e2e_step():
            dz.copy_(hz, non_blocking=True)
            dy.copy_(hy, non_blocking=True)
            dh.copy_(hh, non_blocking=True)
            hG.copy_(step(dz, dy, dh), non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for a, b in ee:
            flush.zero_()
            a.record(stream)
            e2e_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms = sum(a.elapsed_time(b) for a, b in ee) / args.steps
        e2e = {"value": units / (e_ms / 1e3), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in (hz, hy, hh)),
               "d2h_bytes_per_step": hG.numel() * hG.element_size()}
    cpu = None
    if not args.no_cpu_baseline:
        import oracle
        n_tok, done, t0 = 8, 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            t0_blk = (done // hw.K) % (hw.N - n_tok + 1)
            idx = np.arange(t0_blk, t0_blk + n_tok)
            loss, _ = oracle.noisy_logits_ce(data.z_f64, data.y, hw.v0, hw.S, hw.K, hw.sigma,
                                             hw.seed, 48, tokens=idx)
            rr = oracle.credit(loss, np.array([0, n_tok], dtype=np.int32), hw.gamma)
            g = oracle.output_error(rr, hw.K, hw.sigma, hw.seed, hw.V, 48,
                                    token_offset=int(t0_blk),
                                    chans=np.arange(hw.v0, hw.v0 + hw.S))
            oracle.weight_grad(g, data.h_f64[idx])
            done += n_tok * hw.K
        el = time.perf_counter() - t0
        cpu = {"value": done / el, "unit": UNIT, "cores": oracle.get_threads(),
               "kind": "oracle", "seconds": round(el, 2),
               "sample": f"oracle (fp64 C, OpenMP) head estimator on blocks of {n_tok} tokens "
                         f"(gamma = 0: tokens are independent) for about {args.cpu_seconds:.0f} s"}
    line = {
        "metric": HEAD_METRIC, "value": units / (ms / 1e3), "unit": UNIT, "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "operands": f"{hw.dtype} logits and hidden states",
        "data": "synthetic (seeded; the Dust page's head shape)",
        "config": {"workload": f"{hw.name}: {hw.n_seq}x{hw.seq_len} tokens, vocabulary {hw.V}, "
                               f"slab [{hw.v0}, {hw.v0 + hw.S}), width {hw.d_model}, K={hw.K}, "
                               f"sigma={hw.sigma}, gamma={hw.gamma}",
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": sum(v["launches"] for v in kernels.values()), "clocks": clocks,
        "kernels": kernels,
    }
    print(json.dumps(line), flush=True)


def run_credit_stress(args) -> None:
    """The credit step alone on a stress shape larger than L2 (default K = 64 draws x 4 Mi
    tokens: 1 GiB of losses in, 1 GiB of credit out), packed sequences U[256, 2048]; prints
    the achieved HBM bandwidth of the algorithmic bytes (8 K N per launch)."""
    import torch

    import zeroth_order_transformer_b200 as dust
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    K, N = args.stress_K, args.stress_N
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    loss = torch.randn((K, N), generator=g, device=dev, dtype=torch.float32)
    r = torch.empty_like(loss)
    cu = torch.from_numpy(workloads.random_segments(77, N, 256, 2048)).to(dev)
    ws = torch.empty(dust.dust_workspace_size(dust.DUST_OP_CREDIT, dust.DUST_F32, N, 0, 0, K),
                     dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        dust.dust_credit(loss, cu, 0.99, r, ws)
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for a, b in evs:
        a.record()
        dust.dust_credit(loss, cu, 0.99, r, ws)
        b.record()
    torch.cuda.synchronize(dev)
    ms = sum(a.elapsed_time(b) for a, b in evs) / args.steps
    st = dust.dust_last_device_error()[0]
    peaks = measured_peaks()
    gbs = 8.0 * K * N / (ms / 1e3) / 1e9
    print(json.dumps({"stage": "credit_scan", "K": K, "N": N, "ms": ms, "GB/s": gbs,
                      "frac_hbm": gbs / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
                      "peak_source": peaks["source"], "status": st,
                      "note": "inputs exceed L2 (2 GiB moved per launch); no flush needed"}),
          flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--cpu-tokens", type=int, default=1024)
    ap.add_argument("--ref-tokens", type=int, default=256)
    ap.add_argument("--optimizer", choices=["none", "sgd", "adam"], default="none",
                    help="also time the optimizer step fused into the weight estimate (reported "
                         "under 'optimizer'; the headline value stays the estimator alone)")
    ap.add_argument("--credit-stress", action="store_true",
                    help="time dust_credit alone on a shape larger than L2 and exit")
    ap.add_argument("--stress-K", type=int, default=64)
    ap.add_argument("--stress-N", type=int, default=1 << 22)
    ap.add_argument("--head", choices=sorted(workloads.HEAD_WORKLOADS), default=None,
                    help="time the LM-head estimator on cached logits instead and exit")
    ap.add_argument("--attn", choices=sorted(workloads.ATTN_WORKLOADS), default=None,
                    help="time the attention-reward estimate of a projection instead and exit")
    ap.add_argument("--spsa", action="store_true",
                    help="time the SPSA/MeZO contrast estimator on the workload's first layer")
    ap.add_argument("--spsa-probes", type=int, default=16)
    args = ap.parse_args()
    if args.credit_stress:
        run_credit_stress(args)
        return
    if args.head:
        run_head(args)
        return
    if args.attn:
        run_attn(args)
        return
    if args.spsa:
        run_spsa(args)
        return
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
