#!/usr/bin/env python
"""Benchmark of the Dust estimator hot path on B200.

One step = the whole path over one batch of seeded synthetic input resident in HBM:
  dust_noisy_linear_fwd (noise + per-draw loss change) -> dust_credit (centring + discounted
  credit scan) -> dust_weight_grad (output-error estimate g + weight estimate G_W),
for every layer of the workload (by default the 48 linear layers of a 12-block GPT-2-small
stack, through the grouped calls: one launch per stage for all layers), and, on N > 1 GPUs,
the all-reduce of G_W (each rank holds its own batch; weak scaling), in buckets of layers
overlapped with the weight estimate.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload C] [--gamma G]
                        [--impl ours|reference]
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
# The 48-layer stack is the largest single-GPU workload; its gamma is swept over {0, 0.9,
# 0.99}, and the headline takes the middle value.
HEADLINE_GAMMA = 0.9

# ALU roofline of the noise kernels, per pipe.  Rates are operations per clock per SM (the
# CUDA C programming guide's arithmetic-throughput table): 32-bit integer multiply 64 (a
# 32x32->64 widening multiply gives two results), special functions (lg2, rsqrt, sin, cos)
# 16, logical/shift/integer add 64, fp32 add/multiply/fma 128 on the two FMA pipes that the
# integer multiplies share, and one warp instruction per clock per scheduler (128 lanes).
PIPE_RATE = {"imad": 64.0, "xu": 16.0, "alu": 64.0, "fma_pipes": 128.0, "issue": 128.0}
# Per-normal operation counts, from the algorithm (not from compiled code):
#   Philox4x32-10: per 4 normals, 10 rounds x (2 widening multiplies + 2 three-input XORs);
#     the kernels walk runs of counters that differ in one word, where the first two rounds
#     share one product each over the run: 18 multiplies and 19 XORs per block
#     -> imad 9 results, alu 4.75;  uniforms: the word's mantissa field (shift, add) -> alu 2;
#     the near-one test once per block (max, compare, branch) -> alu 0.75
#   instructions: 4.5 multiplies + 4.75 XORs + 2 + 0.75 + 2 special functions + 0.75 packed fp32
#   Box-Muller per pair: lg2, rsqrt, sin, cos -> xu 2;  radius uniform, angle, -sqrt as
#     packed f32x2 pairs -> fp32 1.5 (0.75 instructions)
#   consumer: forward 2 fp32 per normal (1 packed instruction); draw reduction r x nq per
#     pair and 1 fma per normal -> 1.5 (0.75 instructions); LM head sigma a, a degree-5 series
#     of exp(sigma a) - 1 and the weighted sum -> 7 (4 instructions)
_GEN = {"imad": 9.0, "xu": 2.0, "alu": 7.5, "fp32": 1.5, "instr": 14.75}
#   SPSA directions: rho x (cos or sin) and the bf16 pair conversion -> 1 fp32 (1 instruction);
#     SPSA estimate: the same product and p_j z -> 2 fp32 (1 packed instruction)
_CONSUMER = {"fwd": (2.0, 1.0), "ghat": (1.5, 0.75), "lmhead": (7.0, 4.0), "spsa_dir": (1.0, 1.0),
             "spsa_est": (2.0, 1.0)}
ALU_KERNELS = {"fwd_bf16_noise_loss": "fwd", "fwd_bf16_noise_loss_grouped": "fwd",
               "ghat_reduce_draws": "ghat", "ghat_reduce_draws_grouped": "ghat",
               "lmhead_ce_noise": "lmhead", "spsa_directions": "spsa_dir",
               "spsa_estimate": "spsa_est"}

# DRAM bytes (read + write) per launch of a dominant kernel from one ncu capture, with the
# digest of the CUDA sources that build that kernel: a value is reported only while those files
# still have that digest (a changed kernel reports null until it is captured again).  Each
# entry: (kernel, workload) -> (bytes per launch, source files, their digest, summary).
_FWD_SOURCES = ("dust_fwd.cu", "dust_device.cuh", "dust_internal.h")
MEASURED_TRAFFIC = {
    # the full 48-layer launch, one pass (dram__bytes_read.sum + dram__bytes_write.sum)
    ("fwd_bf16_noise_loss_grouped", "gpt2s-12-block-stack-48-layers"): (
        2783402752 + 372459008, _FWD_SOURCES, "030dab1ab282d541",
        "profiles/ncu_dram_stack_48_layers.md"),
}
HEAD_METRIC = "Dust LM-head estimator tokens*draws/s"
ATTN_METRIC = "Dust attention-reward estimator tokens*draws/s"


def source_digest(files=None) -> str:
    """sha256 (first 16 hex digits) of the library's CUDA sources (all of them and the public
    header, or only the named files of csrc/)."""
    import glob
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "zeroth_order_transformer_b200", "csrc")
    if files is None:
        paths = sorted(glob.glob(os.path.join(csrc, "*.cu")) + glob.glob(os.path.join(csrc, "*.cuh"))
                       + glob.glob(os.path.join(csrc, "*.h"))
                       + glob.glob(os.path.join(ROOT, "include", "*.h")))
    else:
        paths = [os.path.join(csrc, f) for f in files]
    for f in paths:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    e = MEASURED_TRAFFIC.get((kernel, workload))
    if e is None or e[2] != source_digest(e[1]):
        return None, None
    return e[0], e[3]


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


def alu_bounds(kind: str, sms: int, mhz: float):
    """Gnormal/s that each pipe allows a noise kernel of the given consumer kind, and the
    binding (smallest) one."""
    c_fp32, c_instr = _CONSUMER[kind]
    ops = {"imad": _GEN["imad"], "xu": _GEN["xu"], "alu": _GEN["alu"],
           "fma_pipes": _GEN["imad"] + _GEN["fp32"] + c_fp32, "issue": _GEN["instr"] + c_instr}
    clk = sms * mhz * 1e6
    bounds = {p: round(clk * PIPE_RATE[p] / n / 1e9, 1) for p, n in ops.items()}
    binding = min(bounds, key=bounds.get)
    return bounds, binding, ops


def alu_roofline(kernel: str, achieved: float, sms: int, peaks) -> dict:
    bounds, binding, ops = alu_bounds(ALU_KERNELS[kernel], sms, peaks["sm_max_mhz"])
    peak = bounds[binding]
    return {"kernel": kernel, "bound": "alu", "achieved": round(achieved, 2), "peak": peak,
            "unit": "Gnormal/s", "frac": round(achieved / peak, 4), "traffic": None,
            "peak_source": "derived", "binding_pipe": binding, "pipe_bounds": bounds,
            "peak_basis": (f"min over pipes of {sms} SMs x {peaks['sm_max_mhz']:.0f} MHz x "
                           f"(pipe ops per clock per SM) / (that pipe's ops per normal); ops "
                           f"per normal {ops}; clock from MEASURED_PEAKS.json")}


def describe(wl, gamma=None) -> str:
    shapes = sorted({(l.d_in, l.d_out) for l in wl.layers})
    s = ", ".join(f"{a}->{b}" for a, b in shapes)
    g = wl.gamma if gamma is None else gamma
    return (f"{wl.name} (cfg {wl.cfg_id}): {wl.n_seq}x{wl.seq_len} tokens"
            f"{' packed' if wl.packed else ''}, {len(wl.layers)} layer(s) {s}, K={wl.K}, "
            f"sigma={wl.sigma}, gamma={g}, {wl.dtype}")


def headline_gamma(wl, arg):
    if arg is not None:
        return float(arg)
    return HEADLINE_GAMMA if HEADLINE_GAMMA in wl.gammas else wl.gamma


# ------------------------------------------------------------------------------ CPU oracle
def oracle_sample(data, n_tokens: int, max_seconds: float, gamma=None, first: int = 0):
    """Run the oracle's whole estimator on the first n_tokens of each layer in turn (from layer
    `first`) until max_seconds of work; returns (token*draws processed per layer, seconds,
    threads, description)."""
    import oracle
    wl = data.wl
    g = wl.gamma if gamma is None else gamma
    done = 0
    t0 = time.perf_counter()
    layers_run = 0
    while True:
        L = data.layers[(first + layers_run) % len(data.layers)]
        n = min(n_tokens, wl.N)
        cu = np.asarray(data.cu_seqlens, dtype=np.int64)
        cu = np.unique(np.clip(cu, 0, n)).astype(np.int32)
        oracle.dust_layer(L.x_f64[:n], L.W_f64, L.u_f64[:n], wl.K, wl.sigma, g, cu,
                          wl.seed, L.shape.layer_id)
        done += n * wl.K
        layers_run += 1
        el = time.perf_counter() - t0
        if el >= max_seconds or layers_run >= 64:
            break
    desc = (f"oracle (fp64 C, OpenMP) whole estimator on the first {min(n_tokens, wl.N)} tokens "
            f"of {layers_run} layer pass(es) of the workload, cycling through its layers "
            f"(credit segments truncated to the sample)")
    return done, el, oracle.get_threads(), desc


def run_reference(args, rank: int, world: int) -> None:
    if rank != 0:
        return
    wl0 = workloads.WORKLOADS[args.workload]
    # enough layers for the sample to visit every layer shape of the workload
    data = workloads.generate(args.workload, n_layers=min(len(wl0.layers), 4))
    wl = data.wl
    gamma = headline_gamma(wl, args.gamma)
    n_tok = args.ref_tokens
    times = []
    for k in range(args.warmup + args.steps):
        done, el, cores, desc = oracle_sample(data, n_tok, 0.0, gamma, first=k)
        if k >= args.warmup:
            times.append(el)
    tot = sum(times)
    value = done * len(times) / tot
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(wl0, gamma), "sample_tokens": min(n_tok, wl.N)},
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
    if name in ALU_KERNELS:
        return "alu", sum(N * s.d_out * K for s in shapes), "normals"
    if name.startswith("gw_bf16_tcgen05"):
        return "tensor", sum(2.0 * N * s.d_in * s.d_out for s in shapes), "flops"
    if name.startswith("credit_scan"):
        return "hbm", 8.0 * K * N * len(shapes), "bytes"
    return None, None, None


def _time_probe(fn, torch, reps: int = 10) -> float:
    """Milliseconds per call of fn (3 untimed calls, then reps between CUDA events on the
    current stream)."""
    for _ in range(3):
        fn()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(reps):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


def generator_ceiling(dust, torch, dev) -> dict:
    """Rates of the generator-only probe (Philox, Box-Muller and one add per normal) and of
    the Philox-only probe (the words XORed together), over a grid of 8 x 256 threads per SM,
    1024 normals (256 blocks) per thread: what the noise kernels' generator, and its integer
    part alone, reach on the device."""
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    n, nq = sms * 8 * 256, 256
    out = torch.empty(n, dtype=torch.float32, device=dev)
    wout = torch.empty(n, dtype=torch.int32, device=dev)
    key = dust.NoiseKey(0x5EED0000, 0)
    ms_n = _time_probe(lambda: dust.dust_debug_normal_sum(key, n, nq, out), torch)
    ms_w = _time_probe(lambda: dust.dust_debug_word_sum(key, n, nq, wout), torch)
    return {"generator_gnormal_s": round(4.0 * n * nq / (ms_n / 1e3) / 1e9, 2),
            "philox_gword_s": round(4.0 * n * nq / (ms_w / 1e3) / 1e9, 2)}


def _prof_avg(prof, prefix):
    t = [ms for name, ms in prof if name.startswith(prefix)]
    return (sum(t) / len(t), len(t)) if t else (None, 0)


def _single_layer_inputs(dust, torch, dev, cfg):
    data = workloads.generate(cfg)
    L = data.layers[0]

    def to_dev(st):
        return torch.from_numpy(np.ascontiguousarray(st).view(np.int16)).view(
            torch.bfloat16).to(dev)

    x, W, u = to_dev(L.x_store), to_dev(L.W_store), to_dev(L.u_store)
    return data, L, x, W, u, torch.from_numpy(data.cu_seqlens).to(dev)


def measure_targets(dust, torch, dev, peaks, flush, reps: int) -> dict:
    """The hot path's numeric targets, each measured here with CUDA events on the launching
    stream (the library's per-launch profile records):
      gw_cfg3            the weight-estimate contraction on the packed 32k x 1024 -> 1024
                         workload, TFLOP/s against the measured dense bf16 peak (target 0.6);
      credit_stress      the credit scan on K = 64 x 4 Mi tokens (larger than L2), GB/s of
                         its 8 K N algorithmic bytes against the measured HBM copy bandwidth;
      reduction_streams  the draw reduction on the 16k x 2048 -> 8192, K = 64 workload: its
                         HBM streams (credit read 4 K N + bf16 g write 2 N d_out bytes) in GB/s
                         against the HBM peak, and its normals against the ALU bound that in
                         fact binds it;
      credit_latency     the credit step of each workload (its own K, N and segments)."""
    out = {}
    sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def run_wgrad(cfg, terms=(dust.G_TERMS,)):
        """Profile records of reps weight-estimate calls (L2 flushed before each) per number of
        bf16 terms of g, on the workload's own credit."""
        data, L, x, W, u, cu = _single_layer_inputs(dust, torch, dev, cfg)
        wl, s = data.wl, L.shape
        ws = torch.empty(max(dust.dust_workspace_size(op, 1, wl.N, s.d_in, s.d_out, wl.K)
                             for op in range(3)), dtype=torch.uint8, device=dev)
        key = dust.NoiseKey(wl.seed, s.layer_id)
        dl = dust.dust_noisy_linear_fwd(x, W, u, wl.K, wl.sigma, key, workspace=ws)
        r = dust.dust_credit(dl, cu, wl.gamma, workspace=ws)
        G = torch.empty((s.d_out, s.d_in), dtype=torch.float32, device=dev)
        profs = {}
        for nt in terms:
            for _ in range(3):
                dust.dust_weight_grad(r, x, s.d_out, wl.K, wl.sigma, key, G, False, None, ws,
                                      g_terms=nt)
            torch.cuda.synchronize(dev)
            dust.dust_profile_read()
            dust.dust_profile_enable(1 << 12)
            for _ in range(reps):
                flush.zero_()
                dust.dust_weight_grad(r, x, s.d_out, wl.K, wl.sigma, key, G, False, None, ws,
                                      g_terms=nt)
            profs[nt] = dust.dust_profile_read()
            dust.dust_profile_disable()
        st = dust.dust_last_device_error()[0]
        return wl, s, profs, st

    wl, s, profs, st = run_wgrad(3, (1, 2))
    flops = 2.0 * wl.N * s.d_in * s.d_out
    for nt, key_name in ((1, "gw_cfg3"), (2, "gw_cfg3_two_terms")):
        gw_ms, n = _prof_avg(profs[nt], "gw_bf16_tcgen05")
        sk_ms, _ = _prof_avg(profs[nt], "gw_splitk_reduce")
        tf = flops / (gw_ms / 1e3) / 1e12
        out[key_name] = {
            "workload": describe(wl), "kernel": "gw_bf16_tcgen05", "g_terms": nt, "launches": n,
            "ms": round(gw_ms, 5), "tflops": round(tf, 1),
            "mma_tflops": round(nt * tf, 1), "peak": peaks["bf16_tflops"],
            "frac": round(tf / peaks["bf16_tflops"], 4), "target": 0.6 if nt == 1 else None,
            "splitk_reduce_ms": None if sk_ms is None else round(sk_ms, 5), "status": st,
            "peak_source": peaks["source"] + " (burst)",
            "note": ("g rounded once to bf16: the contraction the 60% target names"
                     if nt == 1 else "g as hi + lo bf16 terms (the default): twice the "
                     "tensor-core work; frac counts the algorithmic 2 N d_in d_out flops only")}

    wl, s, profs, st = run_wgrad(4)
    prof = profs[dust.G_TERMS]
    gh_ms, n = _prof_avg(prof, "ghat_reduce_draws")
    gw4_ms, _ = _prof_avg(prof, "gw_bf16_tcgen05")
    streams = 4.0 * wl.K * wl.N + 2.0 * wl.N * s.d_out
    gbs = streams / (gh_ms / 1e3) / 1e9
    gn = wl.N * s.d_out * wl.K / (gh_ms / 1e3) / 1e9
    roof = alu_roofline("ghat_reduce_draws", gn, sms, peaks)
    out["reduction_streams"] = {
        "workload": describe(wl), "kernel": "ghat_reduce_draws", "launches": n,
        "ms": round(gh_ms, 4), "stream_bytes": streams, "gbs": round(gbs, 2),
        "frac_hbm": round(gbs / peaks["hbm_gbs"], 5), "target_hbm": 0.7,
        "gnormal_s": round(gn, 2), "alu_bound": roof["peak"], "binding_pipe": roof["binding_pipe"],
        "frac_alu": roof["frac"],
        "note": "the noise regeneration (ALU) bounds this kernel; its HBM streams are "
                f"{streams / 1e6:.0f} MB per launch",
        "gw_cfg4_tflops": round(2.0 * wl.N * s.d_in * s.d_out / (gw4_ms / 1e3) / 1e12, 1),
        "status": st}
    torch.cuda.empty_cache()

    # credit scan on a shape larger than L2
    K, N = 64, 1 << 22
    g = torch.Generator(device=dev)
    g.manual_seed(1234)
    loss = torch.randn((K, N), generator=g, device=dev, dtype=torch.float32)
    r = torch.empty_like(loss)
    cu = torch.from_numpy(workloads.random_segments(77, N, 256, 2048)).to(dev)
    ws = torch.empty(dust.dust_workspace_size(dust.DUST_OP_CREDIT, dust.DUST_F32, N, 0, 0, K),
                     dtype=torch.uint8, device=dev)
    # best of five groups of ten back-to-back launches, as the HBM copy peak is a best of ten
    groups = [_time_probe(lambda: dust.dust_credit(loss, cu, 0.99, r, ws), torch, reps=10)
              for _ in range(5)]
    ms = min(groups)
    gbs = 8.0 * K * N / (ms / 1e3) / 1e9
    out["credit_stress"] = {"K": K, "N": N, "segments": "packed U[256, 2048]", "gamma": 0.99,
                            "ms": round(ms, 4), "ms_mean_of_groups": round(sum(groups) / 5, 4),
                            "gbs": round(gbs, 1),
                            "frac_hbm": round(gbs / peaks["hbm_gbs"], 4), "target": 0.7,
                            "status": dust.dust_last_device_error()[0],
                            "note": "2 GiB moved per launch, larger than L2: no flush needed; "
                                    "best of 5 groups of 10 launches (the HBM copy peak is "
                                    "the best of 10 copies)"}
    del loss, r, ws
    torch.cuda.empty_cache()

    # credit latency at each workload's own size (L2-resident; the flush precedes each call)
    lat = {}
    for cfg in (2, 3, 4):
        wl = workloads.WORKLOADS[cfg]
        cu_np = workloads.generate(cfg, n_layers=0).cu_seqlens if wl.packed else \
            workloads.cu_seqlens_from_lengths([wl.seq_len] * wl.n_seq)
        loss = torch.from_numpy(workloads.gaussian_losses(cfg, wl.K, wl.N)).to(dev)
        r = torch.empty_like(loss)
        cu = torch.from_numpy(cu_np).to(dev)
        ws = torch.empty(dust.dust_workspace_size(dust.DUST_OP_CREDIT, 0, wl.N, 0, 0, wl.K),
                         dtype=torch.uint8, device=dev)
        dust.dust_credit(loss, cu, wl.gamma, r, ws)
        torch.cuda.synchronize(dev)
        dust.dust_profile_enable(1 << 10)
        for _ in range(reps):
            flush.zero_()
            dust.dust_credit(loss, cu, wl.gamma, r, ws)
        t, _ = _prof_avg(dust.dust_profile_read(), "credit_scan")
        dust.dust_profile_disable()
        lat[f"cfg{cfg}"] = {"K": wl.K, "N": wl.N, "us": round(t * 1e3, 2),
                            "gbs": round(8.0 * wl.K * wl.N / (t / 1e3) / 1e9, 1)}
    out["credit_latency"] = lat
    return out


def run_gpu(args, rank: int, world: int, local_rank: int) -> None:
    import torch
    import torch.distributed as dist

    import zeroth_order_transformer_b200 as dust
    from zeroth_order_transformer_b200 import distributed as zd

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)
    data = workloads.generate(args.workload, n_layers=args.layers)
    wl = data.wl
    gamma = headline_gamma(wl, args.gamma)
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
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stack = len(layers) > 1
    red = (lambda G: dist.all_reduce(G)) if world > 1 else None

    if stack:
        st = dust.DustStack([(x, W, u, s.layer_id) for s, x, W, u in layers], wl.K)
        GWs = st.G_W
    else:
        s1, x1, W1, u1 = layers[0]
        ws_bytes = max(dust.dust_workspace_size(op, 1 if wl.dtype == "bf16" else 0, wl.N,
                                                s1.d_in, s1.d_out, wl.K) for op in range(3))
        ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        dloss = torch.empty((wl.K, wl.N), dtype=torch.float32, device=dev)
        r = torch.empty((wl.K, wl.N), dtype=torch.float32, device=dev)
        GWs = [torch.empty((s1.d_out, s1.d_in), dtype=torch.float32, device=dev)]

    def step(g=gamma):
        if stack:
            # the grouped calls, one launch per step for all layers; on several GPUs the
            # weight estimates are summed in buckets overlapped with the later layers' work
            st.estimate(cu, wl.sigma, g, wl.seed, 0, rank * wl.N, reduce=red,
                        buckets=args.buckets)
            return GWs
        key = dust.NoiseKey(wl.seed, s1.layer_id, 0, rank * wl.N)
        dust.dust_noisy_linear_fwd(x1, W1, u1, wl.K, wl.sigma, key, dloss, ws)
        dust.dust_credit(dloss, cu, g, r, ws)
        dust.dust_weight_grad(r, x1, s1.d_out, wl.K, wl.sigma, key, GWs[0], False, None, ws)
        if red is not None:
            red(GWs[0])
        return GWs

    def timed(n_steps, g=gamma, profile=False):
        """Device milliseconds per step (max over ranks) of n_steps steps, L2 flushed before
        each, bracketed by barriers and device synchronisation."""
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_steps)]
        stops = [torch.cuda.Event(enable_timing=True) for _ in range(n_steps)]
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        if profile:
            dust.dust_profile_enable(1 << 16)
        for k in range(n_steps):
            flush.zero_()
            starts[k].record(stream)
            step(g)
            stops[k].record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        total = sum(a.elapsed_time(b) for a, b in zip(starts, stops))
        if world > 1:
            t = torch.tensor([total], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            total = float(t.item())
        return total / n_steps

    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()

    # ---- timed region
    sampler = ClockSampler(local_rank) if rank == 0 else None
    ms_per_step = timed(args.steps, profile=True)
    clocks = sampler.stop() if sampler else None
    prof = dust.dust_profile_read()
    dust.dust_profile_disable()
    dev_status = dust.dust_last_device_error()[0]
    units = wl.N * wl.K * len(layers) * world
    # tokens*draws per layer processed per second: N K n_layers n_gpus / step time
    value = units / (ms_per_step / 1e3)

    # ---- the other discounts of the workload (the stack sweeps gamma over {0, 0.9, 0.99})
    sweep = None
    if len(wl.gammas) > 1 and not args.no_sweep:
        sweep = []
        for g in wl.gammas:
            step(g)
            ms = timed(max(3, min(args.steps, 10)), g)
            sweep.append({"gamma": g, "ms_per_step": round(ms, 4),
                          "value": units / (ms / 1e3)})

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

    def work_of(n):
        if stack and not n.endswith("_grouped"):
            return None, None, None
        return kernel_work(n, wl, shapes if n.endswith("_grouped") else [s0])

    for n, info in kernels.items():
        bound, amount, what = work_of(n)
        if amount is None:
            continue
        per_s = amount / (info["ms_avg"] / 1e3)
        info[{"normals": "gnormals_per_s", "flops": "tflops", "bytes": "gbs"}[what]] = round(
            per_s / (1e12 if what == "flops" else 1e9), 2)
    # dominant kernel: the largest total time among kernels with a defined algorithmic work
    dominant = next((n for n in kernels if work_of(n)[1] is not None), None)
    roofline = None
    if dominant:
        bound, amount, what = work_of(dominant)
        avg_s = kernels[dominant]["ms_avg"] / 1e3
        if bound == "alu":
            roofline = alu_roofline(dominant, amount / avg_s / 1e9, sms, peaks)
            roofline.update(generator_ceiling(dust, torch, dev))
            roofline["frac_of_generator"] = round(
                roofline["achieved"] / roofline["generator_gnormal_s"], 4)
        elif bound == "tensor":
            ach = amount / avg_s / 1e12
            roofline = {"kernel": dominant, "bound": "tensor", "achieved": round(ach, 2),
                        "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                        "frac": round(ach / peaks["bf16_tflops_sustained"], 4), "traffic": None,
                        "peak_source": peaks["source"] + " (sustained)"}
        elif bound == "hbm":
            ach = amount / avg_s / 1e9
            roofline = {"kernel": dominant, "bound": "hbm", "achieved": round(ach, 2),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": None,
                        "peak_source": peaks["source"]}
        if roofline is not None:
            roofline["units_per_launch"] = amount
            tr, src = (measured_traffic(dominant, wl.name) if len(layers) == len(wl.layers)
                       else (None, None))
            roofline["traffic"] = tr
            roofline["traffic_source"] = src or ("null: no ncu capture of the current sources "
                                                 "of this kernel on this workload")

    # ---- end to end through the public API, host buffers, copies inside the timed region
    e2e = None
    if not args.no_e2e:
        host_in = []
        h2d = 0
        for s, x, W, u in layers:
            hx, hW, hu = (t.cpu().pin_memory() for t in (x, W, u))
            host_in.append((hx, hW, hu))
            h2d += sum(t.numel() * t.element_size() for t in (hx, hW, hu))
        if stack:
            G_host = torch.empty(st.G_W_flat.shape, dtype=torch.float32, pin_memory=True)
            d2h = G_host.numel() * 4

            def e2e_step():
                st.estimate_from_host(host_in, data.cu_seqlens, wl.sigma, gamma, wl.seed,
                                      G_host, chunks=args.buckets, reduce=red,
                                      token_offset=rank * wl.N)
        else:
            host_layer = dust.DustLayer(wl.N, s1.d_in, s1.d_out, wl.K, tdt, dev)
            G_host = torch.empty(GWs[0].shape, dtype=torch.float32, pin_memory=True)
            d2h = G_host.numel() * 4

            def e2e_step():
                hx, hW, hu = host_in[0]
                host_layer.estimate_from_host(
                    hx, hW, hu, data.cu_seqlens, wl.sigma, gamma,
                    dust.NoiseKey(wl.seed, s1.layer_id, 0, rank * wl.N), G_host,
                    chunks=4, reduce=red)

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
               "ms_per_step": e_ms / args.steps,
               "note": ("inputs uploaded from pinned host memory in buckets of layers (the "
                        "stack) or runs of whole sequences (one layer), each overlapped with the "
                        "previous one's estimate; G_W read back, bucket by bucket for the stack")}
        del host_in

    # ---- optional: the optimizer step fused into the weight estimate (single-layer workloads)
    opt_line = None
    if args.optimizer != "none" and not stack:
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

    # ---- the path's numeric targets, measured in this run (one GPU)
    targets = None
    if world == 1 and not args.no_targets:
        targets = measure_targets(dust, torch, dev, peaks, flush, reps=max(5, min(args.steps, 20)))

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        done, el, cores, desc = oracle_sample(data, args.cpu_tokens, args.cpu_seconds, gamma)
        cpu = {"value": done / el, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": desc, "seconds": round(el, 2)}

    n_launch = sum(v["launches"] for v in kernels.values())
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "operands": "bf16 x, W, u; u32 Philox words",
        "data": "synthetic (seeded; shapes of the Dust page's transformer layers)",
        "config": {"workload": describe(wl, gamma)
                   + (f"; first {len(layers)} layers only" if len(layers) < len(wl.layers) else ""),
                   "tokens_per_gpu": wl.N, "K": wl.K, "layers": len(layers),
                   "layer_shapes": sorted({f"{s.d_in}->{s.d_out}" for s in shapes}),
                   "gamma": gamma,
                   "parallelism": (f"dp{world}: one batch per GPU, NCCL all-reduce of G_W"
                                   + (f" in {args.buckets} buckets overlapped with the weight "
                                      "estimate" if stack else "")),
                   "l2": "flushed (256 MiB write) before every timed step"},
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": n_launch,
        "device_status": dev_status,
        "clocks": clocks,
        "gamma_sweep": sweep,
        "targets": targets,
        "kernels": kernels,
        "source_digest": source_digest(),
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
            roofline = alu_roofline(n, rate / 1e9, sms, peaks)
        elif bound == "hbm":
            roofline = {"kernel": n, "bound": "hbm", "achieved": round(rate / 1e9, 2),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(rate / 1e9 / peaks["hbm_gbs"], 4), "traffic": None}
        elif bound == "tensor":
            roofline = {"kernel": n, "bound": "tensor", "achieved": round(rate / 1e12, 2),
                        "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": round(rate / 1e12 / peaks["bf16_tflops"], 4), "traffic": None}
        roofline.setdefault("peak_source", peaks["source"])
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
        roofline.update(generator_ceiling(dust, torch, dev))
        roofline["frac_of_generator"] = round(roofline["achieved"] / roofline["generator_gnormal_s"],
                                              4)
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
    if roofline is not None:
        roofline["traffic"], roofline["traffic_source"] = measured_traffic(roofline["kernel"],
                                                                           hw.name)
    if roofline is not None and roofline["bound"] == "alu":
        roofline.update(generator_ceiling(dust, torch, dev))
        roofline["frac_of_generator"] = round(roofline["achieved"] / roofline["generator_gnormal_s"],
                                              4)
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
    ap.add_argument("--workload", type=int, default=5, choices=sorted(workloads.WORKLOADS),
                    help="workload id (default 5: the 48 linear layers of a 12-block stack)")
    ap.add_argument("--gamma", type=float, default=None,
                    help="credit discount of the headline (default 0.9 for the stack, else the "
                         "workload's own)")
    ap.add_argument("--layers", type=int, default=None,
                    help="only the first LAYERS layers of a stack workload (small profiling "
                         "cases; the line then says so)")
    ap.add_argument("--buckets", type=int, default=12,
                    help="buckets of consecutive layers: the stack's G_W all-reduce (N > 1) and "
                         "the end-to-end leg's upload pipeline")
    ap.add_argument("--no-sweep", action="store_true", help="skip the gamma sweep")
    ap.add_argument("--no-targets", action="store_true",
                    help="skip the contraction / scan / reduction target measurements")
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
    if args.gpus != world and rank == 0:
        print(f"bench.py: --gpus {args.gpus} but {world} rank(s) were launched; the line reports "
              f"the {world} rank(s) that run (launch N > 1 with torch.distributed.run "
              f"--nproc-per-node N)", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
