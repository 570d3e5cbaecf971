"""Benchmark of the TTT layer forward on B200: head-tokens/s (B x H x T / s).

One step is one call of the layer forward (every stage of the hot path, fused in
one kernel) over the whole workload, inputs resident in HBM.  Defaults: the
TTT-Linear + LN + residual workload with B=16, H=32, d=64, T=8192, b=16 (bf16
Q/K/V).  Under torchrun every rank runs its own batch shard of the same size
(weak scaling, no collective on the data path); the step time is the max over
ranks.  ``--impl reference`` times the fp64 CPU oracle instead, on a bounded
sample of the same workload.

Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from test_sequence_modeling_b200 import inputs as I  # noqa: E402

METRIC = "TTT layer fwd tokens/s (B×H×T/s) on 1 B200; % of roofline (HBM vs tensor)"
UNIT = "head-tokens/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# The sources the tensor-core kernel is compiled from: a committed DRAM-traffic
# record is only reported while these are unchanged.
KERNEL_SOURCES = tuple("test_sequence_modeling_b200/csrc/" + f
                       for f in ("tc_linear.cuh", "sm100.cuh", "device_status.cuh"))


# --- workload accounting --------------------------------------------------------

def flops_per_head_token(cfg) -> float:
    """Dense matmul FLOPs of the dual form per head-token (elementwise work not counted).
    Linear: [K;Q] W (4d^2), K^T G (2d^2), tril(QK^T) (2bd) and its product with G (2bd).
    MLP: 14 d h + 4 b (d + h)."""
    d, b, h = cfg.d, cfg.b, cfg.hidden
    if cfg.variant == "mlp":
        return 14.0 * d * h + 4.0 * b * (d + h)
    return 6.0 * d * d + 4.0 * b * d


def bytes_per_launch(cfg, units=None) -> float:
    """Algorithmic HBM bytes of one call: Q, K, V read once, eta read once, Z written
    once, and each unit's initial state read and final state written once."""
    units = cfg.units if units is None else units
    qkv = 2 if cfg.dtype == "bf16" else 4
    per_token = 3 * cfg.d * qkv + 4 + 4 * cfg.d
    state = 4 * (2 * cfg.d * cfg.hidden if cfg.variant == "mlp" else cfg.d * cfg.d)
    return units * (cfg.T * per_token + 2 * state)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(sources=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(os.path.basename(rel).encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def committed_traffic(workload: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu summary, if it
    was taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t[workload]
        if e.get("kernel_source_sha") == kernel_source_sha(tuple(e["kernel_sources"])):
            return float(e["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


# --- clocks ------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.proc = None
        self.out = []
        self.gpu_id = gpu_id

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            text, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            text, _ = self.proc.communicate()
        return self.summarize(text)

    @staticmethod
    def summarize(text):
        """Median SM clock under load, the max clock, the throttle reasons seen, and a
        verdict: "rejected: ..." for a hardware or thermal slowdown, or for an SM clock
        well below max with no reason (a leftover clock lock); sw_power_cap is kept."""
        rows = [r.split(", ") for r in text.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.strip() == "Active"})
        loaded = [s for s in sm if mx and s > 0.5 * max(mx)] or sm
        info = {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}
        bad = [r for r in reasons if r != "sw_power_cap"]
        if bad:
            info["verdict"] = "rejected: " + ", ".join(bad)
        elif not reasons and info["sm_mhz"] and info["sm_max_mhz"] and info["sm_mhz"] < 0.85 * info["sm_max_mhz"]:
            info["verdict"] = "rejected: SM clock well below max with no reason"
        else:
            info["verdict"] = "ok"
        return info


def gpu_id_for(torch, device) -> str | None:
    try:
        uuid = str(torch.cuda.get_device_properties(device).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:  # noqa: BLE001
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        return vis.split(",")[0] if vis else None


# --- reference arm and CPU baseline: the fp64 oracle on host cores -------------------

def oracle_sample(cfg, units, T, nthreads):
    """Run the oracle on `units` whole units truncated to T tokens; returns seconds."""
    import oracle
    sub = cfg.replace(T=T)
    data = {"Q": [], "K": [], "V": [], "eta": []}
    for bi, hi in units:
        q, k, v, e = I.unit_inputs(cfg, bi, hi, T=T)
        for n, a in zip(("Q", "K", "V", "eta"), (q, k, v, e)):
            data[n].append(a.astype(np.float64))
    Q, K, V = (np.stack(data[n])[:, None] for n in ("Q", "K", "V"))
    eta = np.stack(data["eta"])[:, None]
    # Each sampled unit runs as its own batch row with its head's parameters.
    heads = [hi for _, hi in units]
    P = {k: np.stack([I.head_params(sub, h)[k] for h in heads]).astype(np.float64)
         for k in I.head_params(sub, 0)}
    t0 = time.perf_counter()
    if cfg.variant == "mlp":
        Hn, d, h = len(units), cfg.d, cfg.hidden
        params = np.concatenate([P["W1"].reshape(Hn, -1), P["W2"].reshape(Hn, -1)], axis=1)
        # one "head" per sampled unit: lay the units out as B=1, H=len(units)
        oracle.default().forward(oracle.MLP_LN, Q.transpose(1, 0, 2, 3), K.transpose(1, 0, 2, 3),
                                 V.transpose(1, 0, 2, 3), eta.transpose(1, 0, 2), params, cfg.b,
                                 P["gamma"], P["beta"], cfg.ln_eps, hidden=h, nthreads=nthreads)
    else:
        kind = oracle.LINEAR if cfg.variant == "linear" else oracle.LINEAR_LN
        Hn, d = len(units), cfg.d
        ln = kind == oracle.LINEAR_LN
        oracle.default().forward(kind, Q.transpose(1, 0, 2, 3), K.transpose(1, 0, 2, 3),
                                 V.transpose(1, 0, 2, 3), eta.transpose(1, 0, 2),
                                 P["W0"].reshape(Hn, d * d), cfg.b, P["gamma"] if ln else None,
                                 P["beta"] if ln else None, cfg.ln_eps, nthreads=nthreads)
    return time.perf_counter() - t0


def sample_plan(cfg, budget_cpu_s, cores):
    """Units and tokens of a bounded oracle sample taking about budget_cpu_s of CPU time
    (summed over `cores` threads)."""
    T_cal = min(cfg.T, 1024)
    t_cal = oracle_sample(cfg, [(0, 0)], T_cal, 1)
    per_unit = t_cal * cfg.T / T_cal
    n_units = int(budget_cpu_s / max(per_unit, 1e-6))
    if n_units >= cores:
        n_units = min(cfg.units, max(cores, (n_units // cores) * cores))
        T = cfg.T
    else:  # fewer whole units than cores: shorten the sequences instead
        n_units = min(cfg.units, cores)
        T = max(cfg.b, int(budget_cpu_s / cores / (t_cal / T_cal)) // cfg.b * cfg.b)
        T = min(T, cfg.T)
    rng = np.random.default_rng(123)
    idx = sorted(rng.choice(cfg.units, size=n_units, replace=False).tolist())
    return [divmod(int(u), cfg.H) for u in idx], T


def cpu_baseline(cfg, budget_cpu_s=20.0):
    import oracle
    cores = oracle.default().default_threads()
    units, T = sample_plan(cfg, budget_cpu_s, cores)
    dt = oracle_sample(cfg, units, T, cores)
    return {"value": len(units) * T / dt, "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"{len(units)} of {cfg.units} (batch, head) units x {T} tokens of {cfg.name}, "
                      f"fp64 primal oracle on {cores} threads, {dt:.2f} s"}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    cores = oracle.default().default_threads()
    units, T = sample_plan(cfg, 2.0 * cores, cores)  # ~2 s of wall time per step
    for _ in range(args.warmup):
        oracle_sample(cfg, units, T, cores)
    times = [oracle_sample(cfg, units, T, cores) for _ in range(args.steps)]
    tot = sum(times)
    value = args.steps * len(units) * T / tot
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(cfg, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": f"each step: {len(units)} of {cfg.units} (batch, head) units x "
                                   f"{T} tokens of {cfg.name}, fp64 primal oracle"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def tc_path(cfg, path):
    return cfg.dtype == "bf16" and cfg.b == 16 and path != "simt"


def dtype_of(cfg, path):
    """Arithmetic type of the path that runs.  TTT-Linear on tensor cores: bf16
    operands (fp32 values split into bf16 hi + lo), fp32 accumulation.  TTT-MLP on
    tensor cores: tf32 operands, fp16 for the three contractions over the hidden
    width, fp32 accumulation.  The CUDA-core paths are fp32 throughout."""
    if not tc_path(cfg, path):
        return "f32"
    return "tf32+f16" if cfg.variant == "mlp" else "bf16"


# Nominal dense tf32 : bf16 tensor throughput of a B200 (1.1 vs 2.25 PFLOP/s).
TF32_PER_BF16 = 1.1 / 2.25


def tensor_peak_scale(cfg, path):
    """Peak of the path's contractions relative to the measured bf16 peak.  The
    TTT-MLP tensor-core path runs, per head-token, 8 d h + 4 b d + 2 b h FLOPs as
    tf32 ([K;Q] W1, both state updates, the masked Q K^T products) and 6 d h + 2 b h
    as fp16 (X2 W2, Zq2 W2, G3 W2^T and the Gram Zq2 X2^T); each kind at its own
    peak gives the time at the roofline."""
    if cfg.variant != "mlp" or not tc_path(cfg, path):
        return 1.0
    d, b, h = cfg.d, cfg.b, cfg.hidden
    tf32 = 8.0 * d * h + 4.0 * b * d + 2.0 * b * h
    f16 = 6.0 * d * h + 2.0 * b * h
    return (tf32 + f16) / (tf32 / TF32_PER_BF16 + f16)


def workload_config(cfg, args, world=1):
    return {"workload": cfg.name, "variant": cfg.variant, "B_per_gpu": cfg.B, "H": cfg.H,
            "T": cfg.T, "d": cfg.d, "b": cfg.b, "qkv_dtype": cfg.dtype,
            "global_batch": cfg.B * world, "sharding": f"batch over {world} GPU(s), no collective",
            "l2": "inputs larger than L2 (no flush needed)"
            if bytes_per_launch(cfg) > 4 * L2_BYTES else "L2 flushed between steps",
            "path": args.path}


# --- our arm ----------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="linear_ln_B16H32T8192", choices=I.CONFIG_ORDER)
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--e2e-chunks", type=int, default=16,
                    help="batch chunks whose copies overlap the kernels in the end-to-end line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None, help="override B (smaller profiling cases)")
    ap.add_argument("--seq", type=int, default=None, help="override T (smaller profiling cases)")
    ap.add_argument("--decode", action="store_true",
                    help="time the primal-form decode step (TTT-Linear + LN, B=512 H=32, bf16 q/k/v) "
                         "instead of the forward")
    ap.add_argument("--decode-mlp", action="store_true",
                    help="the same for the TTT-MLP decode step")
    ap.add_argument("--momentum", action="store_true",
                    help="time the whole-sequence forward with the momentum and decay update (TTT-Linear + LN, "
                         "B=16 H=32 T=8192)")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward pass of TTT-Linear + LN on the bench workload (B=16 H=32 T=8192)")
    ap.add_argument("--decode-momentum", action="store_true",
                    help="the decode step with the momentum and decay update (TTT-Linear + LN, or with "
                         "--decode-mlp TTT-MLP)")
    args = ap.parse_args()
    single = args.backward or args.momentum or args.decode or args.decode_mlp or args.decode_momentum
    if single and int(os.environ.get("RANK", "0")) != 0:
        return 0  # these lines are measured on one GPU: under a multi-rank launch only rank 0 runs
    if args.backward:
        return run_backward(args)
    if args.momentum:
        return run_momentum(args)
    if args.decode or args.decode_mlp or args.decode_momentum:
        return run_decode(args, mlp=args.decode_mlp, momentum=args.decode_momentum)
    cfg = I.CONFIGS[args.workload]
    if args.batch is not None or args.seq is not None:
        cfg = cfg.replace(B=args.batch or cfg.B, T=args.seq or cfg.T,
                          name=f"{cfg.name}[B={args.batch or cfg.B},T={args.seq or cfg.T}]")
    if args.impl == "reference":
        return run_reference(args, cfg)

    import torch
    import torch.distributed as dist

    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    small = cfg.units * cfg.T * cfg.d * 3 * 2 < 4 * L2_BYTES
    lib = _lib.load()
    ttt.set_path({"auto": ttt.TTT_PATH_AUTO, "simt": ttt.TTT_PATH_SIMT, "tc": ttt.TTT_PATH_TC}[args.path])

    from test_sequence_modeling_b200 import sharding
    cfg, batch_offset = sharding.shard(cfg, world, rank)
    data = I.make_inputs(cfg, batch_offset=batch_offset)
    if data["qkv_bits"]:
        host = {k: torch.from_numpy(data[k].view(np.int16)).view(torch.bfloat16) for k in "QKV"}
    else:
        host = {k: torch.from_numpy(data[k]) for k in "QKV"}
    for k in ("eta", "W0", "W1", "W2", "gamma", "beta"):
        if k in data:
            host[k] = torch.from_numpy(np.ascontiguousarray(data[k]))
    d_in = {k: v.to(dev) for k, v in host.items()}
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    outs = {"Z": torch.empty(B, H, T, d, device=dev)}
    if cfg.variant == "mlp":
        outs["W1_out"] = torch.empty(B, H, d, cfg.hidden, device=dev)
        outs["W2_out"] = torch.empty(B, H, cfg.hidden, d, device=dev)
    else:
        outs["W_out"] = torch.empty(B, H, d, d, device=dev)
    flush = torch.empty(2 * L2_BYTES // 4, device=dev) if small else None
    stream = torch.cuda.current_stream(dev)

    def step(src=d_in, dst=outs):
        if cfg.variant == "linear":
            ttt.ttt_linear_fwd(src["Q"], src["K"], src["V"], src["eta"], src["W0"], cfg.b,
                               Z=dst["Z"], W_out=dst["W_out"], stream=stream)
        elif cfg.variant == "linear_ln":
            ttt.ttt_linear_ln_fwd(src["Q"], src["K"], src["V"], src["eta"], src["W0"], src["gamma"],
                                  src["beta"], cfg.b, cfg.ln_eps, Z=dst["Z"], W_out=dst["W_out"],
                                  stream=stream)
        else:
            ttt.ttt_mlp_fwd(src["Q"], src["K"], src["V"], src["eta"], src["W1"], src["W2"],
                            src["gamma"], src["beta"], cfg.b, cfg.ln_eps, Z=dst["Z"],
                            W1_out=dst["W1_out"], W2_out=dst["W2_out"], stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error during warm-up")

    clocks = ClockSampler(gpu_id_for(torch, local))
    clocks.start()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    n0 = lib.ttt_launch_count()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    kernel_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(kernel_ms) if flush is not None else t_start.elapsed_time(t_end)
    status = ttt.last_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    total_ms, kernel_avg_ms = sharding.max_over_ranks([total_ms, statistics.mean(kernel_ms)], dist, dev)
    ms_per_step = total_ms / args.steps
    value = world * cfg.head_tokens * args.steps / (total_ms / 1e3)

    # End to end through the public binding: pinned host inputs in, host outputs back.
    e2e = None if args.e2e_steps <= 0 else measure_e2e(args, cfg, host, outs, d_in, step, stream,
                                                       barrier, world, dev, torch, dist)
    peaks, peak_kind = load_peaks()
    nbytes = bytes_per_launch(cfg)
    nflops = flops_per_head_token(cfg) * cfg.head_tokens
    return finish(args, cfg, world, rank, value, ms_per_step, kernel_avg_ms, clock_info, launches,
                  e2e, peaks, peak_kind, nbytes, nflops, dist)


# fp32 FMA peak of the CUDA cores: 148 SMs x 128 FP32 lanes x 2 flops x 1965 MHz.
ALU_F32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def run_momentum_mlp(args):
    """One launch of ttt_mlp_momentum_fwd over the TTT-MLP workload (B=8 H=32 T=8192, b=16)."""
    import torch
    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = I.CONFIGS["mlp_B8H32T8192"]
    cfg = cfg.replace(B=args.batch or cfg.B, T=args.seq or cfg.T)  # smaller profiling cases
    data = I.make_inputs(cfg)
    B, H, T, d, b, h = cfg.B, cfg.H, cfg.T, cfg.d, cfg.b, cfg.hidden
    qkv = {k: torch.from_numpy(data[k].view(np.int16)).to(dev).view(torch.bfloat16) for k in "QKV"}
    t = {k: torch.from_numpy(np.ascontiguousarray(data[k])).to(dev) for k in ("eta", "W1", "W2", "gamma", "beta")}
    alpha, lam = (torch.from_numpy(x).to(dev) for x in I.momentum_rates(cfg))
    stream = torch.cuda.current_stream(dev)
    lib = _lib.load()

    def step():
        return ttt.ttt_mlp_momentum_fwd(qkv["Q"], qkv["K"], qkv["V"], t["eta"], alpha, lam, t["W1"], t["W2"],
                                        t["gamma"], t["beta"], b, cfg.ln_eps, stream=stream)

    outs = step()
    del outs
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(torch, 0))
    clocks.start()
    n0 = lib.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1) / args.steps
    units, N = B * H, T // b
    # Multiply-adds per mini-batch: K W1, X2 W2, G3 W2^T (3 b d h), Q W1 + Q S1 and
    # Zq2 W2 + Zq2 S2 (4 b d h), the two rank-b updates of W and S of both layers
    # (4 b d h), the masked Grams and their products (b^2 (2 h + 2 d)).
    flops = 2.0 * units * N * (11 * b * d * h + 2 * b * b * (h + d))
    achieved = flops / (ms / 1e3) / 1e12
    line = {
        "metric": "TTT-MLP momentum/decay forward tokens/s (B x H x T / s)",
        "value": units * T / (ms / 1e3), "unit": "head-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "momentum_" + cfg.name, "B": B, "H": H, "T": T, "d": d, "b": b,
                   "hidden": h, "qkv_dtype": "bf16", "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": ALU_F32_TFLOPS, "unit": "TFLOP/s",
                     "frac": achieved / ALU_F32_TFLOPS, "traffic": None,
                     "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1965 MHz (CUDA-core fp32 FMA)",
                     "flops_per_launch": flops},
        "clocks": clock_info, "gpu_launches": int(launches),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_backward_mlp(args):
    """One launch of ttt_mlp_bwd over the TTT-MLP workload (B=8 H=32 T=8192, b=16)."""
    import torch
    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = I.CONFIGS["mlp_B8H32T8192"]
    cfg = cfg.replace(B=args.batch or cfg.B, T=args.seq or cfg.T)  # smaller profiling cases
    data = I.make_inputs(cfg)
    B, H, T, d, b, h = cfg.B, cfg.H, cfg.T, cfg.d, cfg.b, cfg.hidden
    qkv = {k: torch.from_numpy(data[k].view(np.int16)).to(dev).view(torch.bfloat16) for k in "QKV"}
    t = {k: torch.from_numpy(np.ascontiguousarray(data[k])).to(dev) for k in ("eta", "W1", "W2", "gamma", "beta")}
    dZ, dW1T, dW2T = (torch.from_numpy(x).to(dev) for x in I.mlp_cotangents(cfg))
    stream = torch.cuda.current_stream(dev)
    lib = _lib.load()

    def step():
        return ttt.ttt_mlp_bwd(qkv["Q"], qkv["K"], qkv["V"], t["eta"], t["W1"], t["W2"], t["gamma"],
                               t["beta"], dZ, b, cfg.ln_eps, dW1_T=dW1T, dW2_T=dW2T, stream=stream)

    outs = step()  # allocates the outputs once; the timed steps reuse the allocator's blocks
    del outs
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(torch, 0))
    clocks.start()
    n0 = lib.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1) / args.steps
    units, N = B * H, T // b
    # Multiply-adds per mini-batch: the checkpoint pass's K W1, X2 W2, G3 W2^T and the
    # two state updates, the reverse pass's recomputation of those three and of
    # Q W1, Z2 W2, and its fourteen [b x d] x [d x h]-sized products (24 b d h in
    # all), plus the masked b x b Grams and their products (b^2 (8 h + 8 d)).
    flops = 2.0 * units * N * (24 * b * d * h + 8 * b * b * (h + d))
    achieved = flops / (ms / 1e3) / 1e12
    line = {
        "metric": "TTT-MLP backward tokens/s (B x H x T / s)",
        "value": units * T / (ms / 1e3), "unit": "head-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "backward_" + cfg.name, "B": B, "H": H, "T": T, "d": d, "b": b,
                   "hidden": h, "qkv_dtype": "bf16", "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": ALU_F32_TFLOPS, "unit": "TFLOP/s",
                     "frac": achieved / ALU_F32_TFLOPS, "traffic": None,
                     "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1965 MHz (CUDA-core fp32 FMA)",
                     "flops_per_launch": flops},
        "clocks": clock_info, "gpu_launches": int(launches),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_momentum(args):
    """The momentum and decay forward's own line: one step = one launch of
    ttt_linear_ln_momentum_fwd over the linear + LN workload (B=16 H=32 T=8192, b=16),
    of ttt_linear_momentum_fwd over another bf16 TTT-Linear (+ LN) workload named by
    ``--workload``, or (``--workload mlp_B8H32T8192``) of ttt_mlp_momentum_fwd over the
    TTT-MLP one.  TTT-Linear (+ LN) runs the tensor-core dual form by default (bf16
    operands, fp32 accumulation) and the exact-fp32 register-state kernel with
    ``--path simt``."""
    if args.workload.startswith("mlp"):
        return run_momentum_mlp(args)
    import torch
    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    base = I.CONFIGS[args.workload]
    if base.dtype != "bf16" or base.variant not in ("linear", "linear_ln"):
        raise SystemExit(f"--momentum takes a bf16 TTT-Linear (+ LN) or the TTT-MLP workload, not {args.workload}")
    cfg = base.replace(B=args.batch or base.B, T=args.seq or base.T)  # smaller profiling cases
    ln = cfg.variant == "linear_ln"
    data = I.make_inputs(cfg)
    B, H, T, d, b = cfg.B, cfg.H, cfg.T, cfg.d, cfg.b
    qkv = {k: torch.from_numpy(data[k].view(np.int16)).to(dev).view(torch.bfloat16) for k in "QKV"}
    eta = torch.from_numpy(np.ascontiguousarray(data["eta"])).to(dev)
    W0 = torch.from_numpy(data["W0"]).to(dev)
    ln_kw = dict(gamma=torch.from_numpy(data["gamma"]).to(dev), beta=torch.from_numpy(data["beta"]).to(dev),
                 eps=cfg.ln_eps) if ln else {}
    alpha, lam = (torch.from_numpy(x).to(dev) for x in I.momentum_rates(cfg))
    Z = torch.empty(B, H, T, d, device=dev)
    W_out, S_out = torch.empty(B, H, d, d, device=dev), torch.empty(B, H, d, d, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = _lib.load()
    ttt.set_path({"auto": ttt.TTT_PATH_AUTO, "simt": ttt.TTT_PATH_SIMT, "tc": ttt.TTT_PATH_TC}[args.path])

    def step():
        ttt.ttt_linear_momentum_fwd(qkv["Q"], qkv["K"], qkv["V"], eta, alpha, lam, W0, b, Z=Z, W_out=W_out,
                                    S_out=S_out, stream=stream, **ln_kw)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(torch, 0))
    clocks.start()
    n0 = lib.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1) / args.steps
    units = B * H
    # Algorithmic bytes: q, k, v (bf16), eta, alpha, lambda in and Z out per token;
    # W0 in and W_out, S_out out per unit.
    nbytes = units * (T * (3 * d * 2 + 3 * 4 + d * 4) + 3 * d * d * 4)
    peaks, peak_kind = load_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    full = args.path != "simt" and (B, T) == (base.B, base.T)
    traffic = committed_traffic("momentum_" + cfg.name) if full else None
    line = {
        "metric": ("TTT-Linear+LN" if ln else "TTT-Linear") + " momentum/decay forward tokens/s (B x H x T / s)",
        "value": units * T / (ms / 1e3), "unit": "head-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if args.path == "simt" else "bf16", "data": "synthetic",
        "config": {"workload": "momentum_" + cfg.name, "B": B, "H": H, "T": T, "d": d, "b": b,
                   "qkv_dtype": "bf16", "path": args.path, "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)", "algorithmic_bytes_per_launch": nbytes},
        "clocks": clock_info, "gpu_launches": int(launches),
    }
    print(json.dumps(line), flush=True)


def run_backward(args):
    """The backward pass's own line: one step = one launch of ttt_linear_ln_bwd over
    the linear + LN workload (B=16 H=32 T=8192, b=16) with its incoming gradients,
    or (``--workload mlp_B8H32T8192``) of ttt_mlp_bwd over the TTT-MLP workload."""
    if args.workload.startswith("mlp"):
        return run_backward_mlp(args)
    import torch
    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    cfg = I.CONFIGS["linear_ln_B16H32T8192"]
    cfg = cfg.replace(B=args.batch or cfg.B, T=args.seq or cfg.T)  # smaller profiling cases
    data = I.make_inputs(cfg)
    B, H, T, d, b = cfg.B, cfg.H, cfg.T, cfg.d, cfg.b
    qkv = {k: torch.from_numpy(data[k].view(np.int16)).to(dev).view(torch.bfloat16) for k in "QKV"}
    eta = torch.from_numpy(np.ascontiguousarray(data["eta"])).to(dev)
    W0, gamma, beta = (torch.from_numpy(data[k]).to(dev) for k in ("W0", "gamma", "beta"))
    dZ, dWT = (torch.from_numpy(x).to(dev) for x in I.cotangents(cfg))
    stream = torch.cuda.current_stream(dev)
    lib = _lib.load()

    def step():
        return ttt.ttt_linear_bwd(qkv["Q"], qkv["K"], qkv["V"], eta, W0, dZ, b, dW_T=dWT, gamma=gamma,
                                  beta=beta, eps=cfg.ln_eps, stream=stream)

    outs = step()  # allocates the outputs once; the timed steps reuse the allocator's blocks
    del outs
    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(torch, 0))
    clocks.start()
    n0 = lib.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1) / args.steps
    units, N = B * H, T // b
    # Multiply-adds of the dual-form backward per mini-batch (LN): the forward pass's
    # K W and K^T E (2 b d^2); the reverse pass's K W, Q W, P W^T, K dW, E dW^T,
    # dY W^T, Q^T P, K^T dY (8 b d^2) and the six masked b x b products (3 b^2 d).
    flops = 2.0 * units * N * (10 * b * d * d + 3 * b * b * d)
    achieved = flops / (ms / 1e3) / 1e12
    line = {
        "metric": "TTT-Linear+LN backward tokens/s (B x H x T / s)",
        "value": units * T / (ms / 1e3), "unit": "head-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": "backward_" + cfg.name, "B": B, "H": H, "T": T, "d": d, "b": b,
                   "qkv_dtype": "bf16", "l2": "inputs larger than L2 (no flush needed)"},
        "roofline": {"bound": "alu", "achieved": achieved, "peak": ALU_F32_TFLOPS, "unit": "TFLOP/s",
                     "frac": achieved / ALU_F32_TFLOPS, "traffic": None,
                     "peak_source": "148 SMs x 128 FP32 lanes x 2 x 1965 MHz (CUDA-core fp32 FMA)",
                     "flops_per_launch": flops},
        "clocks": clock_info, "gpu_launches": int(launches),
    }
    print(json.dumps(line), flush=True)


def run_decode(args, mlp=False, momentum=False):
    """The decode step's own line: one timed step = one mini-batch of 16 decode calls
    (positions 0..15) over B=512 x H=32 (batch, head) units, the state in HBM.
    ``momentum``: the step with the momentum and decay update."""
    import torch
    import test_sequence_modeling_b200 as ttt
    from test_sequence_modeling_b200 import _lib
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    if mlp:
        name = "decode_momentum_mlp_B512H32" if momentum else "decode_mlp_B512H32"
        cfg = I.CONFIGS["mlp_B8H32T8192"].replace(B=512, T=16, name=name)
    else:
        name = "decode_momentum_linear_ln_B512H32" if momentum else "decode_linear_ln_B512H32"
        cfg = I.CONFIGS["linear_ln_B16H32T8192"].replace(B=512, T=16, name=name)
    if args.batch:  # smaller profiling cases
        cfg = cfg.replace(B=args.batch)
    data = I.make_inputs(cfg)
    B, H, T, d = cfg.B, cfg.H, cfg.T, cfg.d
    qkv = {k: torch.from_numpy(data[k].view(np.int16)).to(dev).view(torch.bfloat16) for k in "QKV"}
    tok = [{k: qkv[k][:, :, t].contiguous() for k in "QKV"} for t in range(T)]
    eta = torch.from_numpy(np.ascontiguousarray(data["eta"])).to(dev)
    etas = [eta[:, :, t].contiguous() for t in range(T)]
    gamma = torch.from_numpy(data["gamma"]).to(dev)
    beta = torch.from_numpy(data["beta"]).to(dev)
    if mlp:
        h = cfg.hidden
        W1 = torch.from_numpy(data["W1"]).to(dev).unsqueeze(0).expand(B, H, d, h).contiguous()
        W2 = torch.from_numpy(data["W2"]).to(dev).unsqueeze(0).expand(B, H, h, d).contiguous()
        W1b, W2b = W1.clone(), W2.clone()
        if momentum:
            S1, S2 = torch.zeros_like(W1), torch.zeros_like(W2)
    else:
        W = torch.from_numpy(data["W0"]).to(dev).unsqueeze(0).expand(B, H, d, d).contiguous()
        W_base = W.clone()
        if momentum:
            S = torch.zeros_like(W)
    if momentum:
        alpha, lam = (torch.from_numpy(x).to(dev) for x in I.momentum_rates(cfg))
        als = [alpha[:, :, t].contiguous() for t in range(T)]
        lms = [lam[:, :, t].contiguous() for t in range(T)]
    z = torch.empty(B, H, d, device=dev)
    stream = torch.cuda.current_stream(dev)
    lib = _lib.load()

    def step():
        for t in range(T):
            if mlp and momentum:
                ttt.ttt_mlp_momentum_decode(tok[t]["Q"], tok[t]["K"], tok[t]["V"], etas[t], als[t], lms[t],
                                            W1, W2, W1b, W2b, S1, S2, gamma, beta, cfg.b, t, cfg.ln_eps,
                                            z=z, stream=stream)
            elif mlp:
                ttt.ttt_mlp_decode(tok[t]["Q"], tok[t]["K"], tok[t]["V"], etas[t], W1, W2, W1b, W2b, gamma,
                                   beta, cfg.b, t, cfg.ln_eps, z=z, stream=stream)
            elif momentum:
                ttt.ttt_linear_ln_momentum_decode(tok[t]["Q"], tok[t]["K"], tok[t]["V"], etas[t], als[t],
                                                  lms[t], W, W_base, S, gamma, beta, cfg.b, t, cfg.ln_eps,
                                                  z=z, stream=stream)
            else:
                ttt.ttt_linear_ln_decode(tok[t]["Q"], tok[t]["K"], tok[t]["V"], etas[t], W, W_base, gamma,
                                         beta, cfg.b, t, cfg.ln_eps, z=z, stream=stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(gpu_id_for(torch, 0))
    clocks.start()
    n0 = lib.ttt_launch_count()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = lib.ttt_launch_count() - n0
    clock_info = clocks.stop()
    if ttt.last_device_status() != 0:
        raise RuntimeError("device status error")
    ms = e0.elapsed_time(e1)
    units = B * H
    value = units * T * args.steps / (ms / 1e3)
    # Algorithmic bytes per mini-batch (16 calls) and unit: W_base and W read and W
    # written each call, W_base written once, q/k/v (bf16), eta and z per call.
    if mlp and momentum:  # W1b, W2b, W1, W2, S1, S2 read, W1, W2, S1, S2 written per call
        per_unit = T * (10 * d * cfg.hidden * 4 + 3 * d * 2 + 3 * 4 + d * 4) + 2 * d * cfg.hidden * 4
    elif mlp:  # W1b, W2b, W1, W2 read and W1, W2 written per call; the bases written once
        per_unit = T * (6 * d * cfg.hidden * 4 + 3 * d * 2 + 4 + d * 4) + 2 * d * cfg.hidden * 4
    elif momentum:  # W_base, W, S read and W, S written per call, plus alpha and lambda
        per_unit = T * (5 * d * d * 4 + 3 * d * 2 + 3 * 4 + d * 4) + d * d * 4
    else:
        per_unit = T * (3 * d * d * 4 + 3 * d * 2 + 4 + d * 4) + d * d * 4
    nbytes = units * per_unit
    peaks, peak_kind = load_peaks()
    achieved = nbytes / (ms / args.steps / 1e3) / 1e9
    line = {
        "metric": ("TTT-MLP" if mlp else "TTT-Linear+LN") + (" momentum/decay" if momentum else "")
        + " decode step tokens/s (B x H units, one token each per call)",
        "value": value, "unit": "head-tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "B": B, "H": H, "d": d, "b": cfg.b,
                   "step": "one mini-batch: 16 decode calls, positions 0..15", "qkv_dtype": "bf16",
                   "l2": "state larger than L2 (no flush needed)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)",
                     "algorithmic_bytes_per_step": nbytes},
        "clocks": clock_info, "gpu_launches": int(launches),
    }
    print(json.dumps(line), flush=True)


def measure_e2e(args, cfg, host, outs, d_in, step, stream, barrier, world, dev, torch, dist):
    """Through the C ABI's host-memory forward (ttt_fwd_host, via
    test_sequence_modeling_b200.host): pinned host inputs in, host outputs back,
    every step; the copies of one batch chunk overlap the forward of the next."""
    from test_sequence_modeling_b200.host import HostForward
    pin = {k: v.pin_memory() for k, v in host.items()}
    h_out = {k: torch.empty(v.shape, dtype=v.dtype, pin_memory=True) for k, v in outs.items()}
    h2d = sum(v.numel() * v.element_size() for v in pin.values())
    d2h = sum(v.numel() * v.element_size() for v in h_out.values())
    if cfg.variant == "mlp":
        params = [pin[k] for k in ("W1", "W2", "gamma", "beta")]
        w_shapes = [(cfg.H, cfg.d, cfg.hidden), (cfg.H, cfg.hidden, cfg.d)]
        w_keys = ["W1_out", "W2_out"]
    else:
        params = [pin["W0"]] + ([pin["gamma"], pin["beta"]] if cfg.variant == "linear_ln" else [])
        w_shapes = [(cfg.H, cfg.d, cfg.d)]
        w_keys = ["W_out"]
    fwd = HostForward(cfg.variant, pin["Q"], w_shapes, [p.shape for p in params], chunks=args.e2e_chunks,
                      device=dev)

    def e2e_step(after=None):
        return fwd.run(pin["Q"], pin["K"], pin["V"], pin["eta"], params, cfg.b, cfg.ln_eps, h_out["Z"],
                       [h_out[k] for k in w_keys], after=after)

    e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    done = None
    for i in range(args.e2e_steps):
        done = e2e_step(after=e0 if i == 0 else done)
    stream.wait_event(done)
    e1.record(stream)
    torch.cuda.synchronize()
    from test_sequence_modeling_b200 import sharding
    (te,) = sharding.max_over_ranks([e0.elapsed_time(e1)], dist, dev)
    e2e_value = world * cfg.head_tokens * args.e2e_steps / (te / 1e3)
    return {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": args.e2e_steps,
            "api": f"ttt_fwd_host (C ABI, host buffers; {args.e2e_chunks} batch chunks, copies overlapped) "
                   "through test_sequence_modeling_b200.host.HostForward"}


def finish(args, cfg, world, rank, value, ms_per_step, kernel_avg_ms, clock_info, launches, e2e,
           peaks, peak_kind, nbytes, nflops, dist):
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    scale = tensor_peak_scale(cfg, args.path)
    tensor_peak = peaks["bf16_tflops_sustained"] * scale
    t_tc = nflops / (tensor_peak * 1e12)
    if t_hbm >= t_tc:
        achieved = nbytes / (kernel_avg_ms / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"]}
    else:
        achieved = nflops / (kernel_avg_ms / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tensor_peak,
                "unit": "TFLOP/s", "frac": achieved / tensor_peak}
        if scale != 1.0:
            roof["peak_mix"] = (f"sustained bf16 x {scale:.3f}: tf32 products at the nominal "
                                f"{TF32_PER_BF16:.3f} of bf16, fp16 products at the bf16 rate")
            roof["frac_vs_bf16_peak"] = achieved / peaks["bf16_tflops_sustained"]
    traffic = committed_traffic(cfg.name)
    roof.update({"traffic": traffic, "peak_source": f"{peak_kind} (MEASURED_PEAKS.json)"
                 if peak_kind == "measured" else "fallback",
                 "algorithmic_bytes_per_launch": nbytes, "flops_per_launch": nflops,
                 "kernel_ms": kernel_avg_ms})

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": dtype_of(cfg, args.path),
        "data": "synthetic", "config": workload_config(cfg, args, world),
        "roofline": roof, "clocks": clock_info, "gpu_launches": int(launches), "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(cfg)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
