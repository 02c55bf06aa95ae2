"""Benchmark of the two-stage DDIM denoiser on B200.

One bench step = one full generation of the throughput workload: 100 DDIM steps,
B=16 prompts x 150 frames, CFG 2.0, cond and uncond batched (32 sequences of 151
tokens per network forward), bf16 tensor-core path, random-init weights and
seeded synthetic inputs.  Metric: clips/min (whole job), higher is better.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs one process per GPU (torchrun); every rank generates its own 16
prompts (weak scaling, no collective on the data path); time = max over ranks.
--impl reference times the plain CPU oracle on the host cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = dict(batch=16, frames=150, steps=100, cfg_scale=2.0)
# the one-prompt latency workload, for profiling runs only (--workload c3)
WORKLOAD_C3 = dict(batch=1, frames=180, steps=50, cfg_scale=2.0)
METRIC = "clips/min (150-frame, 100-step DDIM, B=16) + denoiser % of roofline"
UNIT = "clips/min"
L2_FLUSH_BYTES = 256 << 20
GEMM_FLOP_PER_TOKEN = 268_435_456      # 2 * 16 * (3d^2 + d^2 + 2 d F), per network forward


def workload_config(n_gpus):
    w = WORKLOAD
    return {"workload": f"{w['steps']}-step DDIM two-stage generation, B={w['batch']} prompts x {w['frames']} "
                        f"frames, CFG {w['cfg_scale']}, cond+uncond batched ({2 * w['batch']} x {w['frames'] + 1} "
                        f"tokens per forward)",
            "batch_per_gpu": w["batch"], "frames": w["frames"], "ddim_steps": w["steps"],
            "cfg_scale": w["cfg_scale"], "global_batch": w["batch"] * n_gpus,
            "parallelism": f"replicas x{n_gpus} (independent prompts per GPU)",
            "l2": "flushed between timed iterations (256 MiB write)"}


def rank_inputs(rank: int):
    """Seeded inputs of one rank: distinct prompts and noise per rank."""
    import synth
    w = WORKLOAD
    emb = synth.text_embeddings(w["batch"], seed=synth.SEED_TEXT + 1000 * rank)
    noise = synth.noise(w["batch"], w["frames"], seed=synth.SEED_NOISE + 1000 * rank)
    null = synth.null_embeddings(1)[0]
    lengths = np.full(w["batch"], w["frames"], np.int32)
    return emb, null, noise, lengths


def clips_per_min(n_gpus: int, steps: int, seconds: float) -> float:
    return n_gpus * WORKLOAD["batch"] * steps * 60.0 / seconds


def tokens_per_s(n_gpus: int, steps: int, seconds: float) -> float:
    w = WORKLOAD
    toks = 2 * 2 * w["batch"] * (w["frames"] + 1) * w["steps"]   # 2 nets x (cond, uncond)
    return n_gpus * toks * steps / seconds


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of per-rank timings (one all-reduce; identity at N=1)."""
    import torch
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"kimodo_bench_clocks_{os.getpid()}_{device_index}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9 and p[1].replace(".", "").isdigit():
                rows.append(p)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = max(float(r[2]) for r in rows)
        under = [s for s in sm if s > 0.3 * mx] or sm
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(under), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# --------------------------------------------------------------------------- roofline

def _measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


GEMM_SOURCES = ("gemm_tc.cu", "gemm_tc2.cu", "epilogue.cuh", "ptx.cuh", "launch.cuh")


def gemm_source_sha256():
    h = hashlib.sha256()
    for name in GEMM_SOURCES:
        h.update(open(os.path.join(ROOT, "transformer_denoiser_b200", "csrc", name), "rb").read())
    return h.hexdigest()


def _ncu_traffic():
    """DRAM bytes per tensor-core GEMM launch (mean over the captured launches of the
    throughput workload) from the committed ncu summary, or None if any GEMM source
    changed since those counters were taken."""
    path = os.path.join(ROOT, "profiles", "gemm_tc_traffic.txt")
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if "=" in line and not line.lstrip().startswith("#"):
            k, v = line.split("=", 1)
            vals[k.strip()] = v.strip()
    if vals.get("gemm_source_sha256") != gemm_source_sha256():
        return None
    try:
        return float(vals["dram_bytes_per_launch_c4"])
    except (KeyError, ValueError):
        return None


# Algorithmic work of one denoiser step (both networks).  FLOPs: the four projections
# per token per network forward.  Bytes: the bf16 layer weights, read once per network
# forward, plus the activations: 18,432 bf16 values per token and layer (one read or
# write of every GEMM operand and output, LayerNorm as its own pass), 36,864 bytes.
PROJ_FLOP_PER_TOKEN = 268435456
ACT_BYTES_PER_TOKEN_LAYER = 36864
WEIGHT_BYTES_PER_STEP = 2 * 16 * 8388608 * 2


def step_roofline(nseq, tokens_per_seq, ms_per_step):
    """Roofline of one DDIM step of the two-stage denoiser at nseq sequences (cond and
    uncond counted) of tokens_per_seq tokens: the slower of its FLOPs at the measured
    burst bf16 peak and its weight-plus-activation bytes at the measured HBM peak, and
    the fraction of it that ms_per_step achieves."""
    peaks, kind = _measured_peaks()
    tokens = nseq * tokens_per_seq
    flops = 2 * (tokens * PROJ_FLOP_PER_TOKEN + 16 * nseq * 4 * tokens_per_seq ** 2 * 1024)
    nbytes = WEIGHT_BYTES_PER_STEP + 2 * 16 * ACT_BYTES_PER_TOKEN_LAYER * tokens
    t_flop = flops / (float(peaks["bf16_tflops"]) * 1e12)
    t_byte = nbytes / (float(peaks["hbm_gbs"]) * 1e9)
    floor = max(t_flop, t_byte)
    t_weights = WEIGHT_BYTES_PER_STEP / (float(peaks["hbm_gbs"]) * 1e9)
    return {"bound": "tensor" if t_flop >= t_byte else "hbm", "floor_us": round(floor * 1e6, 2),
            "flop": flops, "bytes": nbytes, "achieved_us": round(ms_per_step * 1e3, 2),
            "frac": round(floor / (ms_per_step * 1e-3), 4),
            "weights_only_frac": round(t_weights / (ms_per_step * 1e-3), 4),
            "peaks": f"{kind} burst bf16 {peaks['bf16_tflops']} TFLOP/s, HBM {peaks['hbm_gbs']} GB/s"}


def roofline(prof):
    peaks, kind = _measured_peaks()
    g = prof["gemm_tc"]
    achieved = g["flops"] / (g["ms"] * 1e-3) / 1e12
    peak = float(peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]))
    return {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
            "frac": round(achieved / peak, 4), "traffic": _ncu_traffic(),
            "kernel": "tcgen05 bf16 GEMMs (gemm_tc2 CTA-pair kernel for the layer projections, gemm_tc for the rest)",
            "launches_per_step": g["launches"], "ms_per_step": round(g["ms"], 3),
            "peak_source": f"{kind} sustained bf16 GEMM (MEASURED_PEAKS.json)" if kind == "measured" else
                           "fallback sustained bf16 figure",
            "other_kernels_ms": {k: round(v["ms"], 3) for k, v in prof.items() if k != "gemm_tc" and v["launches"]}}


# --------------------------------------------------------------------------- CPU oracle leg

_ORACLE_PARAMS = None


def oracle_sample(target_s: float = 12.0):
    """Time the CPU oracle on a bounded sample of the workload: DDIM steps of one
    sequence (cond + uncond chains, 4 transformer forwards per step) until
    ~target_s of CPU work; returns (clips/min, seconds per sequence-step, desc, threads)."""
    import synth
    from oracle import kimodo_oracle as ko
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [os.cpu_count()])
    except Exception:
        threads = os.cpu_count()
    w = WORKLOAD
    global _ORACLE_PARAMS
    if _ORACLE_PARAMS is None:
        _ORACLE_PARAMS = ko.unpack_weights(synth.weight_blob())
    params = _ORACLE_PARAMS
    emb, null, noise, lengths = rank_inputs(0)
    ab = ko.alphabar_linear()
    ts = ko.ddim_timesteps(w["steps"])
    x = noise[0].astype(np.float64)
    n = 0
    t0 = time.perf_counter()
    while True:
        t, tp = ts[n % len(ts)]
        x, _ = ko.ddim_step(params, x, emb[0], null, w["frames"], t, tp, w["cfg_scale"], ab)
        n += 1
        el = time.perf_counter() - t0
        if el >= target_s or n >= len(ts):
            break
    per_step = el / n
    clips = 60.0 / (per_step * w["steps"])
    desc = (f"{n} DDIM steps of 1 sequence (150 frames, cond+uncond = 4 forwards/step), fp64 numpy, "
            f"extrapolated x100 steps per clip")
    return clips, per_step, desc, threads


# --------------------------------------------------------------------------- our arm

def secondary_workloads(model, dev, flush, reps=3):
    """The other two generation workloads, timed like the headline one (device inputs,
    L2 flushed, CUDA events, warm graph): 50-step latency of one 180-frame prompt, and a
    ragged batch of 64 prompts (lengths U{60..300} padded to 300 frames, CFG 2.5, garbage
    in the padding) on the packed token layout (lengths in host memory) and on the padded
    one (lengths in device memory)."""
    import torch
    import synth

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        best = None
        for _ in range(reps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        return best

    emb1 = torch.from_numpy(synth.text_embeddings(1)).to(dev)
    null = torch.zeros(4096, device=dev)
    n1 = torch.from_numpy(synth.noise(1, 180)).to(dev)
    l1 = torch.full((1,), 180, dtype=torch.int32, device=dev)
    c3_ms = timed(lambda: model.ddim_sample(emb1, null, n1, l1, 50, 2.0))
    B, T = 64, 300
    lengths = synth.lengths_uniform(B, 60, 300)
    emb = torch.from_numpy(synth.text_embeddings(B)).to(dev)
    noise = torch.from_numpy(synth.fill_padding(synth.noise(B, T), lengths)).to(dev)
    packed_ms = timed(lambda: model.ddim_sample(emb, null, noise, lengths, 50, 2.5))
    d_len = torch.from_numpy(lengths).to(dev)
    padded_ms = timed(lambda: model.ddim_sample(emb, null, noise, d_len, 50, 2.5))
    valid_tokens = 2 * 2 * int((lengths + 1).sum()) * 50
    return {"c3_latency": {"workload": "50-step DDIM, 1 prompt x 180 frames, CFG 2.0", "ms": round(c3_ms, 3),
                           "step_roofline": step_roofline(2, 181, c3_ms / 50)},
            "c5_ragged": {"workload": "50-step DDIM, 64 prompts, lengths U{60..300} padded to 300 frames, CFG 2.5",
                          "clips_per_min_packed": round(B * 60e3 / packed_ms, 2),
                          "clips_per_min_padded": round(B * 60e3 / padded_ms, 2),
                          "valid_tokens_per_s_packed": round(valid_tokens / (packed_ms / 1e3), 1),
                          "ms_packed": round(packed_ms, 2), "ms_padded": round(padded_ms, 2)}}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import synth
    import transformer_denoiser_b200 as kb

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    model = kb.Kimodo(synth.weight_blob(), kb.BF16, local_rank)
    emb, null, noise, lengths = rank_inputs(rank)
    d_emb = torch.from_numpy(emb).to(dev)
    d_null = torch.from_numpy(null).to(dev)
    d_noise = torch.from_numpy(noise).to(dev)
    d_len = torch.from_numpy(lengths).to(dev)
    d_out = torch.empty_like(d_noise)
    w = WORKLOAD
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    ddim_steps = args.ddim_steps or w["steps"]

    def step(out=d_out):
        model.ddim_sample(d_emb, d_null, d_noise, d_len, ddim_steps, w["cfg_scale"], out=out)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    model.sync_status()

    def barrier():
        if world > 1:
            dist.barrier()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            flush.zero_()
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = ev0.elapsed_time(ev1)
    launches_per_step = model.last_launch_count()
    model.sync_status()

    # end-to-end: HOST (pinned) inputs and output through the same C-ABI call
    h_emb = torch.from_numpy(emb).pin_memory()
    h_null = torch.from_numpy(null).pin_memory()
    h_noise = torch.from_numpy(noise).pin_memory()
    h_len = torch.from_numpy(lengths).pin_memory()
    h_out = torch.empty(h_noise.shape, dtype=torch.float32).pin_memory()
    model.ddim_sample(h_emb, h_null, h_noise, h_len, ddim_steps, w["cfg_scale"], out=h_out)
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        flush.zero_()
        model.ddim_sample(h_emb, h_null, h_noise, h_len, ddim_steps, w["cfg_scale"], out=h_out)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = e0.elapsed_time(e1)
    h2d = h_emb.numel() * 4 + h_null.numel() * 4 + h_noise.numel() * 4 + h_len.numel() * 4
    d2h = h_out.numel() * 4

    # per-kernel live timing of one generation (CUDA events around every launch)
    model.profile_enable(True)
    flush.zero_()
    step()
    prof = model.profile_read(6)
    model.profile_enable(False)
    model.sync_status()

    ms_max, e2e_max = max_over_ranks([ms, e2e_ms], dev, world)
    secondary = None
    if world == 1 and not args.no_secondary and not args.ddim_steps:
        secondary = secondary_workloads(model, dev, flush)
        model.sync_status()
    model.close()
    if rank != 0:
        return None
    sec = ms_max / 1e3
    line = {
        "metric": METRIC, "value": round(clips_per_min(world, args.steps, sec), 3), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_max / args.steps, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) embeddings and noise; "
                                                         "random-init N(0,0.02) weights)",
        "config": workload_config(world),
        "denoiser_tokens_per_s": round(tokens_per_s(world, args.steps, sec), 1),
        "e2e": {"value": round(clips_per_min(world, e2e_steps, e2e_max / 1e3), 3), "unit": UNIT,
                "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
        "gpu_launches": int(launches_per_step * args.steps),
        "roofline": roofline(prof),
        "clocks": clk.summary(),
    }
    if secondary is not None:
        line["secondary"] = secondary
    if args.ddim_steps or args.workload != "c4":
        line["note"] = (f"profiling case: workload {args.workload}, {ddim_steps} DDIM steps per generation; "
                        f"not a benchmark number")
    if world == 1 and not args.no_cpu_baseline:
        clips, per_step, desc, threads = oracle_sample()
        line["cpu_baseline"] = {"value": round(clips, 6), "unit": UNIT, "cores": threads, "kind": "oracle",
                                "sample": desc}
    return line


def run_reference(args, rank):
    if rank != 0:
        return None
    t0 = time.perf_counter()
    vals = []
    desc, threads = "", 1
    for _ in range(max(1, args.steps)):
        clips, per_step, desc, threads = oracle_sample(target_s=min(12.0, 120.0 / max(1, args.steps)))
        vals.append(clips)
    v = float(statistics.median(vals))
    return {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(60e3 * WORKLOAD["batch"] / v, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(1),
            "cpu_baseline": {"kind": "oracle", "cores": threads, "sample": desc, "value": round(v, 6)},
            "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 1)}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the c3 latency and c5 ragged-batch measurements")
    ap.add_argument("--ddim-steps", type=int, default=0,
                    help="profiling only: DDIM steps per generation (default: the workload's 100)")
    ap.add_argument("--workload", choices=["c4", "c3"], default="c4",
                    help="profiling only: c3 runs the one-prompt 180-frame workload in the timed loop")
    args = ap.parse_args(argv)
    if args.workload == "c3":
        WORKLOAD.update(WORKLOAD_C3)
        args.no_secondary = True
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        line = run_reference(args, rank)
    else:
        if world > 1:
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local_rank)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                    device_id=torch.device("cuda", local_rank))
        try:
            line = run_ours(args, rank, world, local_rank)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
