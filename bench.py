#!/usr/bin/env python
"""Training-step throughput of the nanochat decoder (forward + backward: loss
and every weight gradient) through the C ABI.  Default workload d20:
depth 20 (C=1280, 10 query heads of 128 + 1 shared KV head, MLP 5120),
vocab 65,536, B=16 rows of T=2048 Zipf(1.1) tokens per GPU, bf16 storage with
fp32 accumulation, random-init weights of that architecture.  --config picks
one of the five workloads (d4 fp32, d12, d20, d24, d32).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config d20]

The timed steps run with the library's per-launch accounting off; a second,
separate pass of the same steps with it on gives the per-kernel times, rates
and the roofline of the dominant kernel.

N > 1 runs one process per GPU under torch.distributed.run; each rank runs its
own shard of B rows (data parallel, weak scaling) and the timing is the
maximum over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "train tokens/sec (fwd+bwd) at d20 on 1 B200; MFU vs bf16 dense peak"
DEFAULT_WORKLOAD = "d20"
FULL_BLOCK_WINDOW = 1024  # the short window of the pages' "SSSL" layers


def metric_for(name: str, full_block: bool = False) -> str:
    m = METRIC if name == DEFAULT_WORKLOAD else METRIC.replace("at d20", f"at {name}")
    return m.replace(" on 1 B200", " (full reference block) on 1 B200") if full_block else m


def host_cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


# algorithmic flops per token: 6 N_mm + 6 T C L (causal attention), N_mm = every
# matmul weight including the unembedding (the embedding gather has no flops)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def model_flops_per_token(depth: int, C: int, V: int, T: int, windows=None) -> float:
    """windows: per-layer sliding window (0 or None: causal).  A windowed
    layer's query sees w - w^2/(2T) keys on average (T/2 when causal)."""
    n_mm = depth * (2 * C * C + 2 * 128 * C + 8 * C * C) + V * C
    if not windows:
        return 6.0 * n_mm + 6.0 * T * C * depth
    keys = sum((w - w * w / (2.0 * T)) if (w and w < T) else T / 2.0 for w in windows)
    return 6.0 * n_mm + 12.0 * C * keys


def model_flops_per_token_noncausal(depth: int, C: int, V: int, T: int) -> float:
    """The same count with attention taken dense (every query against all T keys)."""
    return model_flops_per_token(depth, C, V, T) + 6.0 * T * C * depth


def mufu_fraction(ms_per_step: float, tokens: int, vocab: int, num_sms: int, sm_mhz: float,
                  ops_per_logit: float = 2.0) -> float:
    """Fraction of the MUFU (special-function) roofline the CE kernel reaches:
    ops_per_logit operations per logit (tanh, one exponential) against 16 per
    clock per SM at the clock sampled during the run."""
    ops_per_s = ops_per_logit * vocab * tokens / (ms_per_step / 1000.0)
    return ops_per_s / (16.0 * num_sms * sm_mhz * 1e6)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel: str):
    """Per-launch DRAM traffic of `kernel` from the committed ncu summary, if it
    was taken on the current source of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_sha = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    m_b = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    m_src = re.search(r"source_file:\s*(\S+)", text)
    if not (m_sha and m_b and m_src):
        return None
    src = os.path.join(ROOT, m_src.group(1))
    if not os.path.exists(src):
        return None
    if hashlib.sha256(open(src, "rb").read()).hexdigest() != m_sha.group(1):
        return None
    return float(m_b.group(1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def start(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if not self.proc:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.flush()
        self.out.seek(0)
        rows = [r.split(",") for r in self.out.read().strip().splitlines() if r.strip()]
        os.unlink(self.out.name)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx),
                "samples": len(sm), "reasons": sorted(reasons)}


def cpu_oracle_sample(W64, depth, V, T_sample, seed):
    """Time the fp64 oracle on one row of T_sample tokens of the workload."""
    import numpy as np

    import oracle
    import synth
    tok, tgt = synth.token_rows(seed, 1, T_sample, V, "zipf")
    t0 = time.perf_counter()
    oracle.loss_and_grads(W64, tok, tgt, depth)
    dt = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    return T_sample / dt, dt, cores


def dist_setup(gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != gpus:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def reduce_max(x: float, world: int, device: str = "cuda") -> float:
    """Maximum of x over the ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s token rows: every rank draws its own B rows."""
    return seed + 1000 * rank


def job_rate(tokens_per_rank: int, ms_max: float, world: int) -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    return world * tokens_per_rank / (ms_max / 1000.0)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def run_reference(args):
    """The fp64 oracle on the host cores, each step one bounded sample of the
    workload: one row of T=128 tokens through the full d20 model."""
    import numpy as np

    import oracle
    import synth
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[args.config]
    lay = oracle.param_layout(wl.depth, wl.vocab)
    _, W64 = synth.make_weights(lay, wl.seed, wl.dtype)
    T_sample = 128
    times = []
    cores = None
    for i in range(args.warmup + args.steps):
        tps, dt, cores = cpu_oracle_sample(W64, wl.depth, wl.vocab, T_sample, wl.seed + 100 + i)
        if i >= args.warmup:
            times.append(dt)
    ms = 1000.0 * sum(times) / len(times)
    value = T_sample / (ms / 1000.0)
    D = oracle.dims(wl.depth, wl.vocab)
    line = {
        "impl": "reference", "metric": metric_for(wl.name), "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(wl, args.gpus, sample=f"B=1, T={T_sample}"),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "cpu": host_cpu_model(),
                         "kind": "oracle",
                         "sample": f"one row of {T_sample} tokens through the full {wl.name} model per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "model_flops_per_token": model_flops_per_token(wl.depth, D["C"], wl.vocab, T_sample),
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(wl, n_gpus, sample=None, full_block=False):
    d = {
        "workload": (f"{wl.name}: depth {wl.depth}, width {64 * wl.depth}, "
                     f"{64 * wl.depth // 128} query heads x128 + 1 shared KV head, "
                     f"MLP {256 * wl.depth}, vocab {wl.vocab}, B={wl.B} x T={wl.T} per GPU, "
                     f"{wl.tokens} tokens, {wl.dtype}"),
        "global_batch": wl.B * n_gpus, "seq_len": wl.T,
        "parallelism": (f"dp{n_gpus}: NCCL all-reduce (mean) of the gradient buckets, overlapped with the backward"
                        if n_gpus > 1 else "dp1"),
        "l2": "inputs larger than L2 (activations and logits ~20 GB per GPU)",
    }
    if sample:
        d["sample"] = sample
    if full_block:
        d["block"] = (f"full reference block: SSSL sliding windows of {FULL_BLOCK_WINDOW} tokens (last layer "
                      "full), gated value embeddings on even layers, resid/x0 scalars (1.0 / 0.1)")
    return d


def run_ours(args):
    import numpy as np
    import torch

    import synth
    from decoder_only_transformer_nanochat_b200 import build as nc_build

    world, rank, local = dist_setup(args.gpus)
    if rank == 0:
        nc_build.build()
    barrier(world)
    import decoder_only_transformer_nanochat_b200 as nc
    from decoder_only_transformer_nanochat_b200 import Model

    wl = synth.WORKLOADS[args.config]
    if args.full_block:
        # the pages' full block: SSSL windows of 1,024, value embeddings, residual scalars
        model = Model(wl.depth, vocab=wl.vocab, seq=wl.seq, dtype=wl.dtype, window=FULL_BLOCK_WINDOW,
                      value_embeds=True, resid_scalars=True)
        n_ve = (wl.depth + 1) // 2
        values = synth.full_block_values(wl.depth, n_ve)
    else:
        model = Model(wl.depth, vocab=wl.vocab, seq=wl.seq, dtype=wl.dtype)
        values = None
    lay = [(n, r, c) for n, _, r, c in model.layout]
    flat, W64 = synth.make_weights(lay, wl.seed, wl.dtype, values=values)
    if args.full_block:
        W64 = None  # the CPU baseline times the baseline oracle only
    if wl.dtype == "bf16":
        weights = torch.from_numpy(flat.view(np.int16)).cuda().view(torch.bfloat16)
    else:
        weights = torch.from_numpy(flat).cuda()
    del flat
    if not (rank == 0 and world == 1 and not args.no_cpu_baseline):
        W64 = None
    tok, tgt = synth.token_rows(shard_seed(wl.seed, rank), wl.B, wl.T, wl.vocab, wl.tokens)
    tokens = torch.from_numpy(tok).cuda()
    targets = torch.from_numpy(tgt).cuda()
    grads = torch.empty(model.n_params, dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    model.workspace(wl.B, wl.T)
    stream = torch.cuda.current_stream()

    if world > 1:
        # data parallel: the ranks' gradients are averaged by NCCL all-reduces of
        # the gradient buckets, each started as soon as the backward finishes it
        from decoder_only_transformer_nanochat_b200.dp import DataParallel
        dpar = DataParallel(model)

        def step():
            dpar.step(weights, tokens, targets, grads, loss)
    else:
        def step():
            model.fwd_bwd(weights, tokens, targets, grads=grads, loss=loss)

    for _ in range(args.warmup):
        step()
    rc = model.sync_status(600000)
    if rc != 0:
        raise RuntimeError(f"device status after warm-up: {nc.nc_strerror(rc)}")
    nc.nc_profile_read(model.handle)  # drop warm-up accounting

    # ---------------- device-timed region (no per-launch accounting) ----------------
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    sampler = ClockSampler(gpu_index)
    nc.nc_profile(model.handle, 0)
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms_local = t_start.elapsed_time(t_end) / args.steps
    status = model.sync_status(60000)
    if status != 0:
        raise RuntimeError(f"device status after the timed steps: {nc.nc_strerror(status)}")
    nc.nc_profile_read(model.handle)  # launch counts of the timed steps: not used
    ms = reduce_max(ms_local, world)
    tokens_per_step = wl.B * wl.T
    value = job_rate(tokens_per_step, ms, world)

    # ---------------- accounting pass: the same steps, every launch between two events ----------------
    nc.nc_profile(model.handle, 1)
    torch.cuda.synchronize()
    for _ in range(args.steps):
        step()
    torch.cuda.synchronize()
    nc.nc_profile(model.handle, 0)
    rc, stats = nc.nc_profile_read(model.handle)
    status = model.sync_status(60000)
    if status != 0:
        raise RuntimeError(f"device status after the accounting steps: {nc.nc_strerror(status)}")

    # ---------------- end to end: host buffers through the public API ----------------
    tok_h = torch.from_numpy(tok).pin_memory()
    tgt_h = torch.from_numpy(tgt).pin_memory()
    loss_h = torch.empty(1, dtype=torch.float32).pin_memory()
    tok_d = torch.empty_like(tokens)
    tgt_d = torch.empty_like(targets)

    def e2e_step():
        tok_d.copy_(tok_h, non_blocking=True)
        tgt_d.copy_(tgt_h, non_blocking=True)
        if world > 1:
            dpar.step(weights, tok_d, tgt_d, grads, loss)
        else:
            model.fwd_bwd(weights, tok_d, tgt_d, grads=grads, loss=loss)
        loss_h.copy_(loss, non_blocking=True)

    e2e_step()
    barrier(world)
    torch.cuda.synchronize()
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e_end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = reduce_max(e_start.elapsed_time(e_end) / args.steps, world)
    e2e_value = job_rate(tokens_per_step, e2e_ms, world)
    loss_val = float(loss_h.item())

    if world > 1:
        dpar.close()
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    # ---------------- roofline of the dominant kernel ----------------
    peaks, peak_src = load_peaks()
    by = {s["name"]: s for s in stats}
    dominant = max(stats, key=lambda s: s["ms"])
    kernels = {}
    for s in stats:
        per = s["ms"] / s["launches"] if s["launches"] else 0.0
        k = {"launches_per_step": s["launches"] / args.steps, "ms_per_step": s["ms"] / args.steps,
             "avg_launch_us": 1000.0 * per}
        if s["flops"] > 0 and s["ms"] > 0:
            k["tflops"] = s["flops"] / (s["ms"] / 1000.0) / 1e12
        if s["bytes"] > 0 and s["ms"] > 0:
            k["gbs"] = s["bytes"] / (s["ms"] / 1000.0) / 1e9
            k["hbm_frac"] = k["gbs"] / peaks["hbm_gbs"]
        kernels[s["name"]] = k
    if "ce_fused" in kernels and clocks and clocks.get("sm_mhz"):
        try:  # an optional figure: it must never cost the bench line
            kernels["ce_fused"]["mufu_frac"] = mufu_fraction(
                kernels["ce_fused"]["ms_per_step"], tokens_per_step, wl.vocab,
                torch.cuda.get_device_properties(local).multi_processor_count, clocks["sm_mhz"])
        except Exception as exc:  # noqa: BLE001
            kernels["ce_fused"]["mufu_frac_error"] = repr(exc)
    if dominant["flops"] > 0:
        achieved = dominant["flops"] / (dominant["ms"] / 1000.0) / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"kernel": dominant["name"], "bound": "tensor", "achieved": achieved, "peak": peak,
                "unit": "TFLOP/s", "frac": achieved / peak,
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside a long step)"}
    else:
        achieved = dominant["bytes"] / (dominant["ms"] / 1000.0) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": dominant["name"], "bound": "hbm", "achieved": achieved, "peak": peak,
                "unit": "GB/s", "frac": achieved / peak, "peak_source": f"{peak_src} hbm_gbs"}
    tr = traffic_record(dominant["name"])
    roof["traffic"] = tr
    roof["algorithmic_per_launch"] = (dominant["flops"] or dominant["bytes"]) / dominant["launches"]

    D = model.dims
    fpt = model_flops_per_token(wl.depth, D["width"], wl.vocab, wl.T, model.windows)
    fpt_nc = model_flops_per_token_noncausal(wl.depth, D["width"], wl.vocab, wl.T)
    model_tflops = value * fpt / 1e12
    launches = sum(s["launches"] for s in stats)  # the accounting pass ran the same steps

    line = {
        "metric": metric_for(wl.name, args.full_block), "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": wl.dtype,
        "data": "synthetic (seeded Zipf tokens, random-init weights)",
        "config": config_dict(wl, world, full_block=args.full_block),
        "mfu": model_tflops / (world * peaks["bf16_tflops"]),
        "mfu_sustained_peak": model_tflops / (world * peaks["bf16_tflops_sustained"]),
        "model_tflops": model_tflops, "model_flops_per_token": fpt,
        "model_flops_per_token_noncausal": fpt_nc,
        "mfu_noncausal": value * fpt_nc / 1e12 / (world * peaks["bf16_tflops"]),
        "peaks": {"source": peak_src, "bf16_tflops": peaks["bf16_tflops"],
                  "bf16_tflops_sustained": peaks["bf16_tflops_sustained"], "hbm_gbs": peaks["hbm_gbs"]},
        "roofline": roof,
        "kernels": kernels,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(tok.nbytes + tgt.nbytes), "d2h_bytes_per_step": 4},
        "gpu_launches": launches,
        "kernels_timing": "separate pass of the same steps with per-launch events (the timed steps run without them)",
        "clocks": clocks,
        "loss": loss_val,
    }
    if world == 1 and not args.no_cpu_baseline and W64 is not None:
        T_sample = 128
        tps, dt, cores = cpu_oracle_sample(W64, wl.depth, wl.vocab, T_sample, wl.seed + 7)
        line["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": cores, "cpu": host_cpu_model(),
                                "kind": "oracle",
                                "sample": f"one row of {T_sample} tokens through the full {wl.name} "
                                          f"model ({dt:.1f} s)"}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--config", default=DEFAULT_WORKLOAD, choices=["d4", "d12", "d20", "d24", "d32"])
    ap.add_argument("--full-block", action="store_true",
                    help="the full reference block (SSSL windows, value embeddings, residual scalars)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
