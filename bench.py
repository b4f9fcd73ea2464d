#!/usr/bin/env python
"""Benchmark of the B200 fused linear cross-entropy (FLCE): forward+backward
tokens/s at V=131072 and the fraction of the dense bf16 tensor-core peak.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl own|reference]

One step = one forward and one backward of the whole hot path over one batch
of the workload `v131k_zipf` (N=16384 tokens as [2, 8192], H=4096, V=131072,
Zipf(1.1) labels, 5% ignored, 'sum'), with inputs resident in HBM.  The inputs
(hidden 128 MiB + weight 1 GiB bf16) are larger than the 126 MB L2, so no L2
flush is needed between steps.  Multi-GPU runs are independent replicas (one
problem per GPU, no collective on the data path): weak scaling.

`--impl reference` times the float64 CPU oracle on a bounded token sample of
the same workload (the pages publish no GPU implementation to run).
"""
from __future__ import annotations

import argparse
import csv
import ctypes
import datetime
import hashlib
import io
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

import flce_inputs as fi  # noqa: E402

METRIC = "FLCE fwd+bwd tokens/s at V=131072; % of B200 dense bf16 tensor peak"
UNIT = "tokens/s"
WORKLOAD = "v131k_zipf"
KIND_NAMES = ["fwd_gemm_softmax_stats", "fwd_merge_loss", "bwd_dz_gemm", "bwd_dhidden_dweight_gemm",
              "unused", "helper", "fp32_simt"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["own", "reference"], default="own")
    p.add_argument("--workload", default=WORKLOAD)
    p.add_argument("--cpu-sample-tokens", type=int, default=1536)
    p.add_argument("--cpu-full", action="store_true",
                   help="time the float64 oracle's forward+backward on the whole workload "
                        "on the host cores (minutes; no GPU) and print one JSON line")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--option", action="append", default=[], metavar="NAME=VALUE",
                   help="set a library option (flce_set_option) for this run, e.g. "
                        "grad_tile_n=256; may be repeated")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_uuid):
        self.uuid = gpu_uuid
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                   "-lms", "100"]
            if self.uuid:
                cmd += ["-i", self.uuid]
            self.proc = subprocess.Popen(cmd, stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.tmp.read())) if len(r) >= 9]
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        top = max(sm)
        loaded = [s for s in sm if s >= 0.5 * top] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- cpu baseline
def oracle_step_sample(inp, w, tokens, W64):
    """One fwd+bwd of the oracle on the first `tokens` rows; returns seconds."""
    import oracle  # test infrastructure: the CPU baseline is the oracle itself
    h = inp.hidden[:tokens].astype(np.float64)
    y = inp.labels[:tokens]
    t = time.perf_counter()
    oracle.forward(h, W64, y, fi.IGNORE_INDEX, w.softcap, w.reduction)
    oracle.backward(h, W64, y, fi.IGNORE_INDEX, w.softcap, w.reduction)
    return time.perf_counter() - t


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 0) for d in threadpool_info() if d.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


CPU_FULL = os.path.join(ROOT, "profiles", "cpu_oracle_full_{}.json")


def cpu_full_record(workload):
    """The committed record of `bench.py --cpu-full` for this workload, if any."""
    path = CPU_FULL.format(workload)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        return json.load(f)


def cpu_baseline(inp, w, tokens):
    W64 = inp.weight.astype(np.float64)
    secs = oracle_step_sample(inp, w, tokens, W64)
    out = {"value": tokens / secs, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
           "sample": f"float64 numpy oracle fwd+bwd on the first {tokens} tokens of "
                     f"{w.name} (H={w.H}, V={w.V}), {secs:.2f} s",
           "value_is": "the sampled rate, measured in this run"}
    full = cpu_full_record(w.name)
    if full is not None:
        out["full_problem"] = {k: full[k] for k in ("wall_s", "tokens_per_s", "cores", "tokens",
                                                    "command") if k in full}
        out["full_problem"]["measured"] = "separately, by the command given (not in this run)"
    return out


def run_cpu_full(args):
    """--cpu-full: the oracle's forward and backward over the whole workload, timed
    once on the host cores (the float64 baseline at full size)."""
    import oracle  # test infrastructure: the CPU baseline is the oracle itself
    w = fi.WORKLOADS[args.workload]
    inp = fi.make_inputs(w)
    h = inp.hidden.astype(np.float64)
    W64 = inp.weight.astype(np.float64)
    t0 = time.perf_counter()
    f = oracle.forward(h, W64, inp.labels, fi.IGNORE_INDEX, w.softcap, w.reduction)
    t1 = time.perf_counter()
    oracle.backward(h, W64, inp.labels, fi.IGNORE_INDEX, w.softcap, w.reduction)
    t2 = time.perf_counter()
    line = {"kind": "oracle", "workload": w.name, "tokens": w.N, "hidden": w.H, "vocab": w.V,
            "forward_s": t1 - t0, "backward_s": t2 - t1, "wall_s": t2 - t0,
            "tokens_per_s": w.N / (t2 - t0), "cores": blas_threads(),
            "cpu_count": os.cpu_count(), "loss": f["loss"],
            "command": f"python bench.py --cpu-full --workload {w.name}"}
    print(json.dumps(line), flush=True)


def run_reference(args, rank):
    """--impl reference: the oracle on the host cores, rank 0 only."""
    if rank != 0:
        return
    w = fi.WORKLOADS[args.workload]
    inp = fi.make_inputs(w)
    W64 = inp.weight.astype(np.float64)
    tokens = max(8, min(args.cpu_sample_tokens // 4, 64))
    for _ in range(args.warmup):
        oracle_step_sample(inp, w, tokens, W64)
    secs = [oracle_step_sample(inp, w, tokens, W64) for _ in range(args.steps)]
    total = sum(secs)
    value = tokens * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": w.name, "tokens": w.N, "hidden": w.H, "vocab": w.V,
                   "sample_tokens_per_step": tokens, "labels": w.labels,
                   "reduction": w.reduction},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"float64 oracle fwd+bwd on {tokens} tokens per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest value of `x` over all ranks (the slowest rank's time)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank_step: int, steps: int, ms: float) -> float:
    """Units all ranks processed per second, timed by the slowest rank."""
    return world * units_per_rank_step * steps / (ms / 1e3)


# ---------------------------------------------------------------- own arm
def source_digest():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lm_head_linear_tmem_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def dram_traffic(kind_name):
    """Per-launch DRAM bytes from the committed ncu summary, if it matches the
    current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("source_digest") != source_digest():
        return None
    ent = d.get("kernels", {}).get(kind_name)
    return None if ent is None else ent.get("bytes_per_launch_full_size")


def run_own(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import lm_head_linear_tmem_b200 as flce
    from lm_head_linear_tmem_b200 import _native

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    lib = _native.load()
    for kv in args.option:
        name, val = kv.split("=")
        _native.set_option(name, int(val))
    options = {name: _native.get_option(name) for name in _native.OPTIONS}
    w = fi.WORKLOADS[args.workload]
    inp = fi.make_inputs(w)
    N, H, V = w.N, w.H, w.V

    def bf16(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    h_host = bf16(inp.hidden_bits).pin_memory()
    y_host = torch.from_numpy(inp.labels).pin_memory()
    h = h_host.to(dev)
    W = bf16(inp.weight_bits).to(dev)
    y = y_host.to(dev)
    ws = flce.alloc_workspace(N, H, V, torch.bfloat16, dev)
    lse = torch.empty(N, dtype=torch.float32, device=dev)
    dh = torch.empty(N, H, dtype=torch.float32, device=dev)
    dw = torch.empty(V, H, dtype=torch.float32, device=dev)

    def step(hb=None, yb=None):
        hb = h if hb is None else hb
        yb = y if yb is None else yb
        f = flce.forward(hb, W, yb, fi.IGNORE_INDEX, w.softcap, w.reduction, workspace=ws,
                         lse=lse)
        flce.backward(hb, W, yb, lse, ignore_index=fi.IGNORE_INDEX, softcap=w.softcap,
                      reduction=w.reduction, workspace=ws, d_hidden=dh, d_weight=dw)
        return f

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    _native.check(lib.flce_get_status(ctypes.c_void_p(ws.data_ptr()),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)),
                  "warm-up status")
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
        if uuid and not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
    except Exception:
        uuid = None

    # ---- device-resident timing (the headline value): K steps, no per-kernel events
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(uuid)
    sampler.start()
    st = torch.cuda.current_stream()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    launches0 = lib.flce_launch_count()
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    launches = lib.flce_launch_count() - launches0
    clocks = sampler.stop()
    ms = e0.elapsed_time(e1)
    barrier()
    ms = max_over_ranks(ms, world, dev)
    ms_step = ms / args.steps
    value = whole_job_rate(world, N, args.steps, ms)

    # ---- per-kernel accounting: the same K steps again, with a CUDA event pair
    # recorded by the library around every kernel it launches (on this stream)
    lib.flce_profile_enable(1)
    for k in range(len(KIND_NAMES)):  # drop anything recorded before
        lib.flce_profile_read(k, ctypes.byref(ctypes.c_double()), ctypes.byref(ctypes.c_int64()))
    torch.cuda.synchronize()
    e0.record(st)
    for _ in range(args.steps):
        step()
    e1.record(st)
    torch.cuda.synchronize()
    lib.flce_profile_enable(0)
    ms_prof = e0.elapsed_time(e1)
    kinds = {}
    for k, name in enumerate(KIND_NAMES):
        t = ctypes.c_double()
        n = ctypes.c_int64()
        lib.flce_profile_read(k, ctypes.byref(t), ctypes.byref(n))
        if n.value:
            kinds[name] = {"ms_total": t.value, "launches": n.value,
                           "share": t.value / ms_prof if ms_prof > 0 else None}

    # ---- end to end through the API with host buffers.  Every step copies its
    # inputs (hidden, labels) from pinned host memory and reads its loss and
    # token count back, all inside the timed region.  The copy of step i+1 runs
    # on a copy stream into the second of two device input buffers while step
    # i computes (a data loader's double buffering); the first copy is exposed.
    e2e_steps = args.e2e_steps or max(3, args.steps // 2)
    loss_host = torch.empty((), dtype=torch.float32).pin_memory()
    ntok_host = torch.empty((), dtype=torch.int64).pin_memory()
    h_dev = [h, torch.empty_like(h)]
    y_dev = [y, torch.empty_like(y)]
    cp = torch.cuda.Stream(device=dev)
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    barrier()
    torch.cuda.synchronize()
    e0.record(st)
    cp.wait_event(e0)
    for i in range(e2e_steps + 1):
        if i < e2e_steps:  # inputs of step i
            b = i % 2
            with torch.cuda.stream(cp):
                if i >= 2:
                    cp.wait_event(freed[b])
                h_dev[b].copy_(h_host, non_blocking=True)
                y_dev[b].copy_(y_host, non_blocking=True)
                copied[b].record(cp)
        if i >= 1:  # compute step i-1
            b = (i - 1) % 2
            st.wait_event(copied[b])
            f = step(h_dev[b], y_dev[b])
            loss_host.copy_(f.loss, non_blocking=True)
            ntok_host.copy_(f.num_tokens, non_blocking=True)
            freed[b].record(st)
    e1.record(st)
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1)
    barrier()
    ms_e2e = max_over_ranks(ms_e2e, world, dev)
    e2e_value = whole_job_rate(world, N, e2e_steps, ms_e2e)
    h2d = h_host.numel() * 2 + y_host.numel() * 8
    d2h = 4 + 8

    if rank != 0:
        return None

    peaks, peak_src = load_peaks()
    flops_step = w.flops_per_step
    # Work the kernels execute: the forward and backward GEMMs cover the
    # non-ignored rows only (rows with ignore_index take no part in the loss and
    # have exactly zero gradient; they are compacted away) unless the
    # fwd_compact / bwd_compact options are off.  The credited work counts every
    # row: 8*N*H*V.
    n_valid = int((inp.labels != fi.IGNORE_INDEX).sum())
    n_bwd = n_valid if _native.get_option("bwd_compact") != 0 else N
    n_fwd = n_valid if _native.get_option("fwd_compact") != 0 else N
    executed_step = 2.0 * n_fwd * H * V + 6.0 * n_bwd * H * V
    # the dominant kernel (largest device time) and its roofline, from the FLOP
    # each kernel kind executes per step (summed over its launches)
    credited = {"fwd_gemm_softmax_stats": 2.0 * n_fwd * H * V,
                "bwd_dz_gemm": 2.0 * n_bwd * H * V,
                "bwd_dhidden_dweight_gemm": 4.0 * n_bwd * H * V}
    dom = max(kinds, key=lambda k: kinds[k]["ms_total"]) if kinds else None
    roofline = None
    if dom in credited:
        per_launch_flops = credited[dom] * args.steps / kinds[dom]["launches"]
        avg_ms = kinds[dom]["ms_total"] / kinds[dom]["launches"]
        achieved = per_launch_flops / (avg_ms / 1e3) / 1e12
        peak = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
        roofline = {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                    "unit": "TFLOP/s", "frac": achieved / peak,
                    "peak_source": f"{peak_src} bf16_tflops_sustained",
                    "traffic": dram_traffic(dom),
                    "per_launch_flops": per_launch_flops, "avg_launch_ms": avg_ms}
    # every tensor-core kernel kind against the same peak (the dominant one is `roofline`)
    gemm_roofline = {}
    for kind, fl in credited.items():
        if kind in kinds:
            avg = kinds[kind]["ms_total"] / kinds[kind]["launches"]
            ach = fl * args.steps / kinds[kind]["launches"] / (avg / 1e3) / 1e12
            gemm_roofline[kind] = {"achieved_tflops": ach, "avg_launch_ms": avg,
                                   "frac_of_sustained": ach / float(peaks.get(
                                       "bf16_tflops_sustained",
                                       FALLBACK_PEAKS["bf16_tflops_sustained"])),
                                   "dram_bytes_per_launch": dram_traffic(kind)}
    tflops = flops_step / (ms_step / 1e3) / 1e12
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sust = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))

    cpu = None
    if not args.no_cpu_baseline and world == 1:
        cpu = cpu_baseline(inp, w, args.cpu_sample_tokens)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "tokens": N, "batch_shape": list(w.batch_shape),
                   "hidden": H, "vocab": V, "labels": w.labels, "ignored": w.ignore_count,
                   "softcap": w.softcap, "reduction": w.reduction,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "inputs larger than L2 (weight 1 GiB bf16), no flush"},
        "tensor_peak_pct": {"credited_tflops": tflops, "flops_per_step": flops_step,
                            "frac_of_burst": tflops / burst, "frac_of_sustained": tflops / sust,
                            "executed_flops_per_step": executed_step,
                            "executed_tflops": executed_step / (ms_step / 1e3) / 1e12,
                            "executed_frac_of_sustained":
                                executed_step / (ms_step / 1e3) / 1e12 / sust,
                            "forward_rows": n_fwd, "backward_rows": n_bwd, "tokens": N,
                            "peak_source": peak_src},
        "roofline": roofline,
        "gemm_roofline": gemm_roofline,
        "kernels": kinds,
        "kernels_region_ms_per_step": ms_prof / args.steps,
        "library_options": options,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "copies": "pinned H2D of every step's inputs on a copy stream, double-buffered "
                          "(step i+1's copy overlaps step i); loss and count D2H every step"},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)
    return line


def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.cpu_full:
        if rank == 0:
            run_cpu_full(args)
        return
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        run_own(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
