#!/usr/bin/env python
"""Benchmark of the Longformer banded + global attention hot path on B200.

One step = one pass of the whole path over one batch of the fp16
Longformer-large workload (B=1, H=16, L=4096, w=256, 64 prefix globals, last
300 positions padded): the global-index partition and the fused attention,
one kernel launch (lf_attention_forward_idx: the attention kernel's epilogue
warps compute the partition while the first scores are computed).  Inputs
are synthetic and seeded.  The workload's HBM
footprint (~50 MB) fits in L2, so L2 is flushed (a 2 x L2 write) before
every timed step, outside the step's event pair.  The dominant kernel (the
attention kernel, or the whole layer for workload 5) is also timed alone,
with the same flush, for the roofline figures.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                       [--workload N]
Under torchrun each rank runs its own replica of the workload (weak scaling,
no collective on the data path); timings are the max over ranks.
--workload selects another of the synthetic configurations (1: fp32
attention, 3: bf16 batched, 4: fp16 L=16384, 5: one fp16 encoder layer with
its projections, LayerNorms and FFN, 6: workload 2 with its global tokens at
random positions, through the entry point for global tokens anywhere, whose
one call runs the partition fused with the gather of the global rows, and
the attention kernel); 2 is the default and the headline.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_attention_banded_b200 import inputs, metrics  # noqa: E402

METRIC = "Longformer attention tokens/s & TFLOP/s (fp16 L=4096 w=256) and % tensor peak"
WORKLOAD_ID = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", type=int, default=WORKLOAD_ID, choices=[1, 2, 3, 4, 5, 6])
    ap.add_argument("--any-globals", action="store_true",
                    help="workload 5 only: its 64 global tokens at random positions, through the entry points for "
                         "global tokens anywhere")
    ap.add_argument("--layers", type=int, default=1,
                    help="workload 5 only: time an encoder of this many layers (lf_encoder_forward), each with "
                         "its own seeded weights")
    ap.add_argument("--ffn-path", default="auto", choices=["auto", "unfused", "fused"],
                    help="workload 5 only: the FFN path of the layer (two GEMMs, or the fused kernel that keeps "
                         "the intermediate on chip; auto picks the faster for the shape)")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def max_over_ranks(values, device="cpu"):
    """Element-wise max of `values` over all ranks of the default process
    group (every rank calls it with the same length); the values themselves
    on a single rank."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    x = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(x, op=dist.ReduceOp.MAX)
    return x.tolist()


def percentiles(values):
    """p10, median and p90 of a list of timings (nearest rank on the sorted
    list)."""
    s = sorted(values)
    n = len(s)
    if n == 0:
        return {"p10": None, "median": None, "p90": None}

    def q(p):
        return s[min(n - 1, max(0, int(round(p * (n - 1)))))]
    return {"p10": q(0.1), "median": q(0.5), "p90": q(0.9)}


def job_throughput(world: int, units_per_rank: float, steps: int, max_total_ms: float) -> float:
    """Whole-job units/s: every rank processed units_per_rank per step, the
    job took the slowest rank's time."""
    return world * units_per_rank * steps / (max_total_ms * 1e-3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons while running."""
    FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            props = torch.cuda.get_device_properties(device_index)
            self.bus = "%08X:%02X:%02X.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
        except Exception:
            self.bus = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader",
                                          "-lms", "100", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                if self.bus and parts[0].upper()[-len(self.bus):] != self.bus and \
                        not parts[0].upper().endswith(self.bus[4:]):
                    continue
                rows.append(parts)
        os.remove(self.path)
        if not rows:
            return None
        sm = [float(re.sub(r"[^0-9.]", "", r[1]) or 0) for r in rows]
        mx = [float(re.sub(r"[^0-9.]", "", r[2]) or 0) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[k] for r in rows for k in range(4) if r[5 + k].lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- our arm

def traffic_from_profile(kernel_src_hash: str):
    """DRAM bytes per attention launch from the committed ncu counters
    (profiles/attention_tc_workload2.traffic.json), or None when they were
    taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "attention_tc_workload2.traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256") != kernel_src_hash:
        return None
    return float(d["dram_bytes_per_launch"])


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("lf_attn_tc.cu", "lf_pair_math.cuh", "lf_partition.cuh", "sm100.cuh"):
        with open(os.path.join(ROOT, "sparse_attention_banded_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def cpu_baseline(wl, t, lm, gm, budget_s=10.0):
    import numpy as np
    import oracle
    arrs = [t[n].double().numpy() for n in inputs.NAMES]
    lmn, gmn = lm.numpy(), gm.numpy()
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.attention(*arrs, lmn, gmn, wl.w, any_pos=wl.scattered)
        passes += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    el = time.perf_counter() - t0
    return {"value": wl.B * wl.L * passes / el, "unit": "tokens/s", "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": "%d full pass(es) of the workload (%d query rows each), float64 C oracle" %
                      (passes, wl.B * wl.H * wl.L)}


def run_ours(args):
    from sparse_attention_banded_b200 import lf
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    layer = args.workload == 5
    anyg = args.workload == 6  # global tokens at any position: one call = partition + gather + attention
    n_layers = 1
    any_layer = layer and args.any_globals
    if layer:
        wl, x_cpu, wts_cpu, lm_cpu, gm_cpu = inputs.layer_inputs(5)
        if any_layer:
            lm_cpu, gm_cpu = inputs.masks_scattered(wl.B, wl.L, wl.g, wl.pad, seed=1105)
        x = x_cpu.to(dev)
        wts = {n: v.to(dev) for n, v in wts_cpu.items()}
        ffn = wts["W_1"].shape[0]
        n_layers = max(1, args.layers)
        # further layers: the same architecture, weights ~ N(0, 0.02) drawn on the device from a seeded generator
        gen = torch.Generator(device=dev).manual_seed(5000)
        stack = [wts] + [{n: ((torch.randn(v.shape, generator=gen, device=dev) * 0.02).to(v.dtype)
                               if n.startswith("W_") else v.clone()) for n, v in wts.items()}
                         for _ in range(n_layers - 1)]
        lf.lf_set_ffn_path(args.ffn_path)
        ws_fn = lf.lf_encoder_any_globals_workspace_bytes if any_layer else lf.lf_encoder_workspace_bytes
        ws = torch.empty(max(256, ws_fn(n_layers, wl.B, wl.H, wl.L, wl.w, ffn, x.dtype)),
                         dtype=torch.uint8, device=dev)
        args_in = [x]
        t_cpu = None
    else:
        wl, t_cpu, lm_cpu, gm_cpu = inputs.workload_inputs(args.workload)
        t = {n: t_cpu[n].to(dev) for n in inputs.NAMES}
        args_in = [t[n] for n in inputs.NAMES]
    lm, gm = lm_cpu.to(dev), gm_cpu.to(dev)
    out = torch.empty(wl.B, wl.L, wl.H * 64, dtype=args_in[0].dtype, device=dev)
    gidx = torch.empty(wl.B, wl.L, dtype=torch.int32, device=dev)
    gnum = torch.empty(wl.B, dtype=torch.int32, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20) // 4, dtype=torch.float32, device=dev)

    def compute(ins, lm_, gm_):
        if any_layer and n_layers > 1:
            lf.lf_encoder_forward_any_globals(ins[0], lm_, gm_, stack, wl.H, wl.w, out=out, workspace=ws)
        elif any_layer:
            lf.lf_encoder_layer_forward_any_globals(ins[0], lm_, gm_, wts, wl.H, wl.w, out=out, workspace=ws)
        elif layer and n_layers > 1:
            lf.lf_encoder_forward(ins[0], lm_, gm_, stack, wl.H, wl.w, out=out, workspace=ws)
        elif layer:
            lf.lf_encoder_layer_forward(ins[0], lm_, gm_, wts, wl.H, wl.w, out=out, workspace=ws)
        elif anyg:
            lf.lf_attention_forward_any_globals(*ins, lm_, gm_, wl.w, out=out)
        else:
            lf.lf_attention_forward(*ins, lm_, gm_, wl.w, out=out)

    # attention with prefix globals: the partition and the attention are one
    # kernel launch (lf_attention_forward_idx)
    prefix_attn = not (layer or anyg)

    def path(ins, lm_, gm_):
        # one pass of the whole hot path: the partition and the attention
        # (the any-position calls run their partition themselves)
        if anyg or any_layer:
            compute(ins, lm_, gm_)
        elif layer:
            lf.lf_init_global_idx(gm_, wl.w, gidx, gnum, sync=False)
            compute(ins, lm_, gm_)
        else:
            lf.lf_attention_forward_idx(*ins, lm_, gm_, wl.w, out=out, global_idx=gidx, global_token_nums=gnum)

    def step():
        path(args_in, lm, gm)

    def kernel_alone():
        # the dominant kernel alone: the step's one launch for the prefix
        # attention, else the attention (or layer) call
        if prefix_attn:
            path(args_in, lm, gm)
        else:
            compute(args_in, lm, gm)

    lf.lf_device_status(reset=True)
    for _ in range(max(args.warmup, 3)):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    st = lf.lf_device_status(reset=True)
    if st != 0:
        raise RuntimeError("device status after warm-up: %s" % lf.status_string(st))

    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_a = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_f = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    sampler = ClockSampler(local)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)  # let the sampler attach before the timed region
    for k in range(K):
        flush.zero_()
        ev_s[k].record()
        step()
        ev_e[k].record()
    # the dominant kernel (the attention kernel, or the whole layer) alone,
    # with the same L2 flush before every launch
    for k in range(K):
        flush.zero_()
        ev_a[k].record()
        kernel_alone()
        ev_f[k].record()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    step_ms = [ev_s[k].elapsed_time(ev_e[k]) for k in range(K)]
    attn_ms = [ev_a[k].elapsed_time(ev_f[k]) for k in range(K)]
    total_ms = sum(step_ms)
    attn_avg_ms = sum(attn_ms) / K
    step_q, attn_q = percentiles(step_ms), percentiles(attn_ms)
    total_ms, attn_avg_ms = max_over_ranks([total_ms, attn_avg_ms], dev)

    # L2-hot: the same step back to back without the flush (the inputs stay
    # in L2 where they fit); reported beside the primary L2-cold numbers
    Kh = max(10, min(K, 200))
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    eh0, eh1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eh0.record()
    for _ in range(Kh):
        step()
    eh1.record()
    torch.cuda.synchronize()
    hot_ms = max_over_ranks([eh0.elapsed_time(eh1) / Kh], dev)[0]

    # end to end through the public call: pinned host inputs -> device ->
    # partition + attention -> output back to pinned host memory
    E = max(1, args.e2e_steps)
    h_in = [x.cpu().pin_memory() for x in args_in] + [lm_cpu.pin_memory(), gm_cpu.pin_memory()]
    d_in = [torch.empty_like(x, device=dev) for x in h_in]
    h_out = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    h2d = sum(x.numel() * x.element_size() for x in h_in)
    d2h = h_out.numel() * h_out.element_size()

    n_t = len(args_in)

    def e2e_step():
        for h, d in zip(h_in, d_in):
            d.copy_(h, non_blocking=True)
        path(d_in[:n_t], d_in[n_t], d_in[n_t + 1])
        h_out.copy_(out, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(E):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E
    e2e_ms = max_over_ranks([e2e_ms], dev)[0]
    st = lf.lf_device_status(reset=True)
    if st != 0:
        raise RuntimeError("device status after timing: %s" % lf.status_string(st))

    pk, pk_kind = peaks()
    if layer:
        F = n_layers * metrics.layer_flops(wl.B, wl.H, wl.L, wl.w, wl.g, wl.pad, ffn)
        if any_layer:  # the attention part over the scattered key sets
            F += n_layers * (metrics.flops_masks(lm_cpu.numpy(), gm_cpu.numpy(), wl.H, wl.w)
                             - metrics.flops(wl.B, wl.H, wl.L, wl.w, wl.g, wl.pad))
        wbytes = sum(v.numel() * v.element_size() for W in stack for v in W.values())
        By = float(wbytes + 2 * x.numel() * x.element_size() + 2 * wl.B * wl.L * 4)
    else:
        F = (metrics.flops_masks(lm_cpu.numpy(), gm_cpu.numpy(), wl.H, wl.w) if anyg
             else metrics.flops(wl.B, wl.H, wl.L, wl.w, wl.g, wl.pad))
        By = metrics.algorithmic_bytes(wl.B, wl.H, wl.L, wl.w, wl.g, wl.dtype)
    t_attn = attn_avg_ms * 1e-3
    tokens = wl.B * wl.L
    value = job_throughput(world, tokens, K, total_ms)
    tensor_path = wl.dtype in ("f16", "bf16")
    if layer:
        roof = {"bound": "tensor", "achieved": F / t_attn / 1e12, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": F / t_attn / 1e12 / pk["bf16_tflops"], "traffic": None, "peak_kind": pk_kind,
                "algorithmic_bytes_per_launch": By, "flops_per_launch": F}
    else:
        roof = {"bound": "hbm", "achieved": By / t_attn / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": By / t_attn / 1e9 / pk["hbm_gbs"],
                "traffic": traffic_from_profile(kernel_source_hash()) if args.workload == WORKLOAD_ID else None,
                "peak_kind": pk_kind, "algorithmic_bytes_per_launch": By, "flops_per_launch": F}
    res = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype,
        "data": "synthetic (seeded inputs of the workload's shape%s)" %
                (": x ~ N(0,1), weights ~ N(0, 0.02)" if layer else ", N(0,1)*0.5"),
        "config": {"workload": wl.name + (", globals at random positions" if any_layer else "")
                   + (" x %d layers" % n_layers if layer and n_layers > 1 else ""),
                   "B": wl.B, "H": wl.H, "L": wl.L, "w": wl.w, "g": wl.g,
                   "pad": wl.pad, "head_dim": 64, "l2": "flushed before every timed step (2 x L2 write)",
                   **({"ffn_path": args.ffn_path} if layer else {}),
                   "parallelism": "replica per GPU (weak)" if world > 1 else "single GPU"},
        "tflops": F / (total_ms * 1e-3 / K) / 1e12,
        "step_us": {k: (v * 1e3 if v is not None else None) for k, v in step_q.items()},
        "l2_hot": {"ms_per_step": hot_ms, "value": job_throughput(world, wl.B * wl.L, 1, hot_ms), "unit": "tokens/s",
                   "steps": Kh, "note": "no L2 flush between steps (inputs stay in L2 where they fit)"},
        ("layer" if layer else "attention_kernel"): {
            "avg_us": attn_avg_ms * 1e3,
            "us_percentiles": {k: (v * 1e3 if v is not None else None) for k, v in attn_q.items()},
            "tflops": F / t_attn / 1e12,
            "tensor_peak_frac": F / t_attn / 1e12 / pk["bf16_tflops"] if tensor_path else None,
            "tensor_peak_tflops": pk["bf16_tflops"],
            "note": "fp16 and bf16 dense tensor rates are equal; peak = measured bf16 burst (%s)" % pk_kind
                    + ("; the timed call is the fused partition + gather kernel and the attention kernel"
                       if anyg else ""),
        },
        "roofline": roof,
        "e2e": {"value": job_throughput(world, tokens, 1, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        # our kernels per step: any-position attention = partition-and-gather
        # + attention; layer = partition + 5 per layer (projections with Qg,
        # attention, output projection with LN1, then FFN1 and FFN2 with LN2,
        # or the fused FFN and the LN2 kernel); any-position layer =
        # partition + 7 per layer (the row gathers added); prefix attention = 1
        "gpu_launches": (2 if anyg else (1 + 7 * n_layers) if any_layer
                         else 1 + 5 * n_layers if layer
                         else 1) * K,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not layer:
        res["cpu_baseline"] = cpu_baseline(wl, t_cpu, lm_cpu, gm_cpu)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(res))


# ---------------------------------------------------------------- reference arm (the oracle)

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import numpy as np
    import oracle
    wl, t_cpu, lm_cpu, gm_cpu = inputs.workload_inputs(WORKLOAD_ID)
    arrs = [t_cpu[n].double().numpy() for n in inputs.NAMES]
    lmn, gmn = lm_cpu.numpy(), gm_cpu.numpy()
    H = wl.H

    def rows_for(pos0, npos):
        pos = (np.arange(npos) + pos0) % wl.L
        return np.array([[0, h, p] for p in pos for h in range(H)], dtype=np.int32)

    # calibrate: size each step so the whole run takes about a minute
    t0 = time.perf_counter()
    oracle.attention_rows(*arrs, lmn, gmn, wl.w, rows_for(0, 64))
    per_pos = (time.perf_counter() - t0) / 64
    K, W = args.steps, args.warmup
    npos = int(max(1, min(wl.L, 60.0 / max(1, K + W) / per_pos)))
    for k in range(W):
        oracle.attention_rows(*arrs, lmn, gmn, wl.w, rows_for(k * npos, npos))
    t0 = time.perf_counter()
    for k in range(K):
        oracle.attention_rows(*arrs, lmn, gmn, wl.w, rows_for((W + k) * npos, npos))
    el = time.perf_counter() - t0
    value = npos * K / el
    res = {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": el * 1e3 / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1)*0.5 inputs of the workload's shape)",
        "config": {"workload": wl.name, "B": wl.B, "H": wl.H, "L": wl.L, "w": wl.w, "g": wl.g,
                   "pad": wl.pad, "head_dim": 64},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": "%d positions x %d heads per step (float64 C oracle)" % (npos, H)},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res))


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
