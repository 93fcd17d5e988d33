#!/usr/bin/env python3
"""Throughput bench of the RWKV-4 WKV forward+backward step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = wkv4_forward (writing the state checkpoints) followed by
wkv4_backward over one batch of the RWKV-4 169M-width workload
(B=8, T=1024, C=768, float32 k/v/y, fp32 state; w = exp(U(-6,1)),
u ~ U(-1,1), k ~ N(0, 2^2), v, gy ~ N(0,1); seed 0). Inputs are resident in
HBM; L2 is flushed (a 320 MB write) before every timed step and each step is
timed alone with CUDA events on the launching stream. Under torchrun every
rank runs its own replica on its own GPU (no collective on the data path) and
the job time is the max over ranks.

Printed (rank 0, one JSON line): G tok*ch/s = B*T*C*N / step time, the
end-to-end figure through the C ABI with pinned host buffers, the roofline of
the dominant kernel (the backward) against the measured HBM bandwidth, the
fp64 CPU oracle timed on a bounded sample, SM clocks sampled during the timed
region, and the number of library kernels launched.

--impl reference times the fp64 CPU oracle (the only reference this project
has) on the same workload and metric.
"""

from __future__ import annotations

import argparse
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

WORKLOAD = "wkv4_fb_f32_169m"
METRIC = "WKV fwd+bwd throughput (G tok·ch/s)"
UNIT = "G tok*ch/s"
L2_FLUSH_BYTES = 320 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "of measured"
    return 6650.0, "of fallback"


def kernel_source_hash(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel, workload, src_hash):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}:{workload}")
    if not e or e.get("source_hash") != src_hash:
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(parts)
                except ValueError:
                    pass
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ----------------------------------------------------------------------------

def cpu_baseline(inp, budget_s=12.0):
    """Time the fp64 oracle's forward+backward on channel slices of the
    workload until about `budget_s` seconds of CPU work are done."""
    import oracle
    oracle.build()
    B, T, C = inp["k32"].shape
    width = 96
    done_tc = 0
    t_total = 0.0
    c0 = 0
    slices = 0
    while t_total < budget_s and slices < 64:
        cs = slice(c0, min(C, c0 + width))
        args = (inp["w"][cs], inp["u"][cs], inp["k32"][:, :, cs], inp["v32"][:, :, cs])
        t = time.perf_counter()
        oracle.wkv4_forward(*args)
        oracle.wkv4_backward(*args, inp["gy32"][:, :, cs])
        t_total += time.perf_counter() - t
        done_tc += B * T * (cs.stop - cs.start)
        c0 = (c0 + width) % C
        slices += 1
    return {"value": done_tc / t_total / 1e9, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
            "sample": f"{slices} slices of {width} channels x B={B} x T={T} (fwd+bwd, fp64), "
                      f"{done_tc / 1e6:.1f} M tok*ch in {t_total:.1f} s"}


# ----------------------------------------------------------------------------
# reference arm: the CPU oracle
# ----------------------------------------------------------------------------

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from rwkv_wkv_linear_mix_b200 import synth
    rec = synth.WKV4_RECIPES[WORKLOAD]
    inp = synth.wkv4_inputs(rec, seed=0)
    import oracle
    oracle.build()
    B, T, C = rec.B, rec.T, rec.C
    width = 48
    per_step = []
    c0 = 0
    for i in range(args.warmup + args.steps):
        cs = slice(c0, c0 + width)
        a = (inp["w"][cs], inp["u"][cs], inp["k32"][:, :, cs], inp["v32"][:, :, cs])
        t = time.perf_counter()
        oracle.wkv4_forward(*a)
        oracle.wkv4_backward(*a, inp["gy32"][:, :, cs])
        dt = time.perf_counter() - t
        if i >= args.warmup:
            per_step.append(dt)
        c0 = (c0 + width) % C
    tot = sum(per_step)
    val = B * T * width * len(per_step) / tot / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "C": C, "sample_channels_per_step": width},
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
                         "sample": f"each step: {width} of {C} channels x B={B} x T={T}, fwd+bwd in fp64"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args):
    import torch
    rank, world, local = dist_env()
    if world > 1:
        torch.cuda.set_device(local)
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", torch.cuda.current_device())
    from rwkv_wkv_linear_mix_b200 import synth, wkv

    rec = synth.WKV4_RECIPES[WORKLOAD]
    B, T, C = rec.B, rec.T, rec.C
    inp = synth.wkv4_inputs(rec, seed=0)
    tok_ch = B * T * C

    def to_dev(a):
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    w, u, k, v, gy = (to_dev(inp[n]) for n in ("w", "u", "k", "v", "gy"))
    y = torch.empty_like(k)
    gk, gv = torch.empty_like(k), torch.empty_like(k)
    gw = torch.empty(C, dtype=torch.float32, device=dev)
    gu = torch.empty(C, dtype=torch.float32, device=dev)
    ckpt = torch.empty(wkv.ckpt_shape(B, T, C), dtype=torch.float32, device=dev)
    ws = torch.empty(max(16, wkv.wkv4_backward_workspace_bytes(B, T, C, True)), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        wkv.wkv4_forward(w, u, k, v, y=y, ckpt=ckpt)
        wkv.wkv4_backward(w, u, k, v, gy, ckpt, gk=gk, gv=gv, gw=gw, gu=gu, workspace=ws)

    launches_per_step = 3  # forward kernel, backward kernel, batch-sum kernel

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()

    clock = ClockSampler(local) if rank == 0 or world > 1 else None
    if clock:
        clock.start()
        time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    for i in range(args.steps):
        flush.zero_()
        e0, e1, e2 = ev[i]
        e0.record(stream)
        wkv.wkv4_forward(w, u, k, v, y=y, ckpt=ckpt)
        e1.record(stream)
        wkv.wkv4_backward(w, u, k, v, gy, ckpt, gk=gk, gv=gv, gw=gw, gu=gu, workspace=ws)
        e2.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = clock.stop() if clock else None
    t_fwd = [a.elapsed_time(b) for a, b, _ in ev]
    t_bwd = [b.elapsed_time(c) for _, b, c in ev]
    step_ms = sum(f + b for f, b in zip(t_fwd, t_bwd)) / args.steps
    t_local = torch.tensor([step_ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t_local, op=dist.ReduceOp.MAX)
    step_ms_max = float(t_local.item())
    value = tok_ch * world / (step_ms_max * 1e-3) / 1e9

    # ---- end to end through the C ABI with pinned host buffers ----
    hk, hv, hgy = (torch.from_numpy(np.ascontiguousarray(inp[n])).pin_memory() for n in ("k", "v", "gy"))
    hw, hu = (torch.from_numpy(np.ascontiguousarray(inp[n])).pin_memory() for n in ("w", "u"))
    hy, hgk, hgv = (torch.empty(k.shape, dtype=k.dtype).pin_memory() for _ in range(3))
    hgw, hgu = (torch.empty(C, dtype=torch.float32).pin_memory() for _ in range(2))
    h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hgy, hw, hu))
    d2h = sum(t.numel() * t.element_size() for t in (hy, hgk, hgv, hgw, hgu))

    def e2e_step():
        for d, h in ((k, hk), (v, hv), (gy, hgy), (w, hw), (u, hu)):
            d.copy_(h, non_blocking=True)
        step()
        for h, d in ((hy, y), (hgk, gk), (hgv, gv), (hgw, gw), (hgu, gu)):
            h.copy_(d, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(5, min(args.steps, 20))
    e_s.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e_e.record(stream)
    torch.cuda.synchronize()
    e2e_ms = torch.tensor([e_s.elapsed_time(e_e) / e2e_steps], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(e2e_ms, op=dist.ReduceOp.MAX)
        dist.barrier()
    e2e_val = tok_ch * world / (float(e2e_ms.item()) * 1e-3) / 1e9
    assert wkv.device_error(reset=True) == 0, "a kernel recorded a device-side error"

    # ---- roofline of the dominant kernel (the backward) ----
    peak, peak_kind = measured_peaks()
    bwd_ms = statistics.mean(t_bwd)
    fwd_ms = statistics.mean(t_fwd)
    bwd_bytes = 20 * tok_ch   # k, v, gy read; gk, gv written (float32)
    fwd_bytes = 12 * tok_ch   # k, v read; y written
    achieved = bwd_bytes / (bwd_ms * 1e-3) / 1e9
    src_hash = kernel_source_hash(["rwkv_wkv_linear_mix_b200/csrc/wkv4_bwd.cu",
                                   "rwkv_wkv_linear_mix_b200/csrc/wkv_device.cuh"])
    roof = {"bound": "hbm", "kernel": "wkv4_bwd_kernel<float>", "achieved": achieved, "peak": peak,
            "unit": "GB/s", "frac": achieved / peak, "peak_kind": peak_kind,
            "traffic": recorded_traffic("wkv4_bwd_kernel", WORKLOAD, src_hash),
            "algorithmic_bytes_per_launch": bwd_bytes, "avg_launch_ms": bwd_ms,
            "forward": {"achieved": fwd_bytes / (fwd_ms * 1e-3) / 1e9, "avg_launch_ms": fwd_ms,
                        "algorithmic_bytes_per_launch": fwd_bytes}}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms_max, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": WORKLOAD, "B": B, "T": T, "C": C, "global_batch": B * world, "seq_len": T,
                   "parallelism": f"replicas{world}", "l2": "flushed (320 MB write) before every timed step",
                   "ckpt_len": wkv.CKPT_LEN},
        "e2e": {"value": e2e_val, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "roofline": roof,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inp)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
