"""Benchmark of the mixed-precision attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
quantize V to E4M3 (per-tensor scale, GPU block quantizer) and run the fused
attention forward (QK^T in BF16, P and V in E4M3, BF16 output) -- the
"dense context FMHA, QK-BF16 / PV-FP8" workload: B=1, H=40, D=128,
Sq=Skv=32768, non-causal, Q/K/V drawn N(0,1).

Metric: attention TFLOPS = 4*B*H*Sq*Skv*D*density / time (density 1 here).
Prints ONE JSON line (rank 0). ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead (no GPU work).

Multi-GPU (torchrun, one process per GPU): every rank runs its own replica of
the workload (weak scaling, no collective on the data path); the timed
region is bracketed by barriers and the max over ranks is reported.
"""

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOPS (4·B·H·Sq·Skv·D·density) and % of dtype tensor peak"
UNIT = "TFLOPS"
WORKLOADS = {
    # name: (B, H, S, D)
    "dense_pv8_s32768": (1, 40, 32768, 128),
    "dense_pv8_s16384": (1, 40, 16384, 128),
    "dense_pv8_s4096": (1, 40, 4096, 128),
}
DEFAULT_WORKLOAD = "dense_pv8_s32768"


def load_peaks():
    """Measured peaks of this machine's B200s (bf16 tensor burst, HBM copy)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            mp = json.load(f)
        return float(mp["bf16_tflops"]), float(mp["hbm_gbs"]), "measured"
    return 1590.0, 6650.0, "fallback"


def flops(B, H, S, D):
    return 4.0 * B * H * S * S * D


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_bench_{os.getpid()}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu_index), "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
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
        self.f.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                except ValueError:
                    continue
                for n, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ ours ----
def run_ours(args):
    from precision_attention_fmha_b200 import fmha, workloads
    from precision_attention_fmha_b200.fmha import Scale

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    B, H, S, D = WORKLOADS[args.workload]
    w = workloads.dense_pv8(S=S, B=B, H=H, D=D)
    q_h, k_h, v_h = (w[n].pin_memory() for n in ("q", "k", "v"))
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    scale = w["scale"]
    v8 = torch.empty(v.shape, dtype=torch.float8_e4m3fn, device=dev)
    sv = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(fmha.quantize_workspace_bytes("per_tensor", B, S, H, D), dtype=torch.uint8, device=dev)
    o = torch.empty(q.shape, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()

    def step(qd, kd, vd):
        fmha.fmha_quantize_blockwise(vd, torch.float8_e4m3fn, "per_tensor", out=v8, scales=sv, workspace=ws)
        fmha.fmha_fwd(qd, kd, v8, out=o, sf_v=Scale(sv, "per_tensor"), softmax_scale=scale)

    for _ in range(args.warmup):
        step(q, k, v)
    fmha.get_device_error()
    torch.cuda.synchronize()

    # ---- device-timed region: inputs resident in HBM ----
    K = args.steps
    attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(K):
        fmha.fmha_quantize_blockwise(v, torch.float8_e4m3fn, "per_tensor", out=v8, scales=sv, workspace=ws)
        attn_ev[i][0].record(stream)
        fmha.fmha_fwd(q, k, v8, out=o, sf_v=Scale(sv, "per_tensor"), softmax_scale=scale)
        attn_ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    fmha.get_device_error()
    ms = t0.elapsed_time(t1) / K
    attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ev)
    ms = max_over_ranks(ms, world)
    attn_ms = max_over_ranks(attn_ms, world)

    # ---- end-to-end: host (pinned) inputs, H2D + path + D2H of O each step ----
    o_h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    Ke = max(1, min(K, 10))
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(Ke):
        qd, kd, vd = (t.to(dev, non_blocking=True) for t in (q_h, k_h, v_h))
        step(qd, kd, vd)
        o_h.copy_(o, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
    fmha.get_device_error()

    fl = flops(B, H, S, D)
    tflops = world * fl / (ms * 1e-3) / 1e12
    bf16_peak, _, peak_src = load_peaks()
    # QK^T runs at the BF16 rate, PV at the E4M3 rate (2x BF16 nominal): time-weighted peak.
    peak = 1.0 / (0.5 / bf16_peak + 0.5 / (2.0 * bf16_peak))
    achieved = fl / (attn_ms * 1e-3) / 1e12
    cpu = cpu_baseline(B, H, S, D, w) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    bytes_in = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    line = {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16,e4m3", "data": "synthetic (seeded N(0,1), BF16)",
        "config": {"workload": args.workload, "B": B, "H": H, "Sq": S, "Skv": S, "D": D, "causal": False,
                   "q_k": "bf16", "v": "e4m3 per-tensor (quantized in the step)", "p": "e4m3", "o": "bf16",
                   "l2": "inputs larger than L2 (each of Q, K, V is %d MB)" % (q.numel() * 2 // 2**20),
                   "parallelism": f"replicas{world}"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": round(peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_note": f"{peak_src} bf16 burst {bf16_peak} x (QK at 1x, PV at 2x nominal E4M3 rate)",
                     "kernel": "attn_fwd_kernel", "kernel_ms": round(attn_ms, 4),
                     "frac_of_bf16_peak": round(achieved / bf16_peak, 4)},
        "e2e": {"value": round(world * fl / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": bytes_in, "d2h_bytes_per_step": o.numel() * o.element_size(),
                "steps": Ke},
        "gpu_launches": K * 3,
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ------------------------------------------------------------- reference ----
def oracle_sample(w, B, H, S, D, heads=1, rows=256):
    """The CPU oracle on a bounded sample: V quantized (per tensor over the
    sampled heads) then float64 attention for `rows` query rows of `heads`
    heads against the full key length. Returns (seconds, flops done)."""
    from oracle import attention as oa
    from oracle import quant as oq

    q = w["q"][:, :rows, :heads].to(torch.float64).numpy()
    k = w["k"][:, :, :heads].to(torch.float64).numpy()
    v = w["v"][:, :, :heads].to(torch.float32).numpy()
    t = time.perf_counter()
    codes, sc = oq.quantize_blockwise(v, "e4m3", "per_tensor")
    vd = oq.dequantize(codes, sc, "e4m3", "per_tensor")
    oa.attention(q, k, vd, w["scale"])
    dt = time.perf_counter() - t
    return dt, 4.0 * B * heads * rows * S * D


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def cpu_baseline(B, H, S, D, w, rows=1024):
    dt, fl = oracle_sample(w, B, H, S, D, heads=1, rows=rows)
    return {"value": round(fl / dt / 1e12, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"head 0, query rows 0..{rows - 1} against all {S} keys (plus V quantization of that head), "
                      f"float64 NumPy, {dt:.1f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from precision_attention_fmha_b200 import workloads

    B, H, S, D = WORKLOADS[args.workload]
    w = workloads.dense_pv8(S=S, B=B, H=H, D=D)
    rows = 256
    for _ in range(args.warmup):
        oracle_sample(w, B, H, S, D, rows=rows)
    times, fl = [], 0
    for _ in range(args.steps):
        dt, fl = oracle_sample(w, B, H, S, D, rows=rows)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    val = fl / (ms * 1e-3) / 1e12
    sample = f"head 0, query rows 0..{rows - 1} against all {S} keys, float64 NumPy oracle per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), BF16)",
        "config": {"workload": args.workload, "B": B, "H": H, "Sq": S, "Skv": S, "D": D, "causal": False},
        "cpu_baseline": {"value": round(val, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
