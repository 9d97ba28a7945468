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
import tempfile
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "attention TFLOPS (4·B·H·Sq·Skv·D·density) and % of dtype tensor peak"
UNIT = "TFLOPS"
WORKLOADS = {
    # name: (kind, B, Hq, Hkv, S, D, causal)
    "dense_pv8_s32768": ("pv8", 1, 40, 40, 32768, 128, False),
    "dense_pv8_s16384": ("pv8", 1, 40, 40, 16384, 128, False),
    "dense_pv8_s4096": ("pv8", 1, 40, 40, 4096, 128, False),
    # the same with an E4M3 output, O / sf_o with sf_o = V's per-tensor scale (|O| <= max |V|)
    "dense_pv8_o8_s32768": ("pv8_o8", 1, 40, 40, 32768, 128, False),
    "dense_bf16_s16384": ("bf16", 1, 40, 40, 16384, 128, False),
    "dense_bf16_s4096": ("bf16", 1, 40, 40, 4096, 128, False),
    "tiny_bf16": ("bf16", 1, 1, 1, 256, 64, False),
    "all_fp8_s8192": ("fp8", 2, 32, 32, 8192, 128, False),
    "all_fp8_s8192_causal": ("fp8", 2, 32, 32, 8192, 128, True),
    "sage_s16384": ("sage", 1, 24, 24, 16384, 128, False),
    # the same with P split into two E4M3 terms (about 7 significant bits, twice the PV work)
    "sage_p2_s16384": ("sage_p2", 1, 24, 24, 16384, 128, False),
    # a 192-wide Q/K head dim with a 128-wide V / O (flops 2·B·H·Sq·Skv·(192 + 128))
    "wide_qk_bf16_s16384": ("wide_bf16", 1, 40, 40, 16384, 192, False),
    "wide_qk_pv8_s16384": ("wide_pv8", 1, 40, 40, 16384, 192, False),
    "wide_qk_fp8_s16384": ("wide_fp8", 1, 40, 40, 16384, 192, False),
    "sparse_paged_s16384": ("sparse_paged", 4, 64, 8, 16384, 128, False),
    # the same mask, Q and K/V values with K/V contiguous [B, S, Hkv, D] (the paged-overhead control)
    "sparse_contig_s16384": ("sparse_contig", 4, 64, 8, 16384, 128, False),
    # decode step: one query token per sequence against S cached tokens (S is Skv)
    "decode_paged_s16384": ("decode_paged", 4, 64, 8, 16384, 128, False),
    # per-token NVFP4 quantization of S tokens x D channels (B, H unused)
    "nvfp4_t16384_k4096": ("nvfp4", 1, 1, 1, 16384, 4096, False),
    # SageAttention K smoothing of the Sage workload's K: token mean per channel + shifted INT8 quantizer
    "sage_k_smooth_s16384": ("smooth_k", 1, 24, 24, 16384, 128, False),
    # the token-block quantizer alone on the same K: INT8 codes with one scale per 64 tokens of a head
    "sage_k_quant_s16384": ("quant_k", 1, 24, 24, 16384, 128, False),
}
DEFAULT_WORKLOAD = "dense_pv8_s32768"
L2_BYTES = 126 * 2**20          # B200 L2
L2_FLUSH_BYTES = 512 * 2**20    # written between timed steps when the inputs fit in L2 (~80 us)


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
        # raw samples go to a scratch file (set CLOCKS_CSV_DIR to keep them); the summary is in the JSON line
        self.path = os.path.join(os.environ.get("CLOCKS_CSV_DIR") or tempfile.gettempdir(),
                                 f"clocks_bench_{os.getpid()}.csv")

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


from precision_attention_fmha_b200.replicas import barrier, job_throughput, max_over_ranks, teardown  # noqa: E402
from precision_attention_fmha_b200.replicas import setup as replicas_setup  # noqa: E402


def dist_setup(n_gpus):
    """Replicas only: one process per GPU over NCCL, no collective on the data path."""
    return replicas_setup("nccl")


# ------------------------------------------------------------- workloads ----
class Work:
    """One workload: host inputs, GPU quantization prep, the attention call."""

    def __init__(self, name, dev, fmha, workloads, Scale):
        kind, B, Hq, Hkv, S, D, causal = WORKLOADS[name]
        self.name = name
        self.kind, self.B, self.Hq, self.Hkv, self.S, self.D, self.causal = kind, B, Hq, Hkv, S, D, causal
        self.dev, self.fmha, self.Scale = dev, fmha, Scale
        bf16_peak, _, src = load_peaks()
        self.peak_src = src
        E4 = torch.float8_e4m3fn
        if kind == "bf16":
            w = workloads.normal_qkv(workloads.SEED_BASE + 1 + S, B, S, S, Hq, Hkv, D)
            self.host = dict(zip(("q", "k", "v"), w))
            self.peak, self.peak_note, self.dtype = bf16_peak, "bf16 burst", "bf16"
            self.quant = []
        elif kind in ("pv8", "pv8_o8"):
            w = workloads.dense_pv8(S=S, B=B, H=Hq, D=D)
            self.host = {n: w[n] for n in ("q", "k", "v")}
            self.peak = 1.0 / (0.5 / bf16_peak + 0.5 / (2.0 * bf16_peak))
            self.peak_note = f"bf16 burst {bf16_peak} for QK^T, 2x (nominal E4M3 ratio) for PV, time-weighted"
            self.dtype = "bf16,e4m3" if kind == "pv8" else "bf16,e4m3,o:e4m3"
            self.quant = [("v", E4, "per_tensor", None)]
        elif kind == "fp8":
            w = workloads.all_fp8(S=S, B=B, H=Hq, D=D)
            self.host = {n: w[n] for n in ("q", "k", "v")}
            self.peak, self.peak_note, self.dtype = 2.0 * bf16_peak, f"2 x bf16 burst {bf16_peak} (nominal E4M3 ratio)", "e4m3"
            self.quant = [("q", E4, "per_head", None), ("k", E4, "per_head", None), ("v", E4, "per_head", None)]
        elif kind in ("sage", "sage_p2"):
            w = workloads.sage(S=S, B=B, H=Hq, D=D)
            self.host = {n: w[n] for n in ("q", "k", "v")}
            self.peak = 2.0 * bf16_peak
            self.peak_note = f"2 x bf16 burst {bf16_peak} (nominal INT8 and E4M3 ratio)"
            self.dtype = "int8,e4m3"
            self.quant = [("q", torch.int8, "per_token_block", 128), ("k", torch.int8, "per_token_block", 64),
                          ("v", E4, "per_channel", None)]
        elif kind in ("sparse_paged", "decode_paged"):
            gen = workloads.sparse_paged if kind == "sparse_paged" else workloads.decode_paged
            w = gen(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D)
            self.host = {"q": w["q"], "k_pool": w["k_pool"], "v_pool": w["v_pool"], "page_table": w["page_table"],
                         "mask": w["mask"]}
            self.peak, self.peak_note, self.dtype = bf16_peak, "bf16 burst", "bf16"
            self.quant = []
        elif kind in ("wide_bf16", "wide_pv8", "wide_fp8"):
            w = workloads.wide_qk(S=S, B=B, H=Hq, D=D, outliers=kind == "wide_fp8")
            self.host = {n: w[n] for n in ("q", "k", "v")}
            if kind == "wide_bf16":
                self.peak, self.peak_note, self.dtype = bf16_peak, "bf16 burst", "bf16"
                self.quant = []
            elif kind == "wide_pv8":  # QK^T carries 192 / 320 of the flops
                self.peak = 1.0 / (0.6 / bf16_peak + 0.4 / (2.0 * bf16_peak))
                self.peak_note = (f"bf16 burst {bf16_peak} for QK^T, 2x (nominal E4M3 ratio) for PV, "
                                  "flop-weighted 192:128")
                self.dtype = "bf16,e4m3"
                self.quant = [("v", E4, "per_tensor", None)]
            else:
                self.peak, self.peak_note, self.dtype = 2.0 * bf16_peak, f"2 x bf16 burst {bf16_peak} (nominal E4M3 ratio)", "e4m3"
                self.quant = [("q", E4, "per_head", None), ("k", E4, "per_head", None), ("v", E4, "per_head", None)]
        elif kind == "sparse_contig":
            w = workloads.sparse_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D)
            self.host = {"q": w["q"], "k": w["k"], "v": w["v"], "mask": w["mask"]}
            self.peak, self.peak_note, self.dtype = bf16_peak, "bf16 burst", "bf16"
            self.quant = []
        self.scale = 1.0 / math.sqrt(D)
        self.host = {n: t.contiguous().pin_memory() for n, t in self.host.items()}
        self.dev_in = {n: t.to(dev) for n, t in self.host.items()}
        self.Sq = self.host["q"].shape[1]
        self.o8 = kind == "pv8_o8"
        self.Dv = self.host["v_pool" if "v_pool" in self.host else "v"].shape[3]
        self.o = torch.empty((B, self.Sq, Hq, self.Dv), dtype=E4 if self.o8 else torch.bfloat16, device=dev)
        # density = kept score elements / (Sq * Skv)
        self.ws = None
        if kind in ("sparse_paged", "sparse_contig"):
            kept = float(self.host["mask"].to(torch.float64).sum())
            self.density = kept * 128 * 128 / (B * Hkv * S * S)
            self.flop = 4.0 * B * Hq * S * S * D * self.density
        elif kind == "decode_paged":  # every query row sees the kept 128-key blocks of its KV head
            kept = float(self.host["mask"].to(torch.float64).sum())
            self.density = kept * 128 / (B * Hkv * S)
            self.flop = 4.0 * B * Hq * self.Sq * S * D * self.density
            # HBM roofline: the kept K/V bytes (each read once), Q, O, page table and mask
            self.hbm_bytes = (kept * 128 * D * 2 * 2 + 2 * B * self.Sq * Hq * D * 2
                              + self.host["page_table"].numel() * 4 + self.host["mask"].numel())
            self.q_dev = self.dev_in["q"]
            nbytes = fmha.decode_workspace_bytes(self.q_dev, self.dev_in["k_pool"], S)
            self.ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device=dev)
            self.n_parts = fmha.decode_num_parts(self.q_dev, self.dev_in["k_pool"], S)
        else:
            self.density = (S + 1) / (2 * S) if causal else 1.0
            self.flop = 2.0 * B * Hq * S * S * (D + self.Dv) * self.density
        self.qbuf = {}
        for name, dt, gran, rpb in self.quant:
            x = self.dev_in[name]
            xd = x.shape[3]
            shp = fmha.scale_shape(gran, B, S, x.shape[2], xd, rpb)
            self.qbuf[name] = (torch.empty(x.shape, dtype=dt, device=dev), torch.empty(shp, dtype=torch.float32,
                               device=dev), torch.empty(max(4, fmha.quantize_workspace_bytes(gran, B, S, x.shape[2], xd)),
                                                        dtype=torch.uint8, device=dev), gran, rpb, dt)
        # bytes one step reads: all inputs, or for decode the kept K/V blocks
        touched = (self.hbm_bytes if kind == "decode_paged"
                   else sum(t.numel() * t.element_size() for t in self.host.values()))
        self.fits_l2 = touched <= L2_BYTES
        self.sf_p = None
        self.p_terms = 2 if kind == "sage_p2" else 1
        if kind in ("sage", "sage_p2"):  # per-row-block P scale: P stored as 224 p
            self.sf_p = Scale(torch.full((B, Hq, math.ceil(S / 128)), workloads.SAGE_SF_P, device=dev), "per_token_block", 128)
        # our kernels per step: token-block quantization is 1 launch, the grid-wide kinds 2, attention 1
        # (decode: + the split merge when there are several partials)
        self.launches = 1 + sum(1 if g == "per_token_block" else 2 for _, _, g, _ in self.quant)
        if kind == "decode_paged" and self.n_parts > 1:
            self.launches += 1

    def prep(self, inp):
        for name, (out, sc, ws, gran, rpb, dt) in self.qbuf.items():
            self.fmha.fmha_quantize_blockwise(inp[name], dt, gran, rpb, out=out, scales=sc, workspace=ws)

    def attn(self, inp):
        f, S_ = self.fmha, self.Scale
        if self.kind == "sparse_paged":
            f.fmha_fwd_paged(inp["q"], inp["k_pool"], inp["v_pool"], inp["page_table"], self.S, mask=inp["mask"],
                             out=self.o, softmax_scale=self.scale)
            return
        if self.kind == "sparse_contig":
            f.fmha_fwd_block_sparse(inp["q"], inp["k"], inp["v"], inp["mask"], out=self.o, softmax_scale=self.scale)
            return
        if self.kind == "decode_paged":
            f.fmha_fwd_decode(inp["q"], inp["k_pool"], inp["v_pool"], page_table=inp["page_table"], Skv=self.S,
                              mask=inp["mask"], workspace=self.ws, out=self.o, softmax_scale=self.scale)
            return
        ops = {n: inp[n] for n in ("q", "k", "v")}
        sfs = {}
        for name, (out, sc, ws, gran, rpb, dt) in self.qbuf.items():
            ops[name] = out
            sfs["sf_" + name] = S_(sc, gran, rpb or 0)
        if self.o8:  # O is a convex combination of V's rows: V's scale keeps O / sf_o within +-448
            sfs["sf_o"] = S_(self.qbuf["v"][1], "per_tensor", 0)
        f.fmha_fwd(ops["q"], ops["k"], ops["v"], out=self.o, softmax_scale=self.scale, causal=self.causal,
                   sf_p=self.sf_p, p_terms=self.p_terms, **sfs)

    def config(self, world):
        c = {"workload": self.name, "B": self.B,
             "Hq": self.Hq,
             "Hkv": self.Hkv, "Sq": self.Sq, "Skv": self.S, "D": self.D, "Dv": self.Dv, "causal": self.causal,
             "density": round(self.density, 6),
             "quantized_in_step": [f"{n}:{g}" for n, _, g, _ in self.quant], "p_terms": self.p_terms,
             "l2": "inputs fit in L2: flushed before each step (512 MiB write, outside the timed events)"
                   if self.fits_l2 else "inputs larger than L2",
             "parallelism": f"replicas{world}"}
        if self.Dv != self.D:
            c["flops"] = "2·B·H·Sq·Skv·(D + Dv)·density (the metric's 4·…·D when D = Dv)"
        return c


def roofline(W, args, attn_ms, achieved_tflops):
    if W.kind == "decode_paged":  # HBM-bound: algorithmic bytes per launch over the measured copy bandwidth
        _, hbm, src = load_peaks()
        gbs = W.hbm_bytes / (attn_ms * 1e-3) / 1e9
        return {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                "frac": round(gbs / hbm, 4), "traffic": TRAFFIC.get(args.workload),
                "peak_note": f"{src}: HBM copy bandwidth", "algorithmic_bytes": int(W.hbm_bytes),
                "kernel": "attn_fwd_kernel (packed, split-KV) + split_merge_kernel", "kernel_ms": round(attn_ms, 4)}
    r = {"bound": "tensor", "achieved": round(achieved_tflops, 2), "peak": round(W.peak, 1), "unit": "TFLOP/s",
         "frac": round(achieved_tflops / W.peak, 4), "traffic": TRAFFIC.get(args.workload),
         "peak_note": f"{W.peak_src}: {W.peak_note}", "kernel": "attn_fwd_kernel", "kernel_ms": round(attn_ms, 4)}
    return r


def run_nvfp4(args):
    """Per-token NVFP4 quantization of a BF16 [S, D] activation matrix: HBM-bound."""
    from precision_attention_fmha_b200 import fmha

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    _, _, _, _, T, K, _ = WORKLOADS[args.workload]
    rng = np.random.default_rng(1000 + 7 + T)
    xh = torch.from_numpy(rng.standard_normal((T, K), dtype=np.float32)).to(torch.bfloat16).pin_memory()
    x = xh.to(dev)
    codes = torch.empty((T, K // 2), dtype=torch.uint8, device=dev)
    sb = torch.empty((T, K // 16), dtype=torch.uint8, device=dev)
    st = torch.empty((T,), dtype=torch.float32, device=dev)
    step = lambda inp: fmha.quantize_nvfp4(inp, codes=codes, block_scales=sb, token_scales=st)
    for _ in range(args.warmup):
        step(x)
    fmha.get_device_error()
    K_ = args.steps
    stream = torch.cuda.current_stream()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(K_):
        step(x)
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1) / K_, world)
    out_bytes = codes.numel() + sb.numel() + st.numel() * 4
    algo = x.numel() * 2 + out_bytes
    _, hbm, src = load_peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    # end to end: pinned host input in, codes and scales out, every step
    oh = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in (codes, sb, st)]
    Ke = max(1, min(K_, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Ke):
        step(xh.to(dev, non_blocking=True))
        for h, d in zip(oh, (codes, sb, st)):
            h.copy_(d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
    fmha.get_device_error()
    line = {
        "metric": "per-token NVFP4 quantization GB/s (2 B read + 0.5625 B written per element + 4 B per token)",
        "value": round(world * gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": K_, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->e2m1", "data": "synthetic (seeded N(0,1), BF16)",
        "config": {"workload": args.workload, "tokens": T, "K": K, "l2": "inputs fit in L2" if x.numel() * 2 <= 126 * 2**20
                   else "inputs larger than L2", "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "traffic": None, "peak_note": f"{src}: HBM copy bandwidth",
                     "algorithmic_bytes": int(algo), "kernel": "nvfp4_quant_kernel", "kernel_ms": round(ms, 5)},
        "e2e": {"value": round(world * algo / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": x.numel() * 2, "d2h_bytes_per_step": out_bytes, "steps": Ke},
        "gpu_launches": K_,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        from oracle import nvfp4 as on
        n = 512  # about 10 s of the per-row oracle
        tt = time.perf_counter()
        on.quantize_per_token(xh[:n].to(torch.float32).numpy())
        dt = time.perf_counter() - tt
        line["cpu_baseline"] = {"value": round(n * K * 2.5625 / dt / 1e9, 6), "unit": "GB/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": f"rows 0..{n - 1} of {T}, NumPy oracle, {dt:.2f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    teardown(world)


# ------------------------------------------------------------------ ours ----
def run_ours(args):
    from precision_attention_fmha_b200 import fmha, workloads
    from precision_attention_fmha_b200.fmha import Scale

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    W = Work(args.workload, dev, fmha, workloads, Scale)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        W.prep(W.dev_in)
        W.attn(W.dev_in)
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
    if W.fits_l2:
        # The inputs fit in L2: each step is timed alone, after a write of
        # twice the L2 size that evicts them (outside the step's events). The
        # flush kernel is still running when the step is queued behind it, so
        # no host launch gap falls inside the events.
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        for i in range(K):
            flush.zero_()
            attn_ev[i][0].record(stream)
            W.prep(W.dev_in)
            W.attn(W.dev_in)
            attn_ev[i][1].record(stream)
    else:
        t0.record(stream)
        for i in range(K):
            W.prep(W.dev_in)
            attn_ev[i][0].record(stream)
            W.attn(W.dev_in)
            attn_ev[i][1].record(stream)
        t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    fmha.get_device_error()
    if W.fits_l2:  # prep + attention between each step's events
        ms = attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ev)
    else:
        ms = t0.elapsed_time(t1) / K
        attn_ms = statistics.mean(a.elapsed_time(b) for a, b in attn_ev)
    ms = max_over_ranks(ms, world)
    attn_ms = max_over_ranks(attn_ms, world)

    # ---- end-to-end: host (pinned) inputs, H2D + path + D2H of O each step ----
    # Pipelined as a serving loop would run it: step i + 1's inputs are copied
    # host -> device on one stream while step i computes on the current stream,
    # and step i's O goes back on a third (two device buffers of each). Every
    # step's inputs and its O still cross the host link inside the timed region.
    # A decode step's KV cache stays resident (it is the serving state, not a
    # step input): it is copied once, before the timed region; the step's inputs
    # are the query, the page table and the mask.
    Ke = max(1, min(K, 10))
    resident = ("k_pool", "v_pool") if W.kind == "decode_paged" else ()
    h2d, d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    bufs = [{n: (W.dev_in[n] if n in resident else torch.empty(t.shape, dtype=t.dtype, device=dev))
             for n, t in W.host.items()} for _ in range(2)]
    outs = [W.o, torch.empty_like(W.o)]
    o_h = [torch.empty(W.o.shape, dtype=W.o.dtype, pin_memory=True) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(Ke)]
    ev_comp = [torch.cuda.Event() for _ in range(Ke)]
    ev_out = [torch.cuda.Event() for _ in range(Ke)]

    def copy_in(i):
        with torch.cuda.stream(h2d):
            if i >= 2:  # compute of step i - 2 has read this buffer
                h2d.wait_event(ev_comp[i - 2])
            for n, t in W.host.items():
                if n not in resident:
                    bufs[i % 2][n].copy_(t, non_blocking=True)
            ev_in[i].record(h2d)

    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(h2d)
    copy_in(0)
    for i in range(Ke):
        if i + 1 < Ke:
            copy_in(i + 1)
        stream.wait_event(ev_in[i])
        if i >= 2:  # the copy back of step i - 2 has read this O buffer
            stream.wait_event(ev_out[i - 2])
        W.o = outs[i % 2]
        W.prep(bufs[i % 2])
        W.attn(bufs[i % 2])
        ev_comp[i].record(stream)
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_comp[i])
            o_h[i % 2].copy_(outs[i % 2], non_blocking=True)
            ev_out[i].record(d2h)
    e1.record(d2h)  # after the last copy back, which waits for all the rest
    torch.cuda.synchronize()
    W.o = outs[0]
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
    fmha.get_device_error()

    tflops = job_throughput(W.flop, world, ms) / 1e12
    achieved = W.flop / (attn_ms * 1e-3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(W)
    bytes_in = sum(t.numel() * t.element_size() for n, t in W.host.items() if n not in resident)
    line = {
        "metric": METRIC, "value": round(tflops, 2), "unit": UNIT, "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": W.dtype, "data": "synthetic (seeded, BF16 inputs)",
        "config": W.config(world),
        "roofline": roofline(W, args, attn_ms, achieved),
        "e2e": {"value": round(world * W.flop / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                "h2d_bytes_per_step": bytes_in, "d2h_bytes_per_step": W.o.numel() * W.o.element_size(),
                "pipelined": "step i+1's H2D and step i's D2H run on their own streams, overlapping step i",
                "resident": list(resident), "steps": Ke},
        "gpu_launches": K * W.launches,
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(line), flush=True)
    teardown(world)


# DRAM bytes (read + write) of one attention launch from an ncu capture of the
# current kernel, per workload (None when not captured for it):
#   ncu --set full --clock-control none -k regex:attn_fwd -s 3 -c 1
#       python bench.py --workload W --steps 1 --warmup 3 --no-cpu-baseline
# The default S = 32768 launch is the S = 16384 capture times two (every tensor the
# launch moves doubles with S); profiles/attn_fwd_pv8_dram_traffic.md has the numbers.
TRAFFIC = {
    # ncu dram__bytes_read.sum + dram__bytes_write.sum of one attention launch (the first
    # timed one) of the current kernels, one-pass metrics on the full-size workload
    "dense_pv8_s32768": 847.64e6 + 315.26e6,
    "dense_pv8_s16384": 420.51e6 + 144.98e6,
    "dense_bf16_s16384": 504.63e6 + 148.48e6,
    "all_fp8_s8192": 201.43e6 + 103.67e6,
    "sage_s16384": 151.21e6 + 71.01e6,
    "sparse_paged_s16384": 1343.59e6 + 1041.93e6,
    "wide_qk_bf16_s16384": 673.46e6 + 160.15e6,
    "wide_qk_pv8_s16384": 587.59e6 + 153.48e6,
    "wide_qk_fp8_s16384": 336.24e6 + 143.42e6,
    "decode_paged_s16384": 69.26e6 + 1.02e6,  # the attention launch (the merge adds about 1 MB)
}


# ------------------------------------------------------------- reference ----
def oracle_sample(host, kind, B, Hq, Hkv, S, D, causal, rows):
    """The CPU oracle on a bounded sample: the workload's quantization of the
    sampled KV head (over all tokens) and float64 attention for `rows` query
    rows of query head 0 against all keys. Returns (seconds, useful FLOPs)."""
    from oracle import attention as oa
    from oracle import quant as oq

    t = time.perf_counter()
    if kind == "decode_paged":  # every batch, KV head 0 and its query heads, all (one) query rows
        G = Hq // Hkv
        pt = host["page_table"].numpy()
        k = oa.gather_paged(host["k_pool"][:, :, :1].to(torch.float64).numpy(), pt, S)
        v = oa.gather_paged(host["v_pool"][:, :, :1].to(torch.float64).numpy(), pt, S)
        q = host["q"][:, :, :G].to(torch.float64).numpy()
        mask = host["mask"][:, :1].numpy()
        t = time.perf_counter() - t
        t0 = time.perf_counter()
        oa.attention(q, k, v, 1.0 / math.sqrt(D), False, mask)
        dt = time.perf_counter() - t0 + t
        return dt, 4.0 * q.shape[0] * q.shape[1] * G * float(mask.sum()) / q.shape[0] * 128 * D
    if kind == "sparse_contig":
        k = host["k"][:1, :, :1].to(torch.float64).numpy()
        v = host["v"][:1, :, :1].to(torch.float64).numpy()
        q = host["q"][:1, :rows, :1].to(torch.float64).numpy()
        mask = host["mask"][:1, :1].numpy()
        mask = mask[:, :, : -(-rows // 128)]
    elif kind == "sparse_paged":
        pt = host["page_table"].numpy()[:1]
        k = oa.gather_paged(host["k_pool"][:, :, :1].to(torch.float64).numpy(), pt, S)
        v = oa.gather_paged(host["v_pool"][:, :, :1].to(torch.float64).numpy(), pt, S)
        q = host["q"][:1, :rows, :1].to(torch.float64).numpy()
        mask = host["mask"][:1, :1].numpy()
        mask = mask[:, :, : -(-rows // 128)]
    else:
        q32 = host["q"][:1, :rows, :1].to(torch.float32).numpy()
        k32 = host["k"][:1, :, :1].to(torch.float32).numpy()
        v32 = host["v"][:1, :, :1].to(torch.float32).numpy()
        spec = {"bf16": {}, "pv8": {"v": ("e4m3", "per_tensor", None)}, "pv8_o8": {"v": ("e4m3", "per_tensor", None)},
                "fp8": {n: ("e4m3", "per_head", None) for n in "qkv"},
                "sage": {"q": ("int8", "per_token_block", 128), "k": ("int8", "per_token_block", 64),
                         "v": ("e4m3", "per_channel", None)}}
        spec["wide_bf16"], spec["wide_pv8"], spec["wide_fp8"] = spec["bf16"], spec["pv8"], spec["fp8"]
        spec = spec[kind if kind != "sage_p2" else "sage"]
        ops = {"q": q32, "k": k32, "v": v32}
        for n, (dt, g, rpb) in spec.items():
            c, sc = oq.quantize_blockwise(ops[n], dt, g, rpb)
            ops[n] = oq.dequantize(c, sc, dt, g, rpb)
        q, k, v = (np.asarray(ops[n], dtype=np.float64) for n in "qkv")
        mask = None
    Sq = q.shape[1]
    if causal:  # the sampled rows are the first ones; keep their causal view of all keys
        k, v = k[:, :Sq], v[:, :Sq]
    oa.attention(q, k, v, 1.0 / math.sqrt(D), causal, mask)
    dt = time.perf_counter() - t
    dens = ((Sq + 1) / (2 * Sq)) if causal else (float(mask.sum()) * 128 * 128 / (Sq * S) if mask is not None else 1.0)
    keys = Sq if causal else S
    return dt, 2.0 * Sq * keys * (D + v.shape[3]) * min(1.0, dens)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count()


def cpu_baseline(W, rows=1024, target_s=20.0):
    """The oracle on a bounded sample: a 1024-row probe, then as many query rows (up
    to Sq) as the probe says fit in target_s seconds (larger samples run faster per
    row, so the second run takes about half of it: 10 s or so)."""
    dt, fl = oracle_sample(W.host, W.kind, W.B, W.Hq, W.Hkv, W.S, W.D, W.causal, rows)
    grow = min(W.host["q"].shape[1], int(rows * target_s / max(dt, 1e-3)) // 128 * 128)
    if grow > rows:
        rows = grow
        dt, fl = oracle_sample(W.host, W.kind, W.B, W.Hq, W.Hkv, W.S, W.D, W.causal, rows)
    return {"value": round(fl / dt / 1e12, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
            "sample": f"query head 0, rows 0..{rows - 1} against all keys (with the workload's quantization of "
                      f"that head), float64 NumPy, {dt:.1f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from precision_attention_fmha_b200 import workloads

    kind, B, Hq, Hkv, S, D, causal = WORKLOADS[args.workload]
    gen = {"bf16": lambda: dict(zip("qkv", workloads.normal_qkv(workloads.SEED_BASE + 1 + S, B, S, S, Hq, Hkv, D))),
           "pv8": lambda: workloads.dense_pv8(S=S, B=B, H=Hq, D=D),
           "pv8_o8": lambda: workloads.dense_pv8(S=S, B=B, H=Hq, D=D),
           "fp8": lambda: workloads.all_fp8(S=S, B=B, H=Hq, D=D),
           "sage": lambda: workloads.sage(S=S, B=B, H=Hq, D=D),
           "sage_p2": lambda: workloads.sage(S=S, B=B, H=Hq, D=D),
           "sparse_paged": lambda: workloads.sparse_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D),
           "sparse_contig": lambda: workloads.sparse_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D),
           "decode_paged": lambda: workloads.decode_paged(S=S, B=B, Hq=Hq, Hkv=Hkv, D=D),
           "wide_bf16": lambda: workloads.wide_qk(S=S, B=B, H=Hq, D=D),
           "wide_pv8": lambda: workloads.wide_qk(S=S, B=B, H=Hq, D=D),
           "wide_fp8": lambda: workloads.wide_qk(S=S, B=B, H=Hq, D=D, outliers=True)}[kind]
    host = gen()
    rows = 256
    for _ in range(args.warmup):
        oracle_sample(host, kind, B, Hq, Hkv, S, D, causal, rows)
    times, fl = [], 0
    for _ in range(args.steps):
        dt, fl = oracle_sample(host, kind, B, Hq, Hkv, S, D, causal, rows)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    val = fl / (ms * 1e-3) / 1e12
    sample = f"query head 0, rows 0..{rows - 1} against all keys, float64 NumPy oracle per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 6), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, BF16 inputs)",
        "config": {"workload": args.workload, "B": B, "Hq": Hq, "Hkv": Hkv, "Sq": S, "Skv": S, "D": D,
                   "causal": causal},
        "cpu_baseline": {"value": round(val, 6), "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(val, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


SMOOTH_METRIC = ("K smoothing GB/s (token mean per channel + INT8 quantization of K - mean: 4 B read + 1 B written "
                 "per element)")
QUANT_METRIC = "token-block quantization GB/s (INT8 codes of K, one scale per 64-token block: 2 B read + 1 B written per element)"


def run_smooth(args):
    """SageAttention K smoothing of the Sage workload's K (channel mean + shifted INT8
    quantizer), or the token-block quantizer alone (workload kind quant_k). HBM-bound."""
    from precision_attention_fmha_b200 import fmha, workloads

    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    kind, B, H, _, S, D, _ = WORKLOADS[args.workload]
    smooth = kind == "smooth_k"
    kh = workloads.sage(S=S, B=B, H=H, D=D)["k"].contiguous().pin_memory()
    k = kh.to(dev)
    mean = torch.empty((B, H, D), dtype=torch.float32, device=dev)
    mws = torch.empty(max(16, fmha.channel_mean_workspace_bytes(B, S, H, D)), dtype=torch.uint8, device=dev)
    codes = torch.empty(k.shape, dtype=torch.int8, device=dev)
    scales = torch.empty(fmha.scale_shape("per_token_block", B, S, H, D, 64), dtype=torch.float32, device=dev)

    def step(inp):
        if smooth:
            fmha.channel_mean(inp, out=mean, workspace=mws)
        fmha.fmha_quantize_blockwise(inp, torch.int8, "per_token_block", 64, out=codes, scales=scales,
                                     shift=mean if smooth else None)

    for _ in range(args.warmup):
        step(k)
    fmha.get_device_error()
    K_ = args.steps
    stream = torch.cuda.current_stream()
    fits_l2 = k.numel() * 2 <= L2_BYTES
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if fits_l2 else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    for i in range(K_):  # each step alone, L2 flushed before it when K fits there
        if flush is not None:
            flush.zero_()
        evs[i][0].record(stream)
        step(k)
        evs[i][1].record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in evs), world)
    # mean: K read once; quantizer: K read once, codes + scales written; mean written once
    outs = (codes, scales, mean) if smooth else (codes, scales)
    out_bytes = sum(t.numel() * t.element_size() for t in outs)
    algo = (2 if smooth else 1) * k.numel() * 2 + out_bytes
    _, hbm, src = load_peaks()
    gbs = algo / (ms * 1e-3) / 1e9
    oh = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in outs]
    Ke = max(1, min(K_, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(Ke):
        step(kh.to(dev, non_blocking=True))
        for h, d in zip(oh, outs):
            h.copy_(d, non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / Ke, world)
    fmha.get_device_error()
    line = {
        "metric": SMOOTH_METRIC if smooth else QUANT_METRIC,
        "value": round(world * gbs, 1), "unit": "GB/s", "n_gpus": world, "steps": K_, "warmup": args.warmup,
        "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16->int8", "data": "synthetic (seeded; the Sage workload's K, N(0,1) + per-channel N(0,2) bias)",
        "config": {"workload": args.workload, "B": B, "H": H, "S": S, "D": D, "k_scale": "per 64-token block",
                   "l2": "inputs fit in L2: flushed before each step (512 MiB write, outside the timed events)"
                   if fits_l2 else "inputs larger than L2",
                   "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": round(hbm, 1), "unit": "GB/s",
                     "frac": round(gbs / hbm, 4), "traffic": None, "peak_note": f"{src}: HBM copy bandwidth",
                     "algorithmic_bytes": int(algo),
                     "kernel": ("channel_mean_partial_kernel + channel_mean_final_kernel + quant_token_block_kernel"
                                if smooth else "quant_token_block_kernel"),
                     "kernel_ms": round(ms, 5)},
        "e2e": {"value": round(world * algo / (e2e_ms * 1e-3) / 1e9, 1), "unit": "GB/s",
                "h2d_bytes_per_step": k.numel() * 2, "d2h_bytes_per_step": out_bytes, "steps": Ke},
        "gpu_launches": (3 if smooth else 1) * K_,
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        dt, nbytes = smooth_oracle_sample(kh, heads=H, smooth=smooth)  # the whole K: well under a second
        line["cpu_baseline"] = {"value": round(nbytes / dt / 1e9, 6), "unit": "GB/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": f"all {H} heads, NumPy oracle, {dt:.2f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    teardown(world)


def smooth_oracle_sample(kh, heads, smooth=True):
    """The oracle's channel mean + shifted quantizer (or the quantizer alone) on the
    first `heads` heads: (seconds, algorithmic bytes)."""
    from oracle import quant as oq

    x = kh[:, :, :heads].to(torch.float32).numpy()
    t = time.perf_counter()
    mu = oq.channel_mean(x) if smooth else None
    oq.quantize_blockwise(x, "int8", "per_token_block", 64, shift=mu)
    dt = time.perf_counter() - t
    return dt, x.size * (5 if smooth else 3)


def run_reference_smooth(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from precision_attention_fmha_b200 import workloads

    kind, B, H, _, S, D, _ = WORKLOADS[args.workload]
    smooth = kind == "smooth_k"
    kh = workloads.sage(S=S, B=B, H=H, D=D)["k"].contiguous()
    heads = 2  # a bounded sample of the H heads per step
    for _ in range(args.warmup):
        smooth_oracle_sample(kh, heads, smooth)
    times, nbytes = [], 0
    for _ in range(args.steps):
        dt, nbytes = smooth_oracle_sample(kh, heads, smooth)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    val = nbytes / (ms * 1e-3) / 1e9
    print(json.dumps({
        "impl": "reference", "metric": SMOOTH_METRIC if smooth else QUANT_METRIC,
        "value": round(val, 6), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded; the Sage workload's K)",
        "config": {"workload": args.workload, "B": B, "H": H, "S": S, "D": D},
        "cpu_baseline": {"value": round(val, 6), "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"heads 0..{heads - 1} of {H} per step, NumPy oracle"},
        "e2e": {"value": round(val, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


def run_reference_nvfp4(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from oracle import nvfp4 as on
    _, _, _, _, T, K, _ = WORKLOADS[args.workload]
    rng = np.random.default_rng(1000 + 7 + T)
    n = 64  # rows per step: a bounded sample of the T tokens
    x = torch.from_numpy(rng.standard_normal((n, K), dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    for _ in range(args.warmup):
        on.quantize_per_token(x)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        on.quantize_per_token(x)
        times.append(time.perf_counter() - t)
    ms = 1e3 * sum(times) / len(times)
    val = n * K * 2.5625 / (ms * 1e-3) / 1e9
    print(json.dumps({
        "impl": "reference", "metric": "per-token NVFP4 quantization GB/s (2 B read + 0.5625 B written per element + 4 B per token)",
        "value": round(val, 6), "unit": "GB/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic (seeded N(0,1), BF16)",
        "config": {"workload": args.workload, "tokens": T, "K": K},
        "cpu_baseline": {"value": round(val, 6), "unit": "GB/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": f"{n} of {T} rows per step, NumPy oracle"},
        "e2e": {"value": round(val, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}), flush=True)


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
    kind = WORKLOADS[args.workload][0]
    if args.impl == "reference":
        {"nvfp4": run_reference_nvfp4, "smooth_k": run_reference_smooth,
         "quant_k": run_reference_smooth}.get(kind, run_reference)(args)
    else:
        {"nvfp4": run_nvfp4, "smooth_k": run_smooth, "quant_k": run_smooth}.get(kind, run_ours)(args)


if __name__ == "__main__":
    main()
