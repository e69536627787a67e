"""Benchmark of the fine-grained FP8 Linear hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload fprop]
                    [--impl ours|reference]

A step is one pass of the hot path over one batch of synthetic input on the
chosen workload.  The default is the largest configuration by FLOPs, the MoE
grouped Fprop: 16384 tokens X[16384,7168] in BF16, top-8 routing drawn from
a Zipf(1.1) law over 32 experts W_e[2048,7168]; one step is the 1x128
activation quantization, the FP8 dispatch of the token rows into
expert-contiguous groups padded to 128 rows, the 128x128 weight
quantization and the grouped block-scaled FP8 GEMM with FP32 promotion per
128-K block, BF16 output.  Other workloads (--workload fprop|dgrad|wgrad|
wgrad_pow2|pr1|...) run the other passes of the Linear the same way.

The metric is FP8 block-scaled GEMM throughput: 2*M*N*K algorithmic FLOPs
per step divided by the device time of the whole step (quantizers included),
as TFLOP/s summed over all ranks.  For N > 1 (torchrun) every rank runs an
independent replica of the workload (weak scaling: the path needs no
collective); time is the max over ranks.

The JSON line also carries
  roofline      the GEMM kernel's achieved TFLOP/s (CUDA events around its
                launches in the timed region) against the FP8 peak derived
                from the measured BF16 peak x 2 (nominal FP8/BF16 ratio):
                the burst figure when the sampled SM clock stayed at its
                maximum with no power-cap event, else the sustained one; the
                same rate also against the tensor cores' clock-scaled
                ceiling (148 SMs x 16384 FP8 FLOP/clk x sampled SM clock) and
                the 4.5 PFLOP/s dense FP8 specification; the quantizers'
                GB/s against the measured HBM copy bandwidth and the 8 TB/s
                specification;
  cpu_baseline  the CPU oracle timed on this host on a bounded sample of the
                same workload (rank 0, N = 1 only), extrapolated to a step;
  e2e           the same metric through the C ABI with the inputs copied from
                pinned host memory and the output copied back, every step; the
                copies overlap the compute of neighbouring steps (three CUDA
                streams, pipeline.HostPipeline);
  clocks        SM clock / throttle reasons sampled with nvidia-smi during the
                timed region.
`--impl reference` times the CPU oracle as it stands (the reference arm).
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------- peaks

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


SM_COUNT = 148
FP8_FLOP_PER_CLK_SM = 16384          # 8192 E4M3 multiply-adds per clock per SM
FP8_SPEC_TFLOPS = 4500.0             # dense FP8, B200 specification
HBM_SPEC_GBS = 8000.0


def gemm_roofline(gemm_tflops: float, clocks: dict, peaks: dict) -> dict:
    """The GEMM's rate against the FP8 peak that fits how it was timed.

    The FP8 peak is the measured BF16 cuBLAS peak x 2 (nominal FP8 : BF16).
    A short timed region that held the maximum SM clock with no power-cap
    event compares with the burst figure; a region that ran under the power
    cap (or whose clock was not sampled) with the sustained one."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    capped = "sw_power_cap" in clocks.get("reasons", [])
    burst = mhz is not None and mx is not None and mhz >= 0.97 * mx and not capped
    peak = 2.0 * (peaks["bf16"] if burst else peaks["bf16_sustained"])
    alt = 2.0 * (peaks["bf16_sustained"] if burst else peaks["bf16"])
    out = {"bound": "tensor", "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s",
           "frac": gemm_tflops / peak,
           "peak_source": (f"{peaks['source']} {'burst' if burst else 'sustained'} bf16 "
                           f"{peaks['bf16'] if burst else peaks['bf16_sustained']} TFLOP/s x 2 "
                           f"(FP8 : BF16 nominal 2 : 1), chosen because the sampled SM clock "
                           + ("stayed at its maximum with no power-cap event"
                              if burst else "fell below its maximum or a power-cap event was seen")),
           "frac_other_peak": gemm_tflops / alt,
           "frac_spec": gemm_tflops / FP8_SPEC_TFLOPS}
    if mhz:
        ceiling = SM_COUNT * FP8_FLOP_PER_CLK_SM * mhz * 1e6 / 1e12
        out.update(clock_ceiling=ceiling, frac_clock_ceiling=gemm_tflops / ceiling)
    return out


def targets(roof: dict, quant_gbs: float) -> dict:
    """The two targets of the path and the fraction each is measured against: the
    GEMM against the dense FP8 spec (4.5 PFLOP/s, >= 60 %), the quantizers
    against the HBM spec (8 TB/s, >= 75 %).  The measured-peak fractions in
    `roofline` and `quantizers` are the engineering view beside them."""
    g = roof["achieved"] / FP8_SPEC_TFLOPS
    q = quant_gbs / HBM_SPEC_GBS
    return {"gemm": {"measured_against": f"achieved / {FP8_SPEC_TFLOPS} TFLOP/s dense FP8 spec",
                     "frac": g, "threshold": 0.60, "met": g >= 0.60},
            "quantizers": {"measured_against": f"achieved / {HBM_SPEC_GBS} GB/s HBM spec",
                           "frac": q, "threshold": 0.75, "met": q >= 0.75}}


def run_config(desc: dict, world: int, host_inputs) -> dict:
    """The config object of the JSON line (both arms print the same one)."""
    cfg = dict(desc)
    in_bytes = sum(t.numel() * t.element_size() for t in host_inputs) if host_inputs else 0
    cfg.update(parallelism=f"replicas x{world}",
               l2="inputs larger than L2 (no flush)" if in_bytes > L2_BYTES
               else "inputs smaller than L2")
    return cfg


# ---------------------------------------------------------------- ncu traffic

KERNEL_SOURCES = {
    "k_fp8_gemm": ("fp8_fine_grained_x1_b200/csrc/gemm.cu",
                   "fp8_fine_grained_x1_b200/csrc/fp8fg_device.cuh"),
    "k_fp8_gemm_mx": ("fp8_fine_grained_x1_b200/csrc/gemm_mx.cu",
                      "fp8_fine_grained_x1_b200/csrc/fp8fg_device.cuh"),
}


def gemm_kernel(workload: str) -> str:
    """The GEMM kernel a workload's step launches."""
    return "k_fp8_gemm_mx" if workload.endswith("_tc") else "k_fp8_gemm"


def _code_only(text: str) -> str:
    """C/C++ source without comments, trailing blanks and empty lines, so
    that a comment edit does not invalidate a capture of the same code."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (re.sub(r"//.*$", "", ln).rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_source_hash(kernel: str = "k_fp8_gemm") -> str:
    """sha256 (first 16 hex digits) of the kernel's sources, comments removed."""
    import hashlib
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes (read + write) per GEMM launch from the committed ncu summary
    of this workload, if it was captured from the current kernel sources."""
    kernel = gemm_kernel(workload)
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    try:
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line and line.startswith("- "):
                    k, v = line[2:].split(":", 1)
                    fields[k.strip()] = v.strip().strip("`")
        if fields.get("kernel_source_sha256_16") != kernel_source_hash(kernel):
            return None
        return float(fields["traffic_bytes_per_launch"])
    except Exception:
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clocks / throttle reasons every 200 ms while active."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- workloads

def describe(workload):
    """CPU side of a workload: (wl, desc, (M, N, K), quant_bytes, host inputs,
    make) where make(device) builds the device step.  The reference arm uses
    the same desc, so both arms print the same config."""
    import torch
    from fp8_fine_grained_x1_b200 import SCALE_FP32, SCALE_POW2, linear, synth
    if workload in ("fprop", "fprop_pow2_tc"):
        wl = synth.fprop()
        tc = workload == "fprop_pow2_tc"
        M, K = wl["x"].shape
        N = wl["w"].shape[0]
        desc = dict(workload="fprop dense-MLP X[4096,7168] x W[18432,7168]^T, bf16 in, "
                    "1x128 act / 128x128 weight E4M3, bf16 out"
                    + (", pow2 scales applied in the tensor cores (UE8M0 block scaling)"
                       if tc else ""), M=M, N=N, K=K)
        inputs = [wl["x"], wl["w"]]
        quant_bytes = (M * K + N * K) * 3 + (M * K // 128) * 4 + (N * K // 16384) * 4

        def make(d):
            if tc:
                return linear.FpropStep(wl["x"].to(d), wl["w"].to(d), scale_mode=SCALE_POW2,
                                        tensor_core_scaling=True)
            return linear.FpropStep(wl["x"].to(d), wl["w"].to(d))
    elif workload == "pr1":
        wl = synth.pr1()
        M, K = wl["x"].shape
        N = wl["w"].shape[0]
        desc = dict(workload="pr1 tiny fprop X[128,512] x W[256,512]^T fp32 in, fp32 out",
                    M=M, N=N, K=K)
        inputs = [wl["x"], wl["w"]]
        quant_bytes = (M * K + N * K) * 5

        def make(d):
            return linear.FpropStep(wl["x"].to(d), wl["w"].to(d), out_dtype=torch.float32)
    elif workload == "dgrad":
        wl = synth.dgrad()
        M, K = wl["dy"].shape
        N = wl["w"].shape[1]
        desc = dict(workload="dgrad dX[4096,2048] = dY[4096,7168] . W[7168,2048] (W read "
                    "transposed), bf16 out", M=M, N=N, K=K)
        inputs = [wl["dy"], wl["w"]]
        quant_bytes = (M * K + K * N) * 3 + (M * K // 128) * 4

        def make(d):
            return linear.DgradStep(wl["dy"].to(d), wl["w"].to(d))
    elif workload in ("wgrad", "wgrad_pow2", "wgrad_pow2_tc"):
        wl = synth.wgrad()
        mode = SCALE_POW2 if workload.startswith("wgrad_pow2") else SCALE_FP32
        tc = workload == "wgrad_pow2_tc"
        T, C_in = wl["x"].shape
        C_out = wl["dy"].shape[1]
        M, N, K = C_out, C_in, T
        desc = dict(workload=f"wgrad dW[2048,7168] = dY^T . X over 8192 tokens, 128x1 "
                    f"groups, fp32 out, {'pow2' if mode else 'fp32'} scales"
                    + (", scaled in the tensor cores (UE8M0 block scaling)" if tc else ""),
                    M=M, N=N, K=K)
        inputs = [wl["x"], wl["dy"]]
        quant_bytes = (T * C_in + T * C_out) * 3 + (T // 128) * (C_in + C_out) * 4

        def make(d):
            return linear.WgradStep(wl["x"].to(d), wl["dy"].to(d), scale_mode=mode,
                                    tensor_core_scaling=tc)
    elif workload == "wgrad_cached":
        wl = synth.wgrad()
        T, C_in = wl["x"].shape
        C_out = wl["dy"].shape[1]
        M, N, K = C_out, C_in, T
        desc = dict(workload="wgrad dW[2048,7168] = dY^T . X over 8192 tokens, X from its "
                    "cached 1x128 FP8 form requantized to 128x1, dY quantized 128x1, fp32 out",
                    M=M, N=N, K=K)
        inputs = None
        # X: cache read and codes written, 1 + 4/128 B each way; dY: 3 + 4/128 B
        quant_bytes = T * C_in * 2 + 2 * (T // 128) * C_in * 4 + \
            T * C_out * 3 + (T // 128) * C_out * 4

        def make(d):
            import fp8_fine_grained_x1_b200 as fg
            # the forward pass's cache of X, made once outside the timed region
            qx, sx = fg.quant_act_1x128(wl["x"].to(d))
            return linear.WgradCachedStep(qx, sx, wl["dy"].to(d))
    elif workload in ("moe", "moe_pow2_tc"):
        wl = synth.moe()
        tc = workload == "moe_pow2_tc"
        lay = wl["layout"]
        topk = lay.topk.to(torch.int32)
        G, N, K = wl["w"].shape
        T = wl["x"].shape[0]
        M = int(lay.counts.sum())
        desc = dict(workload="moe grouped fprop, 32 experts W_e[2048,7168], 16384 tokens "
                    "top-8 Zipf(1.1): 1x128 quantize tokens straight into their 128-padded "
                    "expert groups, 128x128 quantize weights, grouped GEMM, bf16 out"
                    + (", pow2 scales applied in the tensor cores (UE8M0 block scaling)" if tc else ""),
                    M=M, N=N, K=K, M_padded=lay.m_total, tokens=T)
        inputs = [wl["x"], wl["w"], topk]
        # tokens read once (2 B) and quantized straight into their padded
        # expert rows (1 B code + 4/128 B scale per row element); weights
        # read (2 B) and written as codes (1 B)
        quant_bytes = (T * K * 2 + lay.m_total * K + lay.m_total * K // 32
                       + G * N * K * 3 + G * (N // 128) * (K // 128) * 4)

        def make(d):
            if tc:
                return linear.MoeStep(wl["x"].to(d), topk.to(d), wl["w"].to(d),
                                      scale_mode=SCALE_POW2, tensor_core_scaling=True)
            return linear.MoeStep(wl["x"].to(d), topk.to(d), wl["w"].to(d))
    else:
        raise SystemExit(f"unknown workload {workload}")
    return wl, desc, (M, N, K), quant_bytes, inputs, make


# ---------------------------------------------------------------- oracle (CPU) timing

def _bits(t):
    import torch
    from fp8_fine_grained_x1_b200 import synth
    return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


def oracle_sample(workload, budget_s: float = 20.0, described=None):
    """Time the CPU oracle on a bounded sample of the workload and extrapolate
    one step: each quantizer timed on a row (or token-block) sample, the GEMM
    on sampled outputs with the workload's K, layout and scale granularity."""
    import numpy as np
    import oracle
    from fp8_fine_grained_x1_b200 import SCALE_POW2
    oracle.build()
    wl, desc, (M, N, K), _, _, _ = described or describe(workload)
    rng = np.random.default_rng(0)
    mode = SCALE_POW2 if "pow2" in workload else oracle.SCALE_FP32
    gemm_kw = {}
    t0 = time.perf_counter()
    if workload in ("fprop", "fprop_pow2_tc", "pr1", "dgrad", "moe", "moe_pow2_tc"):
        xa = wl["dy"] if workload == "dgrad" else wl["x"]
        w = wl["w"].reshape(-1, wl["w"].shape[-1])
        ra, rw = min(64, xa.shape[0]), min(256, w.shape[0])
        qa, sa = oracle.quant_act_1x128(_bits(xa[:ra]), mode)
        qb, sb = oracle.quant_w_128x128(_bits(w[:rw]), mode)
        q_done, q_total = ra * xa.shape[1] + rw * w.shape[1], xa.numel() + w.numel()
        if workload == "dgrad":
            # W stored [K][N]: the sample keeps its first 256 K-rows, all N columns
            gemm_kw = dict(b_major=oracle.B_MNMAJOR)
            pts_k, m_hi, n_hi = rw, ra, qb.shape[1]
            qa = np.ascontiguousarray(qa[:, :rw])
            sa = np.ascontiguousarray(sa[:rw // 128])
        else:
            pts_k, m_hi, n_hi = K, ra, rw
    else:                                            # wgrad: 128x1 along 128 tokens
        x, dy = wl["x"][:128], wl["dy"][:128]
        if workload == "wgrad_cached":
            t_cache = time.perf_counter()
            cq, cs = oracle.quant_act_1x128(_bits(x), mode)     # the forward's cache: untimed
            t0 += time.perf_counter() - t_cache
            qb, sb = oracle.requant_1x128_to_128x1(cq, cs, mode)
        else:
            qb, sb = oracle.quant_act_128x1(_bits(x), mode)
        qa, sa = oracle.quant_act_128x1(_bits(dy), mode)
        q_done, q_total = x.numel() + dy.numel(), wl["x"].numel() + wl["dy"].numel()
        gemm_kw = dict(sb_gran=1)
        pts_k, m_hi, n_hi = 128, qa.shape[0], qb.shape[0]
    t_quant = time.perf_counter() - t0
    npts, t_gemm, done = 256, 0.0, 0
    while t_gemm < budget_s * 0.8 and done < 400000:
        pts = np.stack([rng.integers(0, m_hi, npts), rng.integers(0, n_hi, npts)], 1)
        t0 = time.perf_counter()
        oracle.gemm_points(qa, sa, qb, sb, pts, **gemm_kw)
        t_gemm += time.perf_counter() - t0
        done += npts
        npts = min(npts * 2, 65536)
    # an output's cost grows with K: scale the sampled K to the workload's
    per_point = t_gemm / done * (K / pts_k)
    step_s = per_point * M * N + t_quant / q_done * q_total
    flops = 2.0 * M * N * K
    return dict(value=flops / step_s / 1e12, unit="TFLOP/s", cores=oracle.num_threads(),
                kind="oracle",
                sample=f"{workload}: quantization of {q_done} of {q_total} elements and "
                       f"{done} GEMM outputs at K={pts_k} (FP64), extrapolated to one "
                       f"{M}x{N}x{K} step",
                step_s=step_s)


# ---------------------------------------------------------------- ranks

def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest per-rank value over all ranks: each replica's time counts,
    so the job's time is the slowest rank's (NCCL on the GPU, gloo on CPU)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank processes one step's work per step time."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


# ---------------------------------------------------------------- main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="moe",
                    choices=["fprop", "fprop_pow2_tc", "pr1", "dgrad", "wgrad", "wgrad_pow2",
                             "wgrad_pow2_tc", "wgrad_cached", "moe", "moe_pow2_tc"])
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return
        t0 = time.perf_counter()
        described = describe(args.workload)
        M, N, K = described[2]
        res = None
        vals = []
        for _ in range(max(1, args.steps)):
            res = oracle_sample(args.workload, budget_s=max(2.0, 60.0 / max(1, args.steps)),
                                described=described)
            vals.append(res["value"])
        total = time.perf_counter() - t0
        v = sorted(vals)[len(vals) // 2]
        line = {"impl": "reference", "metric": "FP8 block-scaled GEMM TFLOP/s (step incl. "
                "quantization)", "value": v, "unit": "TFLOP/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": 2.0 * M * N * K / (v * 1e12) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": run_config(described[1], args.gpus, described[4]),
                "timing": "the oracle on a bounded sample of the step, extrapolated to a "
                          "whole step (rank 0, host cores)",
                "ms_per_step_extrapolated": True,
                "cpu_baseline": dict({k: res[k] for k in ("unit", "cores", "kind", "sample")},
                                     value=v),
                "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "wall_s": total}
        print(json.dumps(line), flush=True)
        return

    import torch
    import torch.distributed as dist
    import fp8_fine_grained_x1_b200 as fg

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    fg.load_library()
    assert fg.fp8_device_supported(), "needs an sm_100 GPU"

    described = describe(args.workload)
    _, desc, (M_, N_, K_), quant_bytes, host_inputs, make = described
    step, flops = make(device), 2 * M_ * N_ * K_
    if host_inputs is None:          # inputs made on the device (e.g. a forward-pass cache)
        host_inputs = [t.cpu() for t in step.inputs]
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    status = fg.fp8_get_status()
    if status != fg.FP8_OK:
        raise SystemExit(f"device status after warm-up: {fg.status_string(status)}")

    # ---- timed region: K steps, GEMM launches bracketed by events
    ev_q0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_g0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev_g1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        time.sleep(0.3)
        start.record(stream)
        for i in range(args.steps):
            ev_q0[i].record(stream)
            step.quantize()
            ev_g0[i].record(stream)
            step.gemm()
            ev_g1[i].record(stream)
        stop.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = start.elapsed_time(stop)
    gemm_ms = sorted(ev_g0[i].elapsed_time(ev_g1[i]) for i in range(args.steps))
    quant_ms = sorted(ev_q0[i].elapsed_time(ev_g0[i]) for i in range(args.steps))
    gemm_avg = sum(gemm_ms) / len(gemm_ms)
    quant_avg = sum(quant_ms) / len(quant_ms)
    ms_total = max_over_ranks(ms_total, world, device)
    status = fg.fp8_get_status()
    if status != fg.FP8_OK:
        raise SystemExit(f"device status after timing: {fg.status_string(status)}")

    ms_per_step = ms_total / args.steps
    value = job_throughput(world, flops, ms_per_step)
    peaks = measured_peaks()
    clock_summary = clocks.summary()
    gemm_tflops = flops / (gemm_avg * 1e-3) / 1e12
    quant_gbs = quant_bytes / (quant_avg * 1e-3) / 1e9

    # ---- end to end through the C ABI: pinned host inputs in, output back.
    # Every step copies its inputs in and its result out; HostPipeline
    # overlaps batch i+1's copy-in and result i-1's copy-out with step i.
    e2e = None
    if args.e2e_steps > 0:
        from fp8_fine_grained_x1_b200.pipeline import HostPipeline
        pinned = [t.contiguous().pin_memory() for t in host_inputs]
        pipe = HostPipeline([step, make(device)], device)
        outs = [torch.empty(step.output.shape, dtype=step.output.dtype, pin_memory=True)
                for _ in range(2)]
        h2d = sum(t.numel() * t.element_size() for t in pinned)
        d2h = outs[0].numel() * outs[0].element_size()

        def batches(n):
            return [(pinned, outs[i % 2]) for i in range(n)]

        torch.cuda.synchronize()
        pipe.run(batches(2))
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(pipe.copy_in)
        pipe.run(batches(args.e2e_steps))
        e1.record(pipe.copy_out)
        torch.cuda.synchronize()
        e_ms = e0.elapsed_time(e1) / args.e2e_steps
        e_ms = max_over_ranks(e_ms, world, device)
        e2e = {"value": job_throughput(world, flops, e_ms), "unit": "TFLOP/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "overlap": "copy-in, compute and copy-out on three streams, two step copies"}
        status = fg.fp8_get_status()
        if status != fg.FP8_OK:
            raise SystemExit(f"device status after the end-to-end steps: {fg.status_string(status)}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res = oracle_sample(args.workload, described=described)
        cpu = {k: res[k] for k in ("value", "unit", "cores", "kind", "sample")}

    if rank == 0:
        cfg = run_config(desc, world, host_inputs)
        roof = gemm_roofline(gemm_tflops, clock_summary, peaks)
        traffic = profiled_traffic(args.workload)
        roof.update(traffic=traffic, kernel=gemm_kernel(args.workload),
                    traffic_source=("ncu dram__bytes_read.sum + dram__bytes_write.sum of one "
                                    "launch of the same kernel source on this workload, from "
                                    f"profiles/{gemm_kernel(args.workload)}_{args.workload}.md"
                                    if traffic is not None else
                                    "no ncu capture of the current kernel source"))
        line = {
            "metric": "FP8 block-scaled GEMM TFLOP/s (step incl. quantization)",
            "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "e4m3 x e4m3 -> f32",
            "data": "synthetic (seeded torch.Generator draws)", "config": cfg,
            "roofline": roof,
            "quantizers": {"achieved_gbs": quant_gbs, "peak_gbs": peaks["hbm"],
                           "frac": quant_gbs / peaks["hbm"],
                           "frac_spec": quant_gbs / HBM_SPEC_GBS, "ms_per_step": quant_avg,
                           "algorithmic_bytes": quant_bytes},
            "gemm_ms": gemm_avg, "gemm_ms_min": gemm_ms[0],
            "targets": targets(roof, quant_gbs),
            "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": step.kernel_calls * args.steps,
            "clocks": clock_summary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
