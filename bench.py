#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 linear hot path on B200.

One JSON line on stdout (rank 0).  Default workload: the MLP block at 32768 prefill
tokens (X BF16 [32768 x 5120] -> global scale -> NVFP4 quantise -> fused gate|up
GEMM [2 x 17408 rows, separate global scales] with SiLU*mul and NVFP4
re-quantisation in the epilogue -> down-projection GEMM [5120 x 17408] -> BF16).
Other workloads: ``--workload quantize|gdn|linear``.

Multi-GPU (torchrun): every rank runs the same workload on its own GPU with its own
inputs (independent token batches, weak scaling); no collective touches the data
path, a barrier brackets the timed region and the max time over ranks is reported.

``--impl reference`` times the CPU oracle (``oracle/``) on a bounded sample of the
same workload on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 W4A4 linear TFLOPS & % of B200 dense FP4 peak; quantise GB/s vs HBM"
FP4_OVER_BF16 = 4.0   # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------- helpers
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples of one GPU while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", self.gpu_id], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        mhz, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                mhz.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not mhz:
            return None
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(mhz)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


# --------------------------------------------------------------- workloads
class Workload:
    """Inputs resident on the device plus a ``step()`` that runs the hot path once."""
    name = ""
    unit = "TFLOP/s"

    def flops(self) -> float:
        return 0.0


def _dev_bits(bits):
    import numpy as np
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _gpu_student_t(rows, cols, seed, hot=8, hot_factor=100.0):
    """Student-t(3) activations generated on the device (seeded torch RNG), BF16.

    Same recipe as ``synth.student_t_activations`` (t = z / sqrt(chi2_3 / 3), 8 hot
    channels x100) but drawn with torch's generator: large tensors are generated in
    milliseconds on the GPU instead of seconds on the host.
    """
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    hot_idx = torch.randperm(cols, generator=g, device="cuda")[:hot]
    step = max(1, (1 << 25) // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        z = torch.randn((r1 - r0, cols), generator=g, device="cuda")
        chi = torch.randn((r1 - r0, cols, 3), generator=g, device="cuda").pow_(2).sum(-1).div_(3.0)
        t = z / chi.sqrt_()
        t[:, hot_idx] *= hot_factor
        out[r0:r1] = t.to(torch.bfloat16)
    return out


def _gpu_normal(rows, cols, seed, std):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    return (torch.randn((rows, cols), generator=g, device="cuda") * std).to(torch.bfloat16)


class MLPBlock(Workload):
    """MLP block, 32768 tokens: quantise X, gate|up GEMM + SiLU*mul + NVFP4 requant, down GEMM."""
    name = "mlp_block_m32768_h5120_i17408"

    def __init__(self, nv, M=32768, H=5120, I=17408, seed=0):
        import torch
        self.nv, self.M, self.H, self.I = nv, M, H, I
        self.x = _gpu_student_t(M, H, seed)
        wg = _gpu_normal(I, H, seed + 1, 0.02)
        wu = _gpu_normal(I, H, seed + 2, 0.04)
        self.w_gu, self.seg_gu = nv.quantize_fused([wg, wu])
        del wg, wu
        wd = _gpu_normal(H, I, seed + 3, 0.02)
        self.w_d = nv.quantize(wd)
        del wd
        dev = "cuda"
        self.gs_x = torch.empty(1, dtype=torch.float32, device=dev)
        self.xq_codes = torch.empty((M, H // 2), dtype=torch.uint8, device=dev)
        self.xq_scales = torch.empty(nv.scale_bytes(M, H), dtype=torch.uint8, device=dev)
        self.h_codes = torch.empty((M, I // 2), dtype=torch.uint8, device=dev)
        self.h_scales = torch.empty(nv.scale_bytes(M, I), dtype=torch.uint8, device=dev)
        self.out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        # static global scale of H (calibrated once from an unfused pass)
        nv.global_scale(self.x, out=self.gs_x)
        xq = nv.quantize(self.x, self.gs_x, codes=self.xq_codes, scales=self.xq_scales)
        h16 = nv.linear(xq, self.w_gu, segments=self.seg_gu, epilogue="silu_mul", out_dtype="bf16")
        self.gs_h = nv.global_scale(h16)
        del h16
        torch.cuda.synchronize()
        self.launches_per_step = 5  # amax, finalize, quantize, gate|up GEMM, down GEMM

    def flops(self):
        return 2.0 * self.M * (2 * self.I) * self.H + 2.0 * self.M * self.H * self.I

    def step(self, ev=None, x=None):
        nv = self.nv
        x = self.x if x is None else x
        nv.global_scale(x, out=self.gs_x)
        if ev: ev["q0"].record()
        xq = nv.quantize(x, self.gs_x, codes=self.xq_codes, scales=self.xq_scales)
        if ev: ev["q1"].record()
        hq = nv.linear(xq, self.w_gu, segments=self.seg_gu, epilogue="silu_mul", out_dtype="nvfp4",
                       gs_out=self.gs_h, out=self.h_codes, out_scales=self.h_scales)
        if ev: ev["g1"].record()
        nv.linear(hq, self.w_d, out_dtype="bf16", out=self.out)
        if ev: ev["g2"].record()
        return self.out

    def kernel_report(self, times_ms, peaks):
        q_bytes = self.M * self.H * 2.5625
        f_gu = 2.0 * self.M * (2 * self.I) * self.H
        f_d = 2.0 * self.M * self.H * self.I
        rep = {
            "quantize": {"ms": times_ms["quantize"], "GB/s": q_bytes / times_ms["quantize"] / 1e6},
            "gemm_gate_up_silu_requant": {"ms": times_ms["gemm1"], "TFLOP/s": f_gu / times_ms["gemm1"] / 1e9},
            "gemm_down": {"ms": times_ms["gemm2"], "TFLOP/s": f_d / times_ms["gemm2"] / 1e9},
        }
        rep["quantize"]["frac_hbm"] = rep["quantize"]["GB/s"] / peaks["hbm_gbs"]
        return rep


def run_ours(args, ws, rank):
    import torch
    import nvfp4_w4a4_quantized_02_b200 as nv
    from nvfp4_w4a4_quantized_02_b200 import build
    if rank == 0 or ws == 1:
        build.build()
    if ws > 1:
        torch.distributed.barrier()
    peaks, peak_src = load_peaks()
    wl = MLPBlock(nv)
    stream = torch.cuda.current_stream()

    # warm-up
    for _ in range(args.warmup):
        wl.step()
    torch.cuda.synchronize()

    evn = ["q0", "q1", "g1", "g2"]
    evs = [{k: torch.cuda.Event(enable_timing=True) for k in evn} for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    sampler = ClockSampler("GPU-" + str(props.uuid))
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    start.record(stream)
    for i in range(args.steps):
        wl.step(evs[i])
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    elapsed_ms = start.elapsed_time(stop)
    if ws > 1:
        t = torch.tensor([elapsed_ms], device="cuda")
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        elapsed_ms = float(t.item())
        torch.distributed.barrier()
    per = {"quantize": [], "gemm1": [], "gemm2": []}
    for e in evs:
        per["quantize"].append(e["q0"].elapsed_time(e["q1"]))
        per["gemm1"].append(e["q1"].elapsed_time(e["g1"]))
        per["gemm2"].append(e["g1"].elapsed_time(e["g2"]))
    times = {k: sum(v) / len(v) for k, v in per.items()}

    # end to end through the public API with host buffers
    e2e = run_e2e(wl, args, torch)

    ms = elapsed_ms / args.steps
    value = ws * wl.flops() / (ms * 1e-3) / 1e12
    rep = wl.kernel_report(times, peaks)
    fp4_peak = peaks["bf16_tflops_sustained"] * FP4_OVER_BF16
    g = rep["gemm_gate_up_silu_requant"]
    roof = {"kernel": "gemm_kernel (gate|up, SiLU*mul, NVFP4 requant epilogue)", "bound": "tensor",
            "achieved": g["TFLOP/s"], "peak": fp4_peak, "unit": "TFLOP/s", "frac": g["TFLOP/s"] / fp4_peak,
            "traffic": load_traffic("gemm_mlp_gate_up"),
            "peak_note": f"{peak_src} bf16_tflops_sustained x {FP4_OVER_BF16} (nominal FP4/BF16 ratio)"}
    for k in rep:
        if "TFLOP/s" in rep[k]:
            rep[k]["frac_fp4_peak"] = rep[k]["TFLOP/s"] / fp4_peak
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4(e2m1+e4m3)->fp32 acc", "data": "synthetic",
        "config": {"workload": wl.name, "M": wl.M, "hidden": wl.H, "intermediate": wl.I,
                   "step": "global_scale+quantize(X) -> gate|up GEMM (SiLU*mul, NVFP4 requant) -> down GEMM (BF16)",
                   "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
                   "l2": "inputs larger than L2 (X 335 MB, H 285 MB, out 335 MB per step)"},
        "roofline": roof, "kernels": rep, "e2e": e2e, "gpu_launches": wl.launches_per_step * args.steps,
        "clocks": clocks, "peaks_source": peak_src,
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args)
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(wl, args, torch):
    """Same step through the public API with host buffers: pinned H2D of X, the step, D2H of the output."""
    stream = torch.cuda.current_stream()
    x_host = wl.x.cpu().pin_memory()
    out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
    x_dev = torch.empty_like(wl.x)
    n = max(1, min(args.steps, 10))
    for _ in range(2):
        x_dev.copy_(x_host, non_blocking=True)
        out_host.copy_(wl.step(x=x_dev), non_blocking=True)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(n):
        x_dev.copy_(x_host, non_blocking=True)
        out_host.copy_(wl.step(x=x_dev), non_blocking=True)
    e.record(stream)
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    return {"value": round(wl.flops() / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "h2d_bytes_per_step": x_host.numel() * 2, "d2h_bytes_per_step": out_host.numel() * 2,
            "ms_per_step": round(ms, 4), "steps": n}


def load_traffic(key):
    """DRAM bytes per launch from the committed ncu summary, if it matches the current kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        h = hashlib.sha256()
        for fn in sorted(os.listdir(os.path.join(ROOT, "nvfp4_w4a4_quantized_02_b200", "csrc"))):
            with open(os.path.join(ROOT, "nvfp4_w4a4_quantized_02_b200", "csrc", fn), "rb") as f:
                h.update(f.read())
        ent = d.get(key)
        if ent and ent.get("csrc_sha256") == h.hexdigest():
            return ent["bytes_per_launch"]
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- CPU oracle
def cpu_sample_step(rows=32, cols_h=256, K=5120):
    """The MLP block restated by the oracle on a bounded sample: ``rows`` token rows, a
    slice of ``cols_h`` intermediate channels (gate and up), K=5120 in, the down
    projection over those channels for all 5120 outputs.  Returns (flops, seconds)."""
    import numpy as np
    import oracle
    import synth
    x = synth.bf16_to_f32(synth.student_t_activations(rows, K, seed=0))
    wg = synth.bf16_to_f32(synth.gaussian_weights(cols_h, K, seed=1, std=0.02))
    wu = synth.bf16_to_f32(synth.gaussian_weights(cols_h, K, seed=2, std=0.04))
    wd = synth.bf16_to_f32(synth.gaussian_weights(5120, cols_h, seed=3, std=0.02))
    gsg, gsu, gsd = oracle.global_scale(wg), oracle.global_scale(wu), oracle.global_scale(wd)
    cg, sg = oracle.quantize(wg, gsg)
    cu, su = oracle.quantize(wu, gsu)
    cd, sd = oracle.quantize(wd, gsd)
    t0 = time.perf_counter()
    gsx = oracle.global_scale(x)
    cx, sx = oracle.quantize(x, gsx)
    y = oracle.linear(cx, sx, gsx, np.concatenate([cg, cu]), np.concatenate([sg, su]),
                      [(0, cols_h, gsg), (cols_h, 2 * cols_h, gsu)])
    h = oracle.round_to_bf16(oracle.silu_mul(y[:, :cols_h], y[:, cols_h:])).astype(np.float32)
    gsh = oracle.global_scale(h)
    ch, sh = oracle.quantize(h, gsh)
    oracle.linear(ch, sh, gsh, cd, sd, [(0, 5120, gsd)])
    dt = time.perf_counter() - t0
    flops = 2.0 * rows * 2 * cols_h * K + 2.0 * rows * 5120 * cols_h
    return flops, dt


def cpu_baseline(args, budget_s=12.0):
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    flops, secs, n = 0.0, 0.0, 0
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or n == 0:
        f, s = cpu_sample_step()
        flops += f
        secs += s
        n += 1
    return {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} x MLP-block sample (32 token rows, 256 intermediate channels, K=5120; "
                      "global scale + quantise + gate|up + SiLU*mul + requant + down); numpy FP64 oracle"}


def run_reference(args, ws, rank):
    if rank != 0:
        return
    t0 = time.perf_counter()
    for _ in range(args.warmup):
        cpu_sample_step()
    flops, secs = 0.0, 0.0
    for _ in range(args.steps):
        f, s = cpu_sample_step()
        flops += f
        secs += s
    value = flops / secs / 1e12
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic",
            "config": {"workload": MLPBlock.name, "sample": "32 rows x 256 intermediate channels per step"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                             "sample": "MLP-block sample per step (32 rows, 256 channels, K=5120)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 2)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    ws, rank, local = dist_env()
    if args.impl == "reference":
        run_reference(args, ws, rank)
        return
    import torch
    torch.cuda.set_device(local)
    if ws > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        run_ours(args, ws, rank)
    finally:
        if ws > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
