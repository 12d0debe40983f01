#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 linear hot path on B200.

One JSON line on stdout (rank 0).  Workloads (``--workload``):

* ``mlp`` (default): the MLP block at 32768 prefill tokens.  X BF16 [32768 x 5120]
  -> global scale -> NVFP4 quantise -> fused gate|up GEMM [2 x 17408 rows, separate
  global scales] with SiLU*mul and NVFP4 re-quantisation in the epilogue ->
  down-projection GEMM [5120 x 17408] -> BF16.
* ``quantize``: activation quantisation of X BF16 [32768 x 5120] (Student-t, 8 hot
  channels) with a static global scale -> packed E2M1 + swizzled E4M3 scales.
* ``gdn``: GDN fused input projection, X [8192 x 5120] -> one NVFP4 GEMM over
  q|k|v|z|beta|alpha (12352 rows, six global scales) with the gate epilogue.
* ``linear``: the small single linear, X [128 x 1024] x W [1024 x 1024]^T.
* ``sweep``: all 496 linears of the 64-layer hybrid model (48 GDN layers x 2 GEMMs,
  16 attention layers x 2 GEMMs with q|k|v fused, 64 MLPs x 2 GEMMs with gate|up
  fused), each fed by the NVFP4 quantiser, at ``--M`` prefill tokens.
* ``decode``: the same 496 linears for one decode step of ``--M`` (default 32)
  sequences through the split-K linear (weight-bandwidth bound).
* ``kv``: the FP8 KV-cache write of one attention layer's K and V at ``--M`` prefill
  tokens (static per-tensor scales, paged slots).
* ``gdn_rec``: the gated delta-rule recurrence of one GDN layer over ``--M`` prefill
  tokens (sequences of 4096; 16 key / 32 value heads of 128, FP32 state), consuming
  q|k|v rows and the gate epilogue's g / beta; FP32-ALU bound.
* ``gdn_decode``: one decode step of that recurrence for ``--M`` (default 32)
  sequences over their carried states; bound by the state's HBM traffic.

Multi-GPU (torchrun): every rank runs the same workload on its own GPU with its own
inputs (independent token batches, weak scaling); no collective touches the data
path, a barrier brackets the timed region and the max time over ranks is reported.

``--impl reference`` times the CPU oracle (``oracle/``) on a bounded sample of the
same workload on the host cores, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
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
NOMINAL_FP4_TFLOPS = 9000.0  # datasheet dense NVFP4 tensor peak of one B200
NOMINAL_HBM_GBS = 8000.0     # datasheet HBM3e bandwidth of one B200 (~8 TB/s)
# TMA operand bytes one K stage of a 256 x 256 CTA-pair tile brings from L2 into the pair's
# shared memory: per CTA 128 A rows and 128 B rows of 128 bytes (256 FP4), A's scale atoms
# (2 KB) and both halves of B's (4 KB).  At full occupancy the pair GEMM is bound by this
# stream (~12 TB/s measured by timing it on fewer clusters).
PAIR_STAGE_L2_BYTES = 2 * (128 * 128 + 128 * 128 + 2048 + 4096)
SUSTAINED_REGION_MS = 1000.0  # timed regions at least this long use the sustained GEMM peak
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP32_LANES_PER_SM = 128     # FP32 FMA lanes per SM (4 sub-partitions x 32)
SM_MAX_MHZ = 1965.0         # clocks.max.sm of the B200
L2_FLUSH_BYTES = 256 << 20   # > 126 MB L2


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


def max_over_ranks(value: float, device) -> float:
    """Largest ``value`` over the ranks of the default process group (the job's time
    is the slowest rank's)."""
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sources_hash(files):
    h = hashlib.sha256()
    d = os.path.join(ROOT, "nvfp4_w4a4_quantized_02_b200", "csrc")
    for fn in files:
        with open(os.path.join(d, fn), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def pair_gemm_l2_bytes(M, N, K):
    """L2 -> SM operand bytes of one CTA-pair GEMM launch (M > 128, N and K multiples of
    256): tiles x K stages x PAIR_STAGE_L2_BYTES."""
    return -(-M // 256) * (N // 256) * (K // 256) * PAIR_STAGE_L2_BYTES


def load_traffic(key):
    """DRAM bytes per launch of ``key`` (``kernel@workload``) from the committed ncu
    summary ``profiles/traffic.json``, or None when the kernel's sources (the device
    code files listed with the entry) changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            ent = json.load(f).get(key)
        if ent and ent.get("csrc_sha256") == sources_hash(ent["sources"]):
            return ent["bytes_per_launch"]
    except Exception:
        pass
    return None


class KernelTimer:
    """CUDA events around individual launches on the launching (current) stream.

    ``with tm("key"):`` brackets one launch; ``summary()`` gives per key the number
    of launches and their summed / average duration over all recorded steps.
    """

    def __init__(self, torch):
        self.torch = torch
        self.recs = []

    def __call__(self, key):
        return _KernelSpan(self, key)

    def summary(self):
        out = {}
        for key, e0, e1 in self.recs:
            d = out.setdefault(key, {"launches": 0, "ms_total": 0.0})
            d["launches"] += 1
            d["ms_total"] += e0.elapsed_time(e1)
        for d in out.values():
            d["ms_avg"] = d["ms_total"] / d["launches"]
        return out


class _KernelSpan:
    def __init__(self, tm, key):
        self.tm, self.key = tm, key

    def __enter__(self):
        ev = self.tm.torch.cuda.Event
        self.e0, self.e1 = ev(enable_timing=True), ev(enable_timing=True)
        self.e0.record()

    def __exit__(self, *exc):
        self.e1.record()
        self.tm.recs.append((self.key, self.e0, self.e1))
        return False


class _NoTimer:
    def __call__(self, key):
        return self

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


NO_TIMER = _NoTimer()


# --------------------------------------------------------- synthetic inputs
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


def _gpu_outliers(rows, cols, seed, frac=1e-3, factor=50.0):
    """N(0,1) activations with ``frac`` of the entries (seeded permutation) x ``factor``, BF16."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn((rows, cols), generator=g, device="cuda")
    n = int(round(frac * rows * cols))
    if n:
        idx = torch.randperm(rows * cols, generator=g, device="cuda")[:n]
        x.view(-1)[idx] *= factor
    return x.to(torch.bfloat16)


def _gpu_normal(rows, cols, seed, std):
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    step = max(1, (1 << 27) // cols)
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = (torch.randn((r1 - r0, cols), generator=g, device="cuda") * std).to(torch.bfloat16)
    return out


GDN_SEGMENTS = (("q", 2048, 1.0), ("k", 2048, 2.0), ("v", 4096, 4.0), ("z", 4096, 8.0),
                ("beta", 32, 16.0), ("alpha", 32, 1.0))


def _gdn_weight(nv, K, seed):
    """Fused GDN in-projection weight q|k|v|z|beta|alpha, each segment its own global scale."""
    parts = [_gpu_normal(n, K, seed + i, 0.02 * m) for i, (_, n, m) in enumerate(GDN_SEGMENTS)]
    w, segs = nv.quantize_fused(parts)
    del parts
    return w, segs


def _gdn_gate_tensors(torch, M, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    a_log = torch.randn(32, generator=g, device="cuda")
    dt_bias = torch.randn(32, generator=g, device="cuda")
    beta = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    gate = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    n = sum(n for _, n, _ in GDN_SEGMENTS)
    return dict(beta_begin=n - 64, alpha_begin=n - 32, n_heads=32, A_log=a_log, dt_bias=dt_bias,
                beta_out=beta, g_out=gate)


def _gpu_gdn_rec_inputs(M, seq_len, seed, hk=16, hv=32, d=128):
    """GDN recurrence inputs on the device, same recipe as ``synth.gdn_recurrence_inputs``
    (unit-norm q / k heads in BF16, v ~ N(0,1) BF16, g = -c_h U(0.5, 1.5) with c_h
    log-uniform in [2e-5, 0.5], beta ~ U(0.05, 1)), drawn with torch's generator.
    Rows are q | k | v (width 2 hk d + hv d)."""
    import math
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    wk, wv = hk * d, hv * d
    rows = torch.empty((M, 2 * wk + wv), dtype=torch.bfloat16, device="cuda")
    for c in (0, wk):
        x = torch.randn((M, hk, d), generator=g, device="cuda")
        rows[:, c:c + wk] = (x / x.norm(dim=-1, keepdim=True)).reshape(M, wk).to(torch.bfloat16)
    rows[:, 2 * wk:] = torch.randn((M, wv), generator=g, device="cuda").to(torch.bfloat16)
    lo, hi = math.log(2e-5), math.log(0.5)
    rate = torch.exp(lo + (hi - lo) * torch.rand(hv, generator=g, device="cuda"))
    gate = -rate[None, :] * (0.5 + torch.rand((M, hv), generator=g, device="cuda"))
    beta = 0.05 + 0.95 * torch.rand((M, hv), generator=g, device="cuda")
    n = (M + seq_len - 1) // seq_len
    cu = torch.tensor([min(i * seq_len, M) for i in range(n + 1)], dtype=torch.int32, device="cuda")
    return rows, gate.contiguous(), beta.contiguous(), cu


# --------------------------------------------------------------- workloads
class Workload:
    """Inputs resident on the device plus a ``step(tm)`` that runs the hot path once.

    ``unit``: "TFLOP/s" or "GB/s"; ``work()``: FLOPs or bytes per step (the
    algorithmic count); ``dominant``: (timer key, work per launch, bound, label).
    """
    name = ""
    unit = "TFLOP/s"
    flush_l2 = False
    l2_note = ""
    launches_per_step = 0
    x = None      # the step's input (refreshed from host memory in the e2e run)
    out = None    # the step's result (read back in the e2e run)

    def work(self) -> float:
        raise NotImplementedError

    def config(self) -> dict:
        return {}

    def cpu_sample(self):
        """One bounded CPU-oracle sample of this workload: (work in the metric's base unit, seconds)."""
        raise NotImplementedError

    cpu_sample_note = ""
    use_graph = False  # replay the step as a CUDA graph (launch-bound workloads)
    dtype = None       # arithmetic type label (default: by unit)

    def plan(self, x):
        """The step as a list of (phase, launch) pairs; every launch writes preallocated buffers."""
        raise NotImplementedError

    def step(self, tm=NO_TIMER, x=None):
        for phase, launch in self.plan(self.x if x is None else x):
            with tm(phase):
                launch()
        return self.out


class MLPBlock(Workload):
    """MLP block: quantise X, gate|up GEMM + SiLU*mul + NVFP4 requant, down GEMM."""

    def __init__(self, nv, M=32768, H=5120, I=17408, seed=0):
        import torch
        self.nv, self.M, self.H, self.I = nv, M, H, I
        self.name = f"mlp_block_m{M}_h{H}_i{I}"
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
        self.f_gu = 2.0 * M * (2 * I) * H
        self.f_d = 2.0 * M * H * I
        self.l2_note = (f"inputs larger than L2 (X {M * H * 2 / 1e6:.0f} MB, H {M * I * 0.5625 / 1e6:.0f} MB, "
                        f"out {M * H * 2 / 1e6:.0f} MB per step)")
        self.dominant = ("gemm_gate_up", self.f_gu, "tensor",
                         "gemm2_kernel (CTA pair; gate|up, SiLU*mul, NVFP4 requant epilogue)")
        self.phases = {"global_scale": ("GB/s", 2.0 * M * H), "quantize": ("GB/s", 2.5625 * M * H),
                       "gemm_gate_up": ("TFLOP/s", self.f_gu), "gemm_down": ("TFLOP/s", self.f_d)}
        if M > 128:  # CTA-pair kernels: their L2 -> SM operand stream
            self.l2_stream = {"gemm_gate_up": pair_gemm_l2_bytes(M, 2 * I, H),
                              "gemm_down": pair_gemm_l2_bytes(M, H, I)}

    def work(self):
        return self.f_gu + self.f_d

    def config(self):
        return {"M": self.M, "hidden": self.H, "intermediate": self.I,
                "step": "global_scale+quantize(X) -> gate|up GEMM (SiLU*mul, NVFP4 requant) -> down GEMM (BF16)"}

    def plan(self, x):
        nv = self.nv
        xq = nv.NVFP4Tensor(self.xq_codes, self.xq_scales, self.gs_x, self.M, self.H)
        hq = nv.NVFP4Tensor(self.h_codes, self.h_scales, self.gs_h, self.M, self.I)
        return [
            ("global_scale", lambda: nv.global_scale(x, out=self.gs_x)),
            ("quantize", lambda: nv.quantize(x, self.gs_x, codes=self.xq_codes, scales=self.xq_scales)),
            ("gemm_gate_up", lambda: nv.linear(xq, self.w_gu, segments=self.seg_gu, epilogue="silu_mul",
                                               out_dtype="nvfp4", gs_out=self.gs_h, out=self.h_codes,
                                               out_scales=self.h_scales)),
            ("gemm_down", lambda: nv.linear(hq, self.w_d, out_dtype="bf16", out=self.out)),
        ]

    cpu_sample_note = ("MLP-block sample (32 token rows, 256 intermediate channels, K=5120; global scale + "
                       "quantise + gate|up + SiLU*mul + requant + down); numpy FP64 oracle")

    def cpu_sample(self):
        return cpu_mlp_sample()


class QuantizeOnly(Workload):
    """Activation quantisation with a static (calibrated) global scale."""
    unit = "GB/s"

    def __init__(self, nv, M=32768, K=5120, seed=0):
        import torch
        self.nv, self.M, self.K = nv, M, K
        self.name = f"quantize_m{M}_k{K}"
        self.x = _gpu_student_t(M, K, seed)
        self.gs = nv.global_scale(self.x)
        self.gs_dyn = torch.empty(1, dtype=torch.float32, device="cuda")
        self.codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        self.scales = torch.empty(nv.scale_bytes(M, K), dtype=torch.uint8, device="cuda")
        self.out = self.codes
        self.launches_per_step = 1
        self.bytes = 2.5625 * M * K
        self.l2_note = f"input larger than L2 (X {M * K * 2 / 1e6:.0f} MB)"
        self.dominant = ("quantize", self.bytes, "hbm", "quantize_kernel (static global scale)")
        self.phases = {"quantize": ("GB/s", self.bytes)}
        torch.cuda.synchronize()

    def work(self):
        return self.bytes

    def config(self):
        return {"M": self.M, "K": self.K, "gs": "static (calibrated once from amax)",
                "bytes_per_element": 2.5625}

    def plan(self, x):
        return [("quantize", lambda: self.nv.quantize(x, self.gs, codes=self.codes, scales=self.scales))]

    def extra(self, torch):
        """Dynamic mode (amax pass + finalize + quantise), timed separately after the main region."""
        nv = self.nv
        for _ in range(3):
            nv.global_scale(self.x, out=self.gs_dyn)
            nv.quantize(self.x, self.gs_dyn, codes=self.codes, scales=self.scales)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 10
        s.record()
        for _ in range(n):
            nv.global_scale(self.x, out=self.gs_dyn)
            nv.quantize(self.x, self.gs_dyn, codes=self.codes, scales=self.scales)
        e.record()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / n
        b = 4.5625 * self.M * self.K
        return {"dynamic_gs": {"ms": ms, "GB/s": b / ms / 1e6, "bytes_per_element": 4.5625}}

    cpu_sample_note = "quantise of 64 rows x 5120 (Student-t, static gs); numpy oracle"

    def cpu_sample(self):
        import oracle
        import synth
        x = synth.bf16_to_f32(synth.student_t_activations(64, self.K, seed=0))
        gs = oracle.global_scale(x)
        t0 = time.perf_counter()
        oracle.quantize(x, gs)
        return 2.5625 * x.size, time.perf_counter() - t0


class GDNInProj(Workload):
    """GDN fused input projection: quantise X, one GEMM over six segments + gate epilogue."""

    def __init__(self, nv, M=8192, K=5120, seed=0):
        import torch
        self.nv, self.M, self.K = nv, M, K
        self.N = sum(n for _, n, _ in GDN_SEGMENTS)
        self.name = f"gdn_inproj_m{M}_n{self.N}_k{K}"
        self.x = _gpu_outliers(M, K, seed)
        self.w, self.segs = _gdn_weight(nv, K, seed + 1)
        self.gates = _gdn_gate_tensors(torch, M, seed + 100)
        self.gs_x = torch.empty(1, dtype=torch.float32, device="cuda")
        self.xq_codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        self.xq_scales = torch.empty(nv.scale_bytes(M, K), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((M, self.N), dtype=torch.bfloat16, device="cuda")
        self.flops = 2.0 * M * self.N * K
        self.launches_per_step = 4
        self.l2_note = (f"per-step working set {(M * K * 2.5625 + self.N * K * 0.5625 + M * self.N * 2) / 1e6:.0f} MB "
                        "> L2 (X, its codes, W, BF16 out)")
        self.dominant = ("gemm", self.flops, "tensor", "gemm2_kernel (CTA pair; 6 segments, GDN gate epilogue)")
        self.phases = {"global_scale": ("GB/s", 2.0 * M * K), "quantize": ("GB/s", 2.5625 * M * K),
                       "gemm": ("TFLOP/s", self.flops)}
        torch.cuda.synchronize()

    def work(self):
        return self.flops

    def config(self):
        return {"M": self.M, "N": self.N, "K": self.K,
                "segments": "q 2048 | k 2048 | v 4096 | z 4096 | beta 32 | alpha 32",
                "step": "global_scale+quantize(X) -> fused GEMM (per-segment alpha, sigmoid beta, "
                        "-exp(A_log)*softplus(a+dt_bias)) -> BF16 + FP32 gates"}

    def plan(self, x):
        nv = self.nv
        xq = nv.NVFP4Tensor(self.xq_codes, self.xq_scales, self.gs_x, self.M, self.K)
        return [
            ("global_scale", lambda: nv.global_scale(x, out=self.gs_x)),
            ("quantize", lambda: nv.quantize(x, self.gs_x, codes=self.xq_codes, scales=self.xq_scales)),
            ("gemm", lambda: nv.linear(xq, self.w, segments=self.segs, epilogue="gdn_gates", gates=self.gates,
                                       out_dtype="bf16", out=self.out)),
        ]

    def extra(self, torch):
        """The pages' offline repair of the same fused weight (nvfp4_fold_segments on a copy of
        its scale buffer), timed separately: a pass over the 3.9 MB scale buffer."""
        nv = self.nv
        w = nv.NVFP4Tensor(self.w.codes, self.w.scales.clone(), self.w.gs, self.w.rows, self.w.cols)
        gs_c = torch.empty(1, dtype=torch.float32, device="cuda")
        for _ in range(3):
            w.scales.copy_(self.w.scales)
            nv.fold_segments(w, self.segs, gs_out=gs_c)
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = 20
        ms = 0.0
        for _ in range(n):
            w.scales.copy_(self.w.scales)
            s.record()
            nv.fold_segments(w, self.segs, gs_out=gs_c)
            e.record()
            torch.cuda.synchronize()
            ms += s.elapsed_time(e)
        ms /= n
        b = 2.0 * w.scales.numel()
        return {"fold_segments": {"ms": round(ms, 5), "GB/s": round(b / ms / 1e6, 1), "bytes": b}}

    cpu_sample_note = ("GDN in-proj sample: 32 token rows x 320 weight rows (64 each of q/k/v/z + 32 beta + "
                       "32 alpha), K=5120; quantise X + fused linear + gates; numpy FP64 oracle")

    def cpu_sample(self):
        return cpu_gdn_sample(self.K)


class SmallLinear(Workload):
    """Single small W4A4 linear (dynamic activation scale): launch-latency bound."""
    flush_l2 = True

    def __init__(self, nv, M=128, N=1024, K=1024, seed=0):
        import torch
        self.nv, self.M, self.N, self.K = nv, M, N, K
        self.name = f"linear_m{M}_n{N}_k{K}"
        self.x = _gpu_outliers(M, K, seed)
        self.w = nv.quantize(_gpu_normal(N, K, seed + 1, 0.02))
        self.gs_x = torch.empty(1, dtype=torch.float32, device="cuda")
        self.xq_codes = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
        self.xq_scales = torch.empty(nv.scale_bytes(M, K), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        self.flops = 2.0 * M * N * K
        self.launches_per_step = 4
        self.l2_note = "L2 flushed (256 MB write) between timed steps; per-step device time summed"
        self.dominant = ("gemm", self.flops, "tensor", "gemm_kernel (1 segment, BF16 out)")
        self.phases = {"global_scale": ("GB/s", 2.0 * M * K), "quantize": ("GB/s", 2.5625 * M * K),
                       "gemm": ("TFLOP/s", self.flops)}
        torch.cuda.synchronize()

    def work(self):
        return self.flops

    def config(self):
        return {"M": self.M, "N": self.N, "K": self.K,
                "step": "global_scale+quantize(X) -> GEMM -> BF16"}

    def plan(self, x):
        nv = self.nv
        xq = nv.NVFP4Tensor(self.xq_codes, self.xq_scales, self.gs_x, self.M, self.K)
        return [
            ("global_scale", lambda: nv.global_scale(x, out=self.gs_x)),
            ("quantize", lambda: nv.quantize(x, self.gs_x, codes=self.xq_codes, scales=self.xq_scales)),
            ("gemm", lambda: nv.linear(xq, self.w, out_dtype="bf16", out=self.out)),
        ]

    cpu_sample_note = "the whole linear (128 x 1024 x 1024): quantise X + dequantise-then-FP64 matmul"

    def cpu_sample(self):
        import oracle
        import synth
        x = synth.bf16_to_f32(synth.outlier_activations(self.M, self.K, seed=0))
        w = synth.bf16_to_f32(synth.gaussian_weights(self.N, self.K, seed=1))
        gw = oracle.global_scale(w)
        cw, sw = oracle.quantize(w, gw)
        t0 = time.perf_counter()
        gx = oracle.global_scale(x)
        cx, sx = oracle.quantize(x, gx)
        oracle.linear(cx, sx, gx, cw, sw, [(0, self.N, gw)])
        return self.flops, time.perf_counter() - t0


class HybridSweep(Workload):
    """The 496 linears of the 64-layer hybrid model, each fed by the NVFP4 quantiser.

    Layers 4j..4j+2 are GDN, 4j+3 attention (48 + 16); every layer has an MLP.
    GDN: in-proj 5120 -> 12352 (q|k|v|z|beta|alpha, gate epilogue) + out 4096 -> 5120.
    Attention: q|k|v 5120 -> 6144|1024|1024 fused + o 6144 -> 5120.
    MLP: gate|up 5120 -> 2 x 17408 (SiLU*mul, NVFP4 requant) + down 17408 -> 5120.
    Linear count: 48 x 5 + 16 x 4 + 64 x 3 = 496 (fused GEMMs count their modules).
    The inputs of the out / o projections stand in for the mixer outputs (the mixers
    themselves are not linears): fixed Student-t tensors of width 4096 / 6144.
    """

    def __init__(self, nv, M=32768, seed=0, layers=64):
        import torch
        self.nv, self.M = nv, M
        self.n_layers = layers
        self.n_gdn = sum(1 for li in range(layers) if li % 4 != 3)
        self.n_attn = layers - self.n_gdn
        self.n_linears = 5 * self.n_gdn + 4 * self.n_attn + 3 * layers
        self.name = (f"hybrid_sweep_496_linears_m{M}" if layers == 64
                     else f"hybrid_sweep_{self.n_linears}_linears_{layers}_layers_m{M}")
        H, I = 5120, 17408
        dev = "cuda"
        # activations per distinct input width, each with a static calibrated global scale
        self.x = _gpu_student_t(M, H, seed)
        self.x_gdn_core = _gpu_student_t(M, 4096, seed + 1)
        self.x_attn_core = _gpu_student_t(M, 6144, seed + 2)
        self.gs_x = nv.global_scale(self.x)
        self.gs_gc = nv.global_scale(self.x_gdn_core)
        self.gs_ac = nv.global_scale(self.x_attn_core)

        def qbuf(rows, cols):
            return (torch.empty((rows, cols // 2), dtype=torch.uint8, device=dev),
                    torch.empty(nv.scale_bytes(rows, cols), dtype=torch.uint8, device=dev))
        self.qx = qbuf(M, H)
        self.qgc = qbuf(M, 4096)
        self.qac = qbuf(M, 6144)
        self.hq = qbuf(M, I)
        self.out_gdn = torch.empty((M, 12352), dtype=torch.bfloat16, device=dev)
        self.out_qkv = torch.empty((M, 8192), dtype=torch.bfloat16, device=dev)
        self.out = torch.empty((M, H), dtype=torch.bfloat16, device=dev)
        self.gates = _gdn_gate_tensors(torch, M, seed + 100)
        self.layers = []
        s = seed + 1000
        for li in range(layers):
            L = {}
            if li % 4 == 3:
                qkv = [_gpu_normal(6144, H, s, 0.02), _gpu_normal(1024, H, s + 1, 0.02),
                       _gpu_normal(1024, H, s + 2, 0.02)]
                L["qkv"] = nv.quantize_fused(qkv)
                del qkv
                L["o"] = nv.quantize(_gpu_normal(H, 6144, s + 3, 0.02))
            else:
                L["in"] = _gdn_weight(nv, H, s)
                L["out"] = nv.quantize(_gpu_normal(H, 4096, s + 10, 0.02))
            gu = [_gpu_normal(I, H, s + 20, 0.02), _gpu_normal(I, H, s + 21, 0.02)]
            L["gu"] = nv.quantize_fused(gu)
            del gu
            L["down"] = nv.quantize(_gpu_normal(H, I, s + 22, 0.02))
            self.layers.append(L)
            s += 100
        torch.cuda.synchronize()
        # static global scale of the MLP hidden state, calibrated on layer 0
        xq = nv.quantize(self.x, self.gs_x, codes=self.qx[0], scales=self.qx[1])
        w, segs = self.layers[0]["gu"]
        h16 = nv.linear(xq, w, segments=segs, epilogue="silu_mul", out_dtype="bf16")
        self.gs_h = nv.global_scale(h16)
        del h16
        torch.cuda.synchronize()
        ng, na, nl = self.n_gdn, self.n_attn, layers
        per_tok = (ng * 2 * (12352 * H + H * 4096) + na * 2 * (8192 * H + H * 6144)
                   + nl * 2 * (2 * I * H + H * I))
        self.flops = float(per_tok) * M
        self.f_gu = 2.0 * M * 2 * I * H
        self.launches_per_step = ng * 4 + na * 4 + nl * 3
        self.packed_bytes = sum(t.codes.numel() + t.scales.numel()
                                for L in self.layers for v in L.values()
                                for t in ([v[0]] if isinstance(v, tuple) else [v]))
        self.l2_note = f"weights {self.packed_bytes / 2**30:.2f} GiB packed, streamed once per step (> L2)"
        self.dominant = ("gemm_gate_up", self.f_gu, "tensor",
                         "gemm2_kernel (CTA pair; MLP gate|up, SiLU*mul, NVFP4 requant epilogue)")
        self.phases = {"quantize": ("GB/s", 2.5625 * M * (2 * nl * H + ng * 4096 + na * 6144)),
                       "gemm_gdn_in": ("TFLOP/s", ng * 2.0 * M * 12352 * H),
                       "gemm_gdn_out": ("TFLOP/s", ng * 2.0 * M * H * 4096),
                       "gemm_attn_qkv": ("TFLOP/s", na * 2.0 * M * 8192 * H),
                       "gemm_attn_o": ("TFLOP/s", na * 2.0 * M * H * 6144),
                       "gemm_gate_up": ("TFLOP/s", nl * self.f_gu),
                       "gemm_down": ("TFLOP/s", nl * 2.0 * M * H * I)}

    def work(self):
        return self.flops

    def config(self):
        return {"M": self.M, "layers": f"{self.n_gdn} GDN + {self.n_attn} attention, {self.n_layers} MLP",
                "linears": self.n_linears, "gemm_launches_per_step": 2 * self.n_layers + 2 * self.n_layers,
                "packed_weight_gib": round(self.packed_bytes / 2**30, 3),
                "step": "per layer: quantise(input) -> fused NVFP4 GEMM(s) with the layer's epilogue"}

    def plan(self, x):
        nv = self.nv
        H, I, M = 5120, 17408, self.M
        qx = nv.NVFP4Tensor(self.qx[0], self.qx[1], self.gs_x, M, H)
        qgc = nv.NVFP4Tensor(self.qgc[0], self.qgc[1], self.gs_gc, M, 4096)
        qac = nv.NVFP4Tensor(self.qac[0], self.qac[1], self.gs_ac, M, 6144)
        hq = nv.NVFP4Tensor(self.hq[0], self.hq[1], self.gs_h, M, I)
        quant_x = ("quantize", lambda: nv.quantize(x, self.gs_x, codes=self.qx[0], scales=self.qx[1]))
        out = []
        for L in self.layers:
            out.append(quant_x)
            if "qkv" in L:
                w, segs = L["qkv"]
                out.append(("gemm_attn_qkv", lambda w=w, segs=segs: self._lin(
                    qx, w, segments=segs, out_dtype="bf16", out=self.out_qkv)))
                out.append(("quantize", lambda: nv.quantize(self.x_attn_core, self.gs_ac, codes=self.qac[0],
                                                            scales=self.qac[1])))
                out.append(("gemm_attn_o", lambda wo=L["o"]: self._lin(qac, wo, out_dtype="bf16", out=self.out)))
            else:
                w, segs = L["in"]
                out.append(("gemm_gdn_in", lambda w=w, segs=segs: self._lin(
                    qx, w, segments=segs, epilogue="gdn_gates", gates=self.gates, out_dtype="bf16",
                    out=self.out_gdn)))
                out.append(("quantize", lambda: nv.quantize(self.x_gdn_core, self.gs_gc, codes=self.qgc[0],
                                                            scales=self.qgc[1])))
                out.append(("gemm_gdn_out", lambda wo=L["out"]: self._lin(qgc, wo, out_dtype="bf16",
                                                                          out=self.out)))
            out.append(quant_x)
            w, segs = L["gu"]
            out.append(("gemm_gate_up", lambda w=w, segs=segs: self._lin(
                qx, w, segments=segs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=self.gs_h, out=self.hq[0],
                out_scales=self.hq[1])))
            out.append(("gemm_down", lambda wd=L["down"]: self._lin(hq, wd, out_dtype="bf16", out=self.out)))
        return out

    def _lin(self, a, w, **kw):
        return self.nv.linear(a, w, **kw)

    cpu_sample_note = ("one sampled MLP block and one sampled GDN in-proj (32 token rows, 256-320 weight rows, "
                       "full K), FLOP-weighted; numpy FP64 oracle")

    def cpu_sample(self):
        f1, s1 = cpu_mlp_sample()
        f2, s2 = cpu_gdn_sample(5120)
        return f1 + f2, s1 + s2


class KVCacheFP8(Workload):
    """FP8 KV-cache write of one attention layer's prefill: K and V [M x 1024] BF16 (8 KV
    heads x 128) into a paged cache (pages of 16 slots, shuffled) with static scales."""
    unit = "GB/s"

    def __init__(self, nv, M=32768, width=1024, seed=0):
        import torch
        self.nv, self.M, self.width = nv, M, width
        self.name = f"kv_cache_fp8_m{M}_w{width}"
        self.x = _gpu_student_t(M, width, seed, hot=4)
        self.v = _gpu_student_t(M, width, seed + 1, hot=0)
        self.k_scale = nv.fp8_scale(self.x)
        self.v_scale = nv.fp8_scale(self.v)
        g = torch.Generator(device="cuda")
        g.manual_seed(seed + 2)
        num_slots = 2 * M
        pages = torch.randperm(num_slots // 16, generator=g, device="cuda")
        t = torch.arange(M, device="cuda")
        self.slots = (pages[t // 16] * 16 + t % 16).to(torch.int64)
        self.k_cache = torch.empty((num_slots, width), dtype=torch.uint8, device="cuda")
        self.v_cache = torch.empty((num_slots, width), dtype=torch.uint8, device="cuda")
        self.out = self.k_cache
        self.bytes = 2.0 * M * width * 3 + 8.0 * M
        self.launches_per_step = 1
        self.l2_note = f"inputs larger than L2 (K, V {2 * M * width * 2 / 1e6:.0f} MB)"
        self.dominant = ("kv_cache", self.bytes, "hbm", "kv_cache_fp8_kernel (K and V, slot scatter)")
        self.phases = {"kv_cache": ("GB/s", self.bytes)}
        torch.cuda.synchronize()

    def work(self):
        return self.bytes

    def config(self):
        return {"M": self.M, "width": self.width, "scales": "static per tensor (calibrated once)",
                "bytes_per_element": 3, "slots": "pages of 16, shuffled"}

    def plan(self, x):
        nv = self.nv
        return [("kv_cache", lambda: nv.kv_cache_fp8(x, self.v, self.k_scale, self.v_scale, self.slots,
                                                    self.k_cache, self.v_cache))]

    cpu_sample_note = "FP8 KV write of 64 tokens x 1024 (K and V); numpy oracle"

    def cpu_sample(self):
        import numpy as np
        import oracle
        import synth
        k = synth.bf16_to_f32(synth.student_t_activations(64, 1024, seed=0, hot_channels=4))
        v = synth.bf16_to_f32(synth.student_t_activations(64, 1024, seed=1, hot_channels=0))
        ks, vs = oracle.fp8_scale(k), oracle.fp8_scale(v)
        t0 = time.perf_counter()
        oracle.kv_cache_fp8(k, ks, np.arange(64), 64)
        oracle.kv_cache_fp8(v, vs, np.arange(64), 64)
        return 2.0 * 64 * 1024 * 3 + 8.0 * 64, time.perf_counter() - t0


class DecodeSweep(HybridSweep):
    """One decode step of the 496 linears for a batch of M sequences (concurrency 32 by
    default): the split-K linear streams every weight once per step from HBM, so the
    bound is HBM bandwidth over the packed weights.  The step's 704 launches are
    replayed as one CUDA graph (launch overhead would otherwise dominate)."""
    use_graph = True

    def __init__(self, nv, M=32, seed=0, layers=64):
        import torch
        super().__init__(nv, M=M, seed=seed, layers=layers)
        self.name = (f"decode_sweep_496_linears_m{M}" if layers == 64
                     else f"decode_sweep_{self.n_linears}_linears_{layers}_layers_m{M}")
        shapes = [(12352, 5120), (5120, 4096), (8192, 5120), (5120, 6144), (34816, 5120), (5120, 17408)]
        ws = max(nv.splitk_workspace_bytes(M, n, nv.splitk_default(M, n, k)) for n, k in shapes)
        self.workspace = torch.empty(ws, dtype=torch.uint8, device="cuda")
        self.splits = {f"{n}x{k}": nv.splitk_default(M, n, k) for n, k in shapes}
        ng, na, nl = self.n_gdn, self.n_attn, layers
        # + one split-K epilogue launch per GEMM, except where one split lets the decode
        # kernel apply the epilogue itself (element-wise epilogue, BF16 out: every GEMM
        # of the step but the MLP gate|up with its NVFP4 output), or, above 64 rows, runs
        # the plain GEMM
        one = lambda key: int(self.splits[key] == 1)
        direct = (ng * (one("12352x5120") + one("5120x4096")) + na * (one("8192x5120") + one("5120x6144"))
                  + nl * one("5120x17408") + (nl * one("34816x5120") if M > 64 else 0))
        self.launches_per_step = ng * 4 + na * 4 + nl * 3 + (2 * ng + 2 * na + 2 * nl) - direct
        H, I = 5120, 17408
        wb = lambda n, k: n * k * 0.5625  # packed codes + scales

        def gemm_bytes(n, k, count):
            return count * (wb(n, k) + M * k * 0.5625 + M * n * 2)
        self.bytes_gu = wb(2 * I, H) + M * H * 0.5625 + M * I * 0.5625
        self.dominant = ("gemm_gate_up", self.bytes_gu, "hbm",
                         f"nvfp4_linear_splitk (MLP gate|up, SiLU*mul, NVFP4 requant; "
                         f"split_k {self.splits['34816x5120']})")
        self.phases = {"quantize": ("GB/s", 2.5625 * M * (2 * nl * H + ng * 4096 + na * 6144)),
                       "gemm_gdn_in": ("GB/s", gemm_bytes(12352, H, ng)),
                       "gemm_gdn_out": ("GB/s", gemm_bytes(H, 4096, ng)),
                       "gemm_attn_qkv": ("GB/s", gemm_bytes(8192, H, na)),
                       "gemm_attn_o": ("GB/s", gemm_bytes(H, 6144, na)),
                       "gemm_gate_up": ("GB/s", nl * self.bytes_gu),
                       "gemm_down": ("GB/s", gemm_bytes(H, I, nl))}
        self.l2_note = (f"weights {self.packed_bytes / 2**30:.2f} GiB packed, streamed from HBM once per step "
                        "(> L2)")

    def config(self):
        c = super().config()
        c["split_k"] = self.splits
        c["step"] = ("per layer: quantise(input) -> split-K NVFP4 GEMM(s) -> split-K epilogue kernel "
                     "(the layer's epilogue)")
        return c

    def _lin(self, a, w, **kw):
        return self.nv.linear_splitk(a, w, workspace=self.workspace, **kw)

    def report(self, ms_step):
        return {"decode_step": {"ms": round(ms_step, 4), "tokens_per_s_linears_only": round(self.M / ms_step * 1e3, 1),
                                "weight_GB/s": round(self.packed_bytes / ms_step / 1e6, 1)}}


class GDNRecurrence(Workload):
    """Gated delta-rule recurrence of one GDN layer at M prefill tokens (sequences of
    4096, fresh states): 16 key / 32 value heads of 128, q|k|v BF16 rows, g / beta FP32
    [M x 32] as the gate epilogue writes them, FP32 state, BF16 output [M x 4096].
    Algorithmic FLOPs per token and value head: 7 d_k d_v (prediction S^T k 2, decay 1,
    rank-1 write 2, read-out S^T q 2)."""
    unit = "TFLOP/s"
    dtype = "fp32 state; bf16 tensor-core products, fp32 operands split hi/lo (bf16 q/k/v/out)"
    SEQ = 4096

    def __init__(self, nv, M=8192, seed=0):
        import torch
        self.nv, self.M = nv, M
        self.n_seqs = (M + self.SEQ - 1) // self.SEQ
        self.name = f"gdn_recurrence_t{M}_seq{min(M, self.SEQ)}_hk16_hv32_d128"
        self.x, self.g, self.beta, self.cu = _gpu_gdn_rec_inputs(M, self.SEQ, seed)
        self.state = torch.zeros((self.n_seqs, 32, 128, 128), dtype=torch.float32, device="cuda")
        self.out = torch.empty((M, 32 * 128), dtype=torch.bfloat16, device="cuda")
        self.flops = 7.0 * 128 * 128 * 32 * M
        # Tensor-core FLOPs chunk_kernel issues: per (64-token chunk, value head, 64-column
        # block) 2096 mma.sync m16n8k16 (K S0 / Q S0 hi+lo 1024, lower K K^T / Q K^T blocks
        # 320, P U as three split products over the lower triangle 240, K^T W hi+lo 512),
        # 4096 FLOP each; two column blocks per head.
        chunks = sum(-(-min(self.SEQ, M - s0) // 64) for s0 in range(0, M, self.SEQ))
        self.mma_flops = 2096.0 * 4096 * chunks * 32 * 2
        self.launches_per_step = 1
        self.l2_note = (f"inputs larger than L2 (q|k|v rows {M * 8192 * 2 / 1e6:.0f} MB, out "
                        f"{M * 4096 * 2 / 1e6:.0f} MB)")
        self.dominant = ("gdn_recurrence", self.mma_flops, "tensor_bf16",
                         "gdn chunk_kernel (64-token chunks; products on BF16 mma.sync with FP32 operands split "
                         "hi/lo; rate in the tensor FLOPs it issues, against the BF16 tensor peak)")
        self.phases = {"gdn_recurrence": ("ALU", self.flops)}
        torch.cuda.synchronize()

    def work(self):
        return self.flops

    def config(self):
        return {"tokens": self.M, "seq_len": min(self.M, self.SEQ), "n_seqs": self.n_seqs, "key_heads": 16,
                "value_heads": 32, "head_dim": 128, "state": "fp32, fresh per sequence",
                "flops_per_token_head": "7 * 128 * 128 (token recurrence)",
                "tensor_flops_issued_per_launch": self.mma_flops}

    def plan(self, x):
        nv = self.nv
        q, k, v = x[:, :2048], x[:, 2048:4096], x[:, 4096:]
        return [("gdn_recurrence", lambda: nv.gdn_recurrence(q, k, v, self.g, self.beta, self.cu, self.state,
                                                            initial_state=False, out=self.out))]

    cpu_sample_note = "GDN recurrence, 1 sequence x 64 tokens x 4 value heads; numpy oracle (fp64)"

    def cpu_sample(self):
        import oracle
        import synth
        d = synth.gdn_recurrence_inputs([64], 2, 4, seed=0)
        f = lambda c, h: synth.bf16_to_f32(d["rows"][:, c:c + h * 128]).reshape(64, h, 128)
        q, k, v = f(d["q_col"], 2), f(d["k_col"], 2), f(d["v_col"], 4)
        t0 = time.perf_counter()
        oracle.gdn_recurrence(q, k, v, d["g"], d["beta"])
        return 7.0 * 128 * 128 * 4 * 64, time.perf_counter() - t0


class GDNDecode(GDNRecurrence):
    """One decode step of the GDN recurrence for M sequences (one token each) over their
    carried FP32 states [M x 32 x 128 x 128]: every state is read and written once, so
    the bound is HBM bandwidth.  Algorithmic bytes: state 2 x 64 KiB per (sequence, value
    head), q|k|v 16 KiB, g / beta 256 B and BF16 output 8 KiB per sequence."""
    unit = "GB/s"
    SEQ = 1
    use_graph = True  # a ~20 us step: replay it as a graph so host launch gaps do not count

    def __init__(self, nv, M=32, seed=0):
        import torch
        super().__init__(nv, M=M, seed=seed)
        self.name = f"gdn_decode_b{M}_hk16_hv32_d128"
        g = torch.Generator(device="cuda")
        g.manual_seed(seed + 1)
        self.state.copy_(0.3 * torch.randn(self.state.shape, generator=g, device="cuda"))
        self.bytes = M * (32 * 2 * 128 * 128 * 4 + 8192 * 2 + 2 * 32 * 4 + 4096 * 2) + 4.0 * (M + 1)
        self.l2_note = f"states {self.state.numel() * 4 / 1e6:.0f} MB read and written per step (> L2)"
        self.dominant = ("gdn_recurrence", self.bytes, "hbm",
                         "gdn column_kernel (one warp per four state columns; state read + write)")
        self.phases = {"gdn_recurrence": ("GB/s", self.bytes)}

    def work(self):
        return self.bytes

    def config(self):
        return {"sequences": self.M, "tokens_per_sequence": 1, "key_heads": 16, "value_heads": 32,
                "head_dim": 128, "state": "fp32, carried (read and written each step)"}

    def plan(self, x):
        nv = self.nv
        q, k, v = x[:, :2048], x[:, 2048:4096], x[:, 4096:]
        return [("gdn_recurrence", lambda: nv.gdn_recurrence(q, k, v, self.g, self.beta, self.cu, self.state,
                                                            initial_state=True, out=self.out))]

    cpu_sample_note = "GDN decode step, 8 sequences x 32 value heads; numpy oracle (fp64)"

    def cpu_sample(self):
        import numpy as np
        import oracle
        import synth
        d = synth.gdn_recurrence_inputs([1] * 8, 16, 32, seed=0)
        f = lambda c, h: synth.bf16_to_f32(d["rows"][:, c:c + h * 128]).reshape(8, h, 128)
        q, k, v = f(d["q_col"], 16), f(d["k_col"], 16), f(d["v_col"], 32)
        S0 = np.random.default_rng(0).standard_normal((8, 32, 128, 128)) * 0.3
        t0 = time.perf_counter()
        for s in range(8):
            oracle.gdn_recurrence(q[s:s + 1], k[s:s + 1], v[s:s + 1], d["g"][s:s + 1], d["beta"][s:s + 1], S0[s])
        per_seq = 32 * 2 * 128 * 128 * 4 + 8192 * 2 + 2 * 32 * 4 + 4096 * 2
        return 8.0 * per_seq, time.perf_counter() - t0


WORKLOADS = {"mlp": MLPBlock, "quantize": QuantizeOnly, "gdn": GDNInProj, "linear": SmallLinear,
             "sweep": HybridSweep, "decode": DecodeSweep,
             "kv": KVCacheFP8, "gdn_rec": GDNRecurrence, "gdn_decode": GDNDecode}


def make_workload(args, nv):
    cls = WORKLOADS[args.workload]
    kw = {}
    if args.M:
        kw["M"] = args.M
    if args.layers:
        if cls not in (HybridSweep, DecodeSweep):
            raise SystemExit("--layers applies to the sweep and decode workloads")
        kw["layers"] = args.layers
    return cls(nv, **kw)


# ---------------------------------------------------------------- GPU arm
def capture_graph(torch, launches):
    """One CUDA graph holding ``launches`` (callables that launch on the current stream)."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for launch in launches:
            launch()
    return g


def time_replays(torch, g, n):
    """Device time of ``n`` back-to-back replays of graph ``g`` (CUDA events), in ms."""
    g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(n):
        g.replay()
    e.record()
    torch.cuda.synchronize()
    return s.elapsed_time(e)


def run_ours(args, ws, rank):
    import torch
    import nvfp4_w4a4_quantized_02_b200 as nv
    from nvfp4_w4a4_quantized_02_b200 import build
    if rank == 0 or ws == 1:
        build.build()
    if ws > 1:
        torch.distributed.barrier()
    nv.lib()
    peaks, peak_src = load_peaks()
    wl = make_workload(args, nv)
    graph = wl.use_graph or args.graph
    stream = torch.cuda.current_stream()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda") if wl.flush_l2 else None

    for _ in range(args.warmup):
        wl.step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize()
    plan = wl.plan(wl.x)
    g_step = capture_graph(torch, [launch for _, launch in plan]) if graph else None
    if graph:
        for _ in range(2):
            g_step.replay()
        torch.cuda.synchronize()

    tm = KernelTimer(torch) if not graph else NO_TIMER
    steps = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
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
        steps[i][0].record(stream)
        if graph:
            g_step.replay()
        else:
            wl.step(tm)
        steps[i][1].record(stream)
        if flush is not None:
            flush.zero_()
    stop.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if flush is not None:
        elapsed_ms = sum(a.elapsed_time(b) for a, b in steps)
    else:
        elapsed_ms = start.elapsed_time(stop)
    if ws > 1:
        elapsed_ms = max_over_ranks(elapsed_ms, "cuda")
        torch.distributed.barrier()

    # per-phase device time: events around each launch (eager), or one graph per phase
    # holding that phase's launches of one step (graph mode: no host gaps between them)
    per_phase = {}
    if graph:
        for key in wl.phases:
            launches = [launch for ph, launch in plan if ph == key]
            if launches:
                g = capture_graph(torch, launches)
                reps = 5
                per_phase[key] = {"launches": len(launches), "ms_step": time_replays(torch, g, reps) / reps}
                del g
    else:
        for key, d in tm.summary().items():
            per_phase[key] = {"launches": d["launches"] // args.steps, "ms_step": d["ms_total"] / args.steps}
    # FP32 FMA peak of the device: SMs x lanes x 2 FLOP x max SM clock (sampled max, else nominal)
    sm_max = (clocks or {}).get("sm_max_mhz") or SM_MAX_MHZ
    alu_peak = props.multi_processor_count * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
    # Tensor peak: the measured BF16 GEMM rate x the nominal FP4/BF16 ratio, burst for a
    # timed region under a second (the clocks stay at their maximum), sustained (the
    # power-capped rate of a seconds-long GEMM loop) for longer ones.
    region = "sustained" if elapsed_ms >= SUSTAINED_REGION_MS else "burst"
    bf16_peak = peaks["bf16_tflops_sustained"] if region == "sustained" else peaks["bf16_tflops"]
    fp4_peak = bf16_peak * FP4_OVER_BF16
    sm_mhz = (clocks or {}).get("sm_mhz")
    fp4_at_clock = NOMINAL_FP4_TFLOPS * (sm_mhz / SM_MAX_MHZ) if sm_mhz else None
    kernels = {}
    for key, (unit, amount) in wl.phases.items():
        if key not in per_phase:
            continue
        ms = per_phase[key]["ms_step"]
        d = {"launches_per_step": per_phase[key]["launches"], "ms_per_step": round(ms, 5)}
        if unit == "GB/s":
            d["GB/s"] = round(amount / ms / 1e6, 1)
            d["frac_hbm"] = round(d["GB/s"] / peaks["hbm_gbs"], 4)
            d["frac_hbm_nominal"] = round(d["GB/s"] / NOMINAL_HBM_GBS, 4)
        elif unit == "ALU":
            d["TFLOP/s"] = round(amount / ms / 1e9, 2)
            d["frac_fp32_peak"] = round(d["TFLOP/s"] / alu_peak, 4)
        else:
            d["TFLOP/s"] = round(amount / ms / 1e9, 1)
            d["frac_fp4_peak"] = round(d["TFLOP/s"] / fp4_peak, 4)
            d["frac_fp4_nominal"] = round(d["TFLOP/s"] / NOMINAL_FP4_TFLOPS, 4)
        if key in getattr(wl, "l2_stream", {}):
            d["l2_to_sm_TB/s"] = round(wl.l2_stream[key] / (ms / per_phase[key]["launches"]) / 1e9, 2)
        kernels[key] = d

    key, per_launch, bound, label = wl.dominant
    avg_ms = per_phase[key]["ms_step"] / per_phase[key]["launches"]
    extra_fracs = {}
    if bound == "hbm":
        achieved = per_launch / avg_ms / 1e6
        peak, unit = peaks["hbm_gbs"], "GB/s"
        note = f"{peak_src} hbm_gbs (copy bandwidth)"
        extra_fracs = {"frac_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                       "nominal_peak": NOMINAL_HBM_GBS}
    elif bound == "alu":
        achieved = per_launch / avg_ms / 1e9
        peak, unit = round(alu_peak, 2), "TFLOP/s"
        note = (f"derived FP32 FMA peak: {props.multi_processor_count} SMs x {FP32_LANES_PER_SM} lanes x 2 FLOP x "
                f"{sm_max:.0f} MHz")
    elif bound == "tensor_bf16":
        achieved = per_launch / avg_ms / 1e9
        peak, unit = round(bf16_peak, 1), "TFLOP/s"
        bound = "tensor"
        src = "bf16_tflops_sustained" if region == "sustained" else "bf16_tflops (burst)"
        note = f"{peak_src} {src} (BF16 mma.sync products); timed region {elapsed_ms:.0f} ms"
        extra_fracs = {"frac_nominal": round(achieved / (NOMINAL_FP4_TFLOPS / FP4_OVER_BF16), 4),
                       "nominal_peak": NOMINAL_FP4_TFLOPS / FP4_OVER_BF16}
    else:
        achieved = per_launch / avg_ms / 1e9
        peak, unit = round(fp4_peak, 1), "TFLOP/s"
        src = "bf16_tflops_sustained" if region == "sustained" else "bf16_tflops (burst)"
        note = (f"{peak_src} {src} x {FP4_OVER_BF16} (nominal FP4/BF16 ratio); timed region "
                f"{elapsed_ms:.0f} ms")
        extra_fracs = {"frac_nominal": round(achieved / NOMINAL_FP4_TFLOPS, 4),
                       "nominal_peak": NOMINAL_FP4_TFLOPS}
        if fp4_at_clock:
            extra_fracs["frac_nominal_at_median_clock"] = round(achieved / fp4_at_clock, 4)
    if sm_mhz:
        extra_fracs["sm_mhz_median"] = sm_mhz
    if key in getattr(wl, "l2_stream", {}):
        extra_fracs["l2_to_sm"] = {
            "TB/s": round(wl.l2_stream[key] / avg_ms / 1e9, 2), "bytes_per_launch": wl.l2_stream[key],
            "note": "TMA operand bytes from L2 (76 KB per 256x256x256 pair-tile stage) / launch time; at full "
                    "occupancy the pair GEMM runs at this stream's ~12 TB/s limit (same rate for gate|up and down; "
                    "per-tile time falls to the MMA stream's on fewer clusters)"}
    roof = {"kernel": label, "bound": bound, "achieved": round(achieved, 2), "peak": peak, "unit": unit,
            "frac": round(achieved / peak, 4), **extra_fracs, "traffic": load_traffic(f"{key}@{wl.name}"),
            "avg_launch_ms": round(avg_ms, 5), "work_per_launch": per_launch, "peak_note": note,
            "timing": "graph of the phase's launches, CUDA events" if graph else "CUDA events per launch"}

    e2e = run_e2e(wl, args, torch, flush, g_step)
    ms = elapsed_ms / args.steps
    if wl.unit == "GB/s":
        value = ws * wl.work() / (ms * 1e-3) / 1e9
    else:
        value = ws * wl.work() / (ms * 1e-3) / 1e12
    cfg = {"workload": wl.name, **wl.config(),
           "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU", "l2": wl.l2_note,
           "launch": "one CUDA graph per step" if graph else "eager launches"}
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": wl.unit, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.dtype or ("nvfp4(e2m1+e4m3)->fp32 acc" if wl.unit != "GB/s" else "bf16->nvfp4"),
        "data": "synthetic", "config": cfg, "roofline": roof, "kernels": kernels, "e2e": e2e,
        "gpu_launches": wl.launches_per_step * args.steps, "clocks": clocks, "peaks_source": peak_src,
    }
    if hasattr(wl, "extra"):
        line["kernels"].update(wl.extra(torch))
    if hasattr(wl, "report"):
        line["kernels"].update(wl.report(ms))
    if args.workload == "mlp" and ws == 1 and not args.no_other_configs:
        line["other_configs"] = other_configs(nv, torch, peaks)
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)


def time_phases(wl, torch, steps, warmup):
    """Device time of ``steps`` eager steps of ``wl`` after ``warmup`` (CUDA events around
    every launch and around the whole region): (ms per step, {phase: ms per step}, region ms)."""
    for _ in range(warmup):
        wl.step()
    torch.cuda.synchronize()
    tm = KernelTimer(torch)
    stream = torch.cuda.current_stream()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        wl.step(tm)
    e.record(stream)
    torch.cuda.synchronize()
    region = s.elapsed_time(e)
    per = {k: d["ms_total"] / steps for k, d in tm.summary().items()}
    return region / steps, per, region


def other_configs(nv, torch, peaks):
    """The quantiser at 32768 x 5120 with a static global scale, the GDN fused input
    projection at 8192 tokens and one pass of the 496-linear sweep at 4096 tokens, each
    built, timed (CUDA events, eager launches) and freed in turn.  Every timed region is
    well under a second, so the burst tensor peak applies."""
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    res = {}
    props = torch.cuda.get_device_properties(torch.cuda.current_device())
    sampler = ClockSampler("GPU-" + str(props.uuid))
    sampler.start()

    wl = QuantizeOnly(nv)
    ms, per, region = time_phases(wl, torch, steps=20, warmup=3)
    gbs = wl.bytes / per["quantize"] / 1e6
    res["quantize_static_m32768_k5120"] = {
        "ms": round(per["quantize"], 5), "GB/s": round(gbs, 1), "frac_hbm": round(gbs / peaks["hbm_gbs"], 4),
        "frac_hbm_nominal": round(gbs / NOMINAL_HBM_GBS, 4), "bytes": wl.bytes, "steps": 20,
        "kernel": "quantize_kernel"}
    del wl

    wl = GDNInProj(nv)
    ms, per, region = time_phases(wl, torch, steps=20, warmup=3)
    tf = wl.flops / per["gemm"] / 1e9
    res["gdn_inproj_m8192_n12352_k5120"] = {
        "ms_step": round(ms, 5), "ms_gemm": round(per["gemm"], 5), "TFLOP/s": round(tf, 1),
        "frac_fp4_peak": round(tf / fp4_peak, 4), "frac_fp4_nominal": round(tf / NOMINAL_FP4_TFLOPS, 4),
        "step_TFLOP/s": round(wl.flops / ms / 1e9, 1), "steps": 20,
        "kernel": "gemm2_kernel (6 segments, GDN gate epilogue)",
        "step": "global_scale + quantize(X) + fused GEMM"}
    del wl

    wl = HybridSweep(nv, M=4096)
    ms, per, region = time_phases(wl, torch, steps=3, warmup=1)
    tf = wl.flops / ms / 1e9
    gemm_ms = sum(v for k, v in per.items() if k.startswith("gemm"))
    tf_gu = 64 * wl.f_gu / per["gemm_gate_up"] / 1e9
    res["sweep_496_linears_m4096"] = {
        "ms_step": round(ms, 4), "TFLOP/s": round(tf, 1), "frac_fp4_peak": round(tf / fp4_peak, 4),
        "frac_fp4_nominal": round(tf / NOMINAL_FP4_TFLOPS, 4),
        "gemm_only_TFLOP/s": round(wl.flops / gemm_ms / 1e9, 1),
        "gate_up_TFLOP/s": round(tf_gu, 1), "gate_up_frac_fp4_peak": round(tf_gu / fp4_peak, 4),
        "launches_per_step": wl.launches_per_step, "steps": 3,
        "packed_weight_gib": round(wl.packed_bytes / 2**30, 3),
        "step": "496 linears: quantise(input) -> fused NVFP4 GEMM with the layer's epilogue"}
    del wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    res["clocks_during_other_configs"] = sampler.stop()
    res["peak_note"] = f"FP4 peak = bf16_tflops (burst) x {FP4_OVER_BF16} = {fp4_peak:.0f} TFLOP/s"
    return res


def run_e2e(wl, args, torch, flush, g_step=None):
    """The same step through the public API with host buffers: pinned H2D of the step's
    input, the step, D2H of its result, all inside the timed region.  A graph step reads
    the buffer it was captured with, so the input is copied into that buffer.

    When the workload needs no L2 flush between steps (its inputs exceed L2), the steps
    are pipelined as a server would run them: the H2D of step i + 1 (one copy stream)
    and the D2H of step i - 1 (another) overlap step i, through double-buffered device
    staging; the value is the throughput of n such steps, timed from the first H2D to
    the last D2H on the launching stream.  Otherwise each step runs H2D -> step -> D2H in
    order, timed on its own with an L2 flush in between."""
    if flush is None:
        return run_e2e_pipelined(wl, args, torch, g_step)
    stream = torch.cuda.current_stream()
    x_host = wl.x.cpu().pin_memory()
    out_host = torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True)
    x_dev = wl.x if g_step is not None else torch.empty_like(wl.x)

    def one():
        x_dev.copy_(x_host, non_blocking=True)
        if g_step is not None:
            g_step.replay()
            out_host.copy_(wl.out, non_blocking=True)
        else:
            out_host.copy_(wl.step(x=x_dev), non_blocking=True)

    n = max(1, min(args.steps, 10))
    for _ in range(2):
        one()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for a, b in evs:
        a.record(stream)
        one()
        b.record(stream)
        flush.zero_()
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / n
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    return {"value": round(wl.work() / (ms * 1e-3) / scale, 2), "unit": wl.unit,
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": out_host.numel() * out_host.element_size(),
            "ms_per_step": round(ms, 4), "steps": n, "schedule": "sequential, L2 flushed between steps",
            "host_leg": "pinned host buffers and torch copies around the Python binding's C-ABI calls (the C ABI "
                        "itself takes device pointers)"}


def run_e2e_pipelined(wl, args, torch, g_step=None):
    main = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    x_host = wl.x.cpu().pin_memory()
    out_host = [torch.empty(wl.out.shape, dtype=wl.out.dtype, pin_memory=True) for _ in range(2)]
    x_stage = [torch.empty_like(wl.x) for _ in range(2)]
    out_stage = [torch.empty_like(wl.out) for _ in range(2)]
    ev = lambda: torch.cuda.Event()
    in_ready, x_free = [ev(), ev()], [ev(), ev()]
    out_ready, out_free = [ev(), ev()], [ev(), ev()]
    for e in x_free + out_free:
        e.record(main)

    def one(i):
        b = i % 2
        with torch.cuda.stream(s_in):  # H2D of step i into staging buffer b
            s_in.wait_event(x_free[b])
            x_stage[b].copy_(x_host, non_blocking=True)
            in_ready[b].record(s_in)
        main.wait_event(in_ready[b])
        if g_step is not None:
            wl.x.copy_(x_stage[b], non_blocking=True)
            x_free[b].record(main)
            g_step.replay()
            out = wl.out
        else:
            out = wl.step(x=x_stage[b])
            x_free[b].record(main)
        main.wait_event(out_free[b])
        out_stage[b].copy_(out, non_blocking=True)
        out_ready[b].record(main)
        with torch.cuda.stream(s_out):  # D2H of step i from staging buffer b
            s_out.wait_event(out_ready[b])
            out_host[b].copy_(out_stage[b], non_blocking=True)
            out_free[b].record(s_out)

    n = max(2, min(args.steps, 10))
    for i in range(2):
        one(i)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(main)
    s_in.wait_event(start)
    for i in range(n):
        one(i)
    for b in range(2):
        main.wait_event(out_free[b])
    end.record(main)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end) / n
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    return {"value": round(wl.work() / (ms * 1e-3) / scale, 2), "unit": wl.unit,
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": out_host[0].numel() * out_host[0].element_size(),
            "ms_per_step": round(ms, 4), "steps": n,
            "schedule": "pipelined: H2D of step i+1 and D2H of step i-1 overlap step i (two copy streams, "
                        "double-buffered device staging)",
            "host_leg": "pinned host buffers and torch copies around the Python binding's C-ABI calls (the C ABI "
                        "itself takes device pointers)"}


# ---------------------------------------------------------------- CPU oracle
def cpu_mlp_sample(rows=32, cols_h=256, K=5120):
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


def cpu_gdn_sample(K=5120, rows=32):
    """GDN in-projection on a bounded sample: ``rows`` tokens, 64 rows of each of q/k/v/z
    plus the 32 beta and 32 alpha rows, each segment with its own global scale."""
    import numpy as np
    import oracle
    import synth
    x = synth.bf16_to_f32(synth.outlier_activations(rows, K, seed=0))
    names = [("q", 64), ("k", 64), ("v", 64), ("z", 64), ("beta", 32), ("alpha", 32)]
    ws = synth.segmented_weights(names, K, seed=1, multipliers=synth.GDN_INPROJ_MULTIPLIERS)
    cs, ss, segs, n0 = [], [], [], 0
    for _, wb in ws:
        w = synth.bf16_to_f32(wb)
        g = oracle.global_scale(w)
        c, s = oracle.quantize(w, g)
        cs.append(c), ss.append(s), segs.append((n0, n0 + w.shape[0], g))
        n0 += w.shape[0]
    a_log, dt_bias = synth.gdn_gate_params(32)
    t0 = time.perf_counter()
    gx = oracle.global_scale(x)
    cx, sx = oracle.quantize(x, gx)
    y = oracle.linear(cx, sx, gx, np.concatenate(cs), np.concatenate(ss), segs)
    oracle.gdn_gates(y[:, 256:288], y[:, 288:320], a_log, dt_bias)
    return 2.0 * rows * n0 * K, time.perf_counter() - t0


def _cores():
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()


def cpu_baseline(wl, budget_s=12.0):
    work, secs, n = 0.0, 0.0, 0
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or n == 0:
        w, s = wl.cpu_sample()
        work += w
        secs += s
        n += 1
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    return {"value": work / secs / scale, "unit": wl.unit, "cores": _cores(), "kind": "oracle",
            "sample": f"{n} x {wl.cpu_sample_note}"}


class _CpuOnly:
    """Workload descriptor for the reference arm (no GPU objects)."""

    def __init__(self, args):
        cls = WORKLOADS[args.workload]
        self.cls = cls
        self.unit = cls.unit
        self.cpu_sample_note = cls.cpu_sample_note
        obj = object.__new__(cls)
        obj.M = args.M or {"mlp": 32768, "quantize": 32768, "gdn": 8192, "linear": 128, "sweep": 32768,
                           "decode": 32, "kv": 32768, "gdn_rec": 8192, "gdn_decode": 32}[args.workload]
        obj.K = {"quantize": 5120, "gdn": 5120, "linear": 1024}.get(args.workload, 5120)
        obj.N = {"linear": 1024, "gdn": 12352}.get(args.workload, 0)
        obj.flops = 2.0 * obj.M * obj.N * obj.K
        self.obj = obj
        self.name = {"mlp": f"mlp_block_m{obj.M}_h5120_i17408", "quantize": f"quantize_m{obj.M}_k5120",
                     "gdn": f"gdn_inproj_m{obj.M}_n12352_k5120", "linear": f"linear_m{obj.M}_n1024_k1024",
                     "sweep": f"hybrid_sweep_496_linears_m{obj.M}",
                     "decode": f"decode_sweep_496_linears_m{obj.M}",
                     "kv": f"kv_cache_fp8_m{obj.M}_w1024",
                     "gdn_rec": f"gdn_recurrence_t{obj.M}_seq{min(obj.M, 4096)}_hk16_hv32_d128",
                     "gdn_decode": f"gdn_decode_b{obj.M}_hk16_hv32_d128"}[args.workload]

    def cpu_sample(self):
        return self.cls.cpu_sample(self.obj)


def run_reference(args, ws, rank):
    if rank != 0:
        return
    wl = _CpuOnly(args)
    t0 = time.perf_counter()
    for _ in range(args.warmup):
        wl.cpu_sample()
    work, secs = 0.0, 0.0
    for _ in range(args.steps):
        w, s = wl.cpu_sample()
        work += w
        secs += s
    scale = 1e9 if wl.unit == "GB/s" else 1e12
    value = work / secs / scale
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": wl.unit, "n_gpus": ws,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)",
            "data": "synthetic",
            "config": {"workload": wl.name, "sample": wl.cpu_sample_note},
            "cpu_baseline": {"value": value, "unit": wl.unit, "cores": _cores(), "kind": "oracle",
                             "sample": f"per step: {wl.cpu_sample_note}"},
            "e2e": {"value": value, "unit": wl.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 2)}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="mlp")
    ap.add_argument("--M", type=int, default=0, help="token rows (default: the workload's own)")
    ap.add_argument("--layers", type=int, default=0,
                    help="sweep / decode: build only the first L of the 64 layers (small profiling cases)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true", help="replay each step as one CUDA graph")
    ap.add_argument("--no-other-configs", action="store_true",
                    help="mlp: skip the quantiser / GDN in-projection / sweep sub-results")
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
