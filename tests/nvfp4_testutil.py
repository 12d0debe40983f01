"""Helpers shared by the GPU parity tests: move seeded inputs to the device, read the
library's packed outputs back in the oracle's logical form, and error metrics."""
from __future__ import annotations

import numpy as np

import oracle
import synth
from oracle import layout


def cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def to_dev_bf16(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def to_dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=np.float32))).cuda()


def logical(qt):
    """(codes [rows, cols], sf [rows, cols/16]) of a device NVFP4Tensor, via the layout reading."""
    codes = layout.unpack_nibbles(qt.codes.cpu().numpy())
    sf = layout.unswizzle_scales(qt.scales.cpu().numpy(), qt.rows, qt.cols)
    return codes, sf


def oracle_quant(bits: np.ndarray, gs=None):
    x = synth.bf16_to_f32(bits)
    if gs is None:
        gs = oracle.global_scale(x)
    codes, sf = oracle.quantize(x, np.float32(gs))
    return codes, sf, np.float32(gs)


def make_operand(codes: np.ndarray, sf: np.ndarray, gs: float):
    """Device NVFP4Tensor built directly from logical codes / scales (layout reading)."""
    import torch
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Tensor
    rows, cols = codes.shape
    packed = torch.from_numpy(layout.pack_nibbles(codes)).cuda()
    sw = torch.from_numpy(layout.swizzle_scales(sf, rows, cols)).cuda()
    return NVFP4Tensor(packed, sw, to_dev_f32([gs]), rows, cols)


def rel_fro(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return t.float().cpu().numpy().astype(np.float64)


def assert_gemm_close(out_bf16, ref64, fro_tol=1e-3, elem_tol=2e-2):
    """BF16 output vs the FP64 oracle: relative Frobenius error against the oracle
    rounded to BF16 <= fro_tol, and every |err| <= elem_tol * max|ref|."""
    got = bf16_to_f64(out_bf16)
    ref_b = oracle.round_to_bf16(ref64)
    fro = rel_fro(got, ref_b)
    assert fro <= fro_tol, f"relative Frobenius {fro:.3e} > {fro_tol}"
    emax = float(np.max(np.abs(got - ref64)))
    lim = elem_tol * float(np.max(np.abs(ref64)))
    assert emax <= lim, f"max |err| {emax:.3e} > {lim:.3e}"
    return fro, emax
