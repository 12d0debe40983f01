"""Python binding of the B200 NVFP4 W4A4 linear library (``include/nvfp4.h``).

Argument marshalling only: every step of the quantiser and of the linear runs in
the CUDA kernels of ``libnvfp4_w4a4.so``.  PyTorch supplies device memory (the
caller-side output buffers allocated here) and the current CUDA stream.  There is
no CPU fallback: if the library is missing or the device is not sm_100, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

__all__ = [
    "lib", "NVFP4Error", "scale_bytes", "amax", "global_scale", "quantize", "quantize_fused", "linear",
    "linear_splitk", "linear_splitk_noalloc", "noalloc_default_splits", "splitk_default", "splitk_workspace_bytes",
    "NOALLOC_SCRATCH_BYTES", "fold_segments", "fp8_scale", "kv_cache_fp8", "gdn_recurrence",
    "device_status", "selftest_stalled_linear", "unswizzle_scales", "pack_weight", "NVFP4Tensor", "EPILOGUES", "OUT_KINDS",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
# NVFP4_DEBUG=1 selects the bounds-checking build of the same library (built with
# ``python -m nvfp4_w4a4_quantized_02_b200.build --debug``).
DEBUG = os.environ.get("NVFP4_DEBUG", "0") not in ("", "0")
LIB_PATH = os.path.join(_PKG, "libnvfp4_w4a4_debug.so" if DEBUG else "libnvfp4_w4a4.so")

EPILOGUES = {"none": 0, "silu_mul": 1, "gdn_gates": 2}
OUT_KINDS = {"bf16": 0, "f32": 1, "nvfp4": 2}
MAX_SEGMENTS = 16
NOALLOC_SCRATCH_BYTES = 8 << 20  # NVFP4_NOALLOC_SCRATCH_BYTES of include/nvfp4.h

_c_i64 = ctypes.c_int64
_c_vp = ctypes.c_void_p


class Operand(ctypes.Structure):
    _fields_ = [("codes", _c_vp), ("scales", _c_vp), ("rows", _c_i64), ("K", _c_i64)]


class Segment(ctypes.Structure):
    _fields_ = [("n_begin", _c_i64), ("n_end", _c_i64), ("gs_w", _c_vp)]


class EpilogueParams(ctypes.Structure):
    _fields_ = [("beta_begin", _c_i64), ("alpha_begin", _c_i64), ("n_heads", _c_i64),
                ("A_log", _c_vp), ("dt_bias", _c_vp), ("beta_out", _c_vp), ("g_out", _c_vp),
                ("gs_out", _c_vp), ("out_scales", _c_vp)]


class NVFP4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_lib_status_string(status)} ({status})")


_LIB = None
SYMBOLS = ("nvfp4_status_string", "nvfp4_scale_bytes", "nvfp4_global_scale", "nvfp4_quantize",
           "nvfp4_quantize_rows", "nvfp4_linear", "nvfp4_linear_splitk", "nvfp4_splitk_workspace_bytes",
           "nvfp4_splitk_default", "nvfp4_linear_splitk_noalloc", "nvfp4_fold_segments",
           "nvfp4_fp8_scale", "nvfp4_kv_cache_fp8", "nvfp4_gdn_recurrence", "nvfp4_get_device_status",
           "nvfp4_selftest_stalled_linear", "nvfp4_unswizzle_scales", "nvfp4_pack_weight", "nvfp4_amax")


def lib():
    """The loaded C library (ctypes), with argument types declared."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"NVFP4 CUDA library not built ({LIB_PATH} missing): "
            f"run `python -m nvfp4_w4a4_quantized_02_b200.build{' --debug' if DEBUG else ''}`")
    L = ctypes.CDLL(LIB_PATH)
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_status_string.argtypes = [ctypes.c_int]
    L.nvfp4_scale_bytes.restype = ctypes.c_size_t
    L.nvfp4_scale_bytes.argtypes = [_c_i64, _c_i64]
    L.nvfp4_amax.restype = ctypes.c_int
    L.nvfp4_amax.argtypes = [_c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp]
    L.nvfp4_global_scale.restype = ctypes.c_int
    L.nvfp4_global_scale.argtypes = [_c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp]
    L.nvfp4_quantize.restype = ctypes.c_int
    L.nvfp4_quantize.argtypes = [_c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_vp, _c_vp]
    L.nvfp4_quantize_rows.restype = ctypes.c_int
    L.nvfp4_quantize_rows.argtypes = [_c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_vp, _c_i64, _c_i64, _c_vp]
    L.nvfp4_linear.restype = ctypes.c_int
    L.nvfp4_linear.argtypes = [ctypes.POINTER(Operand), _c_vp, ctypes.POINTER(Operand),
                               ctypes.POINTER(Segment), ctypes.c_int, ctypes.c_int,
                               ctypes.POINTER(EpilogueParams), _c_vp, ctypes.c_int, _c_i64, _c_vp]
    L.nvfp4_linear_splitk.restype = ctypes.c_int
    L.nvfp4_linear_splitk.argtypes = [ctypes.POINTER(Operand), _c_vp, ctypes.POINTER(Operand),
                                      ctypes.POINTER(Segment), ctypes.c_int, ctypes.c_int,
                                      ctypes.POINTER(EpilogueParams), _c_vp, ctypes.c_int, _c_i64,
                                      ctypes.c_int, _c_vp, ctypes.c_size_t, _c_vp]
    L.nvfp4_splitk_workspace_bytes.restype = ctypes.c_size_t
    L.nvfp4_splitk_workspace_bytes.argtypes = [_c_i64, _c_i64, ctypes.c_int]
    L.nvfp4_splitk_default.restype = ctypes.c_int
    L.nvfp4_splitk_default.argtypes = [_c_i64, _c_i64, _c_i64]
    L.nvfp4_linear_splitk_noalloc.restype = ctypes.c_int
    L.nvfp4_linear_splitk_noalloc.argtypes = [ctypes.POINTER(Operand), _c_vp, ctypes.POINTER(Operand),
                                              ctypes.POINTER(Segment), ctypes.c_int, ctypes.c_int,
                                              ctypes.POINTER(EpilogueParams), _c_vp, ctypes.c_int, _c_i64,
                                              ctypes.c_int, _c_vp]
    L.nvfp4_fold_segments.restype = ctypes.c_int
    L.nvfp4_fold_segments.argtypes = [_c_vp, _c_i64, _c_i64, ctypes.POINTER(Segment), ctypes.c_int, _c_vp, _c_vp]
    L.nvfp4_fp8_scale.restype = ctypes.c_int
    L.nvfp4_fp8_scale.argtypes = [_c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp]
    L.nvfp4_kv_cache_fp8.restype = ctypes.c_int
    L.nvfp4_kv_cache_fp8.argtypes = [_c_vp, _c_vp, _c_i64, _c_i64, _c_i64, _c_vp, _c_vp, _c_vp, _c_vp, _c_vp,
                                     _c_i64, _c_vp]
    L.nvfp4_gdn_recurrence.restype = ctypes.c_int
    L.nvfp4_gdn_recurrence.argtypes = [_c_vp, _c_vp, _c_i64, _c_vp, _c_i64, _c_vp, _c_vp, _c_i64, _c_vp, _c_i64,
                                       _c_i64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_vp, ctypes.c_int,
                                       _c_vp, _c_i64, ctypes.c_int, _c_vp]
    L.nvfp4_get_device_status.restype = ctypes.c_int
    L.nvfp4_get_device_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
    L.nvfp4_unswizzle_scales.restype = ctypes.c_int
    L.nvfp4_unswizzle_scales.argtypes = [_c_vp, _c_i64, _c_i64, _c_vp, _c_i64, _c_vp]
    L.nvfp4_pack_weight.restype = ctypes.c_int
    L.nvfp4_pack_weight.argtypes = [ctypes.POINTER(Operand), ctypes.c_int, _c_vp, _c_vp, _c_i64, _c_vp]
    L.nvfp4_selftest_stalled_linear.restype = ctypes.c_int
    L.nvfp4_selftest_stalled_linear.argtypes = [ctypes.POINTER(Operand), _c_vp, ctypes.POINTER(Operand),
                                                ctypes.POINTER(Segment), ctypes.c_int, _c_vp, _c_i64, ctypes.c_int,
                                                _c_vp]
    _LIB = L
    return L


def _lib_status_string(status: int) -> str:
    try:
        return lib().nvfp4_status_string(status).decode()
    except Exception:  # pragma: no cover - message formatting only
        return "status"


def _check(status: int, what: str):
    if status != 0:
        raise NVFP4Error(status, what)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return _c_vp(s.cuda_stream)


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def scale_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_scale_bytes(rows, cols))


@dataclass
class NVFP4Tensor:
    """A quantised [rows x cols] matrix: packed codes, swizzled scales, global scale (device)."""
    codes: "torch.Tensor"   # uint8 [rows, cols/2]
    scales: "torch.Tensor"  # uint8 [scale_bytes(rows, cols)]
    gs: "torch.Tensor"      # float32 [1]
    rows: int
    cols: int


def amax(x, out=None, stream=None):
    """max|x| of a 2-D BF16 CUDA tensor, as a float32 [1] device tensor (calibration)."""
    import torch
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().nvfp4_amax(_c_vp(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0), _c_vp(out.data_ptr()),
                            _stream(stream)), "nvfp4_amax")
    return out


def global_scale(x, out=None, stream=None):
    """gs = 2688 / max|x| of a 2-D BF16 CUDA tensor, as a float32 [1] device tensor."""
    import torch
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().nvfp4_global_scale(_c_vp(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0),
                                    _c_vp(out.data_ptr()), _stream(stream)), "nvfp4_global_scale")
    return out


def quantize(x, gs=None, codes=None, scales=None, stream=None) -> NVFP4Tensor:
    """NVFP4-quantise a 2-D BF16 CUDA tensor (row stride x.stride(0), unit column stride).

    ``gs``: float32 [1] device tensor (static scale); None computes it from x first.
    """
    import torch
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda and x.stride(1) == 1
    rows, cols = x.shape
    if gs is None:
        gs = global_scale(x, stream=stream)
    if codes is None:
        codes = torch.empty((rows, cols // 2), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(scale_bytes(rows, cols), 1), dtype=torch.uint8, device=x.device)
    _check(lib().nvfp4_quantize(_c_vp(x.data_ptr()), rows, cols, x.stride(0), _c_vp(gs.data_ptr()),
                                _c_vp(codes.data_ptr()), _c_vp(scales.data_ptr()), _stream(stream)),
           "nvfp4_quantize")
    return NVFP4Tensor(codes, scales, gs, rows, cols)


def quantize_fused(parts, gs_list=None, stream=None):
    """Quantise the modules of a fused weight, each with its own global scale, into one
    NVFP4 weight.  ``parts``: list of 2-D BF16 CUDA tensors (same cols).

    Returns ``(NVFP4Tensor, segments)`` with segments ``[(n_begin, n_end, gs), ...]``.
    """
    import torch
    cols = parts[0].shape[1]
    total = sum(p.shape[0] for p in parts)
    dev = parts[0].device
    codes = torch.empty((total, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(scale_bytes(total, cols), dtype=torch.uint8, device=dev)
    segs, n0 = [], 0
    for i, p in enumerate(parts):
        assert p.dtype == torch.bfloat16 and p.shape[1] == cols and p.stride(1) == 1
        gs = gs_list[i] if gs_list is not None else global_scale(p, stream=stream)
        _check(lib().nvfp4_quantize_rows(_c_vp(p.data_ptr()), p.shape[0], cols, p.stride(0),
                                         _c_vp(gs.data_ptr()), _c_vp(codes.data_ptr()),
                                         _c_vp(scales.data_ptr()), n0, total, _stream(stream)),
               "nvfp4_quantize_rows")
        segs.append((n0, n0 + p.shape[0], gs))
        n0 += p.shape[0]
    return NVFP4Tensor(codes, scales, segs[0][2], total, cols), segs


def _linear_args(a, w, segments, epilogue, out_dtype, out, ldo, gates, gs_out, out_scales):
    """Marshal the arguments shared by nvfp4_linear and nvfp4_linear_splitk."""
    import torch
    M, K = a.rows, a.cols
    N = w.rows
    if segments is None:
        segments = [(0, N, w.gs)]
    if len(segments) > MAX_SEGMENTS:
        raise ValueError("too many segments")
    segs = (Segment * len(segments))(*[Segment(int(n0), int(n1), _ptr(g)) for n0, n1, g in segments])
    nout = N // 2 if epilogue == "silu_mul" else N
    ep = EpilogueParams()
    if epilogue == "gdn_gates":
        g = gates or {}
        ep.beta_begin, ep.alpha_begin, ep.n_heads = int(g["beta_begin"]), int(g["alpha_begin"]), int(g["n_heads"])
        ep.A_log, ep.dt_bias = _ptr(g["A_log"]), _ptr(g["dt_bias"])
        ep.beta_out, ep.g_out = _ptr(g.get("beta_out")), _ptr(g.get("g_out"))
    if out_dtype == "nvfp4":
        if gs_out is None:
            raise ValueError("nvfp4 output needs gs_out")
        if out is None:
            out = torch.empty((M, nout // 2), dtype=torch.uint8, device=a.codes.device)
        if out_scales is None:
            out_scales = torch.empty(scale_bytes(M, nout), dtype=torch.uint8, device=a.codes.device)
        ep.gs_out, ep.out_scales = _ptr(gs_out), _ptr(out_scales)
        ldo = 0
        result = NVFP4Tensor(out, out_scales, gs_out, M, nout)
    else:
        dt = torch.bfloat16 if out_dtype == "bf16" else torch.float32
        if out is None:
            out = torch.empty((M, nout), dtype=dt, device=a.codes.device)
        ldo = out.stride(0) if ldo is None else ldo
        result = out
    A = Operand(a.codes.data_ptr(), a.scales.data_ptr(), M, K)
    W = Operand(w.codes.data_ptr(), w.scales.data_ptr(), N, w.cols)
    args = (ctypes.byref(A), _c_vp(a.gs.data_ptr()), ctypes.byref(W), segs, len(segments),
            EPILOGUES[epilogue], ctypes.byref(ep), _c_vp(out.data_ptr()), OUT_KINDS[out_dtype], int(ldo))
    keep = (A, W, segs, ep)  # keep the ctypes structures alive across the call
    return args, result, keep


def linear(a: NVFP4Tensor, w: NVFP4Tensor, segments: Optional[Sequence] = None, epilogue: str = "none",
           out_dtype: str = "bf16", out=None, ldo: Optional[int] = None, gates: Optional[dict] = None,
           gs_out=None, out_scales=None, stream=None):
    """Fused W4A4 linear ``epilogue(A @ W^T / (gs_a * gs_w[seg]))``.

    segments: list of ``(n_begin, n_end, gs_w_tensor)``; default one segment with ``w.gs``.
    gates (gdn_gates): dict with beta_begin, alpha_begin, n_heads, A_log, dt_bias
    [, beta_out, g_out] (float32 device tensors).
    out_dtype "nvfp4" returns an NVFP4Tensor quantised with ``gs_out``.
    """
    args, result, _keep = _linear_args(a, w, segments, epilogue, out_dtype, out, ldo, gates, gs_out, out_scales)
    _check(lib().nvfp4_linear(*args, _stream(stream)), "nvfp4_linear")
    return result


def splitk_default(M: int, N: int, K: int) -> int:
    return int(lib().nvfp4_splitk_default(M, N, K))


def splitk_workspace_bytes(M: int, N: int, split_k: int) -> int:
    return int(lib().nvfp4_splitk_workspace_bytes(M, N, split_k))


def linear_splitk(a: NVFP4Tensor, w: NVFP4Tensor, segments: Optional[Sequence] = None, epilogue: str = "none",
                  out_dtype: str = "bf16", out=None, ldo: Optional[int] = None, gates: Optional[dict] = None,
                  gs_out=None, out_scales=None, split_k: Optional[int] = None, workspace=None, stream=None):
    """``linear`` with K split over ``split_k`` units per output tile (decode regime).

    ``workspace``: a CUDA tensor of at least ``splitk_workspace_bytes(M, N, split_k)``
    bytes (allocated here when None).  ``split_k`` None: the library's choice.
    """
    import torch
    M, N, K = a.rows, w.rows, a.cols
    if split_k is None:
        split_k = splitk_default(M, N, K)
    need = splitk_workspace_bytes(M, N, split_k)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=a.codes.device)
    args, result, _keep = _linear_args(a, w, segments, epilogue, out_dtype, out, ldo, gates, gs_out, out_scales)
    _check(lib().nvfp4_linear_splitk(*args, int(split_k), _c_vp(workspace.data_ptr()),
                                     workspace.numel() * workspace.element_size(), _stream(stream)),
           "nvfp4_linear_splitk")
    return result


def noalloc_default_splits(M: int, N: int, K: int) -> int:
    """The library's default split count, lowered until the partial sums fit the fixed
    scratch array of ``linear_splitk_noalloc`` (never below 1; one split above 64 rows
    needs no scratch)."""
    s = max(splitk_default(M, N, K), 1)
    while s > 1 and splitk_workspace_bytes(M, N, s) > NOALLOC_SCRATCH_BYTES:
        s -= 1
    return s


def linear_splitk_noalloc(a: NVFP4Tensor, w: NVFP4Tensor, segments: Optional[Sequence] = None,
                          epilogue: str = "none", out_dtype: str = "bf16", out=None, ldo: Optional[int] = None,
                          gates: Optional[dict] = None, gs_out=None, out_scales=None,
                          split_k: Optional[int] = None, stream=None):
    """``linear_splitk`` whose partial sums live in the library's fixed scratch array
    (``NOALLOC_SCRATCH_BYTES``), for callers that cannot hand in a workspace.

    The library allocates nothing for it (the output buffers allocated here when
    ``out`` / ``out_scales`` are None are this wrapper's, not the entry point's).
    Calls that overlap on the GPU share the scratch and race: serialise them.
    """
    M, N, K = a.rows, w.rows, a.cols
    if split_k is None:
        split_k = noalloc_default_splits(M, N, K)
    args, result, _keep = _linear_args(a, w, segments, epilogue, out_dtype, out, ldo, gates, gs_out, out_scales)
    _check(lib().nvfp4_linear_splitk_noalloc(*args, int(split_k), _stream(stream)), "nvfp4_linear_splitk_noalloc")
    return result


def unswizzle_scales(t: NVFP4Tensor, out=None, stream=None):
    """The E4M3 block scales of ``t`` in logical order: uint8 [rows, cols/16] (device)."""
    import torch
    if out is None:
        out = torch.empty((t.rows, t.cols // 16), dtype=torch.uint8, device=t.scales.device)
    _check(lib().nvfp4_unswizzle_scales(_c_vp(t.scales.data_ptr()), t.rows, t.cols, _c_vp(out.data_ptr()),
                                        out.stride(0), _stream(stream)), "nvfp4_unswizzle_scales")
    return out


def pack_weight(parts: Sequence[NVFP4Tensor], rows_out: Optional[int] = None, stream=None):
    """Pack separately quantised modules (same cols) into one fused NVFP4 weight of
    ``rows_out`` rows (default: their total; extra rows are zero padding).  Returns
    ``(NVFP4Tensor, segments)`` with segments ``[(row0, row1, gs), ...]`` of the modules."""
    import torch
    cols = parts[0].cols
    total = sum(p.rows for p in parts)
    rows_out = total if rows_out is None else rows_out
    dev = parts[0].codes.device
    codes = torch.empty((rows_out, cols // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty(scale_bytes(rows_out, cols), dtype=torch.uint8, device=dev)
    ops = (Operand * len(parts))(*[Operand(p.codes.data_ptr(), p.scales.data_ptr(), p.rows, p.cols) for p in parts])
    _check(lib().nvfp4_pack_weight(ops, len(parts), _c_vp(codes.data_ptr()), _c_vp(scales.data_ptr()), rows_out,
                                   _stream(stream)), "nvfp4_pack_weight")
    segs, n0 = [], 0
    for p in parts:
        segs.append((n0, n0 + p.rows, p.gs))
        n0 += p.rows
    return NVFP4Tensor(codes, scales, parts[0].gs, rows_out, cols), segs


def fold_segments(w: NVFP4Tensor, segments: Sequence, gs_out=None, stream=None):
    """Fused-group repair in place: one global scale for all modules of ``w`` (the
    ratios folded into its block scales).  Returns the common scale (float32 [1] device
    tensor); afterwards ``linear(a, w, segments=[(0, w.rows, gs)])`` serves the weight."""
    import torch
    if gs_out is None:
        gs_out = torch.empty(1, dtype=torch.float32, device=w.codes.device)
    segs = (Segment * len(segments))(*[Segment(int(n0), int(n1), _ptr(g)) for n0, n1, g in segments])
    _check(lib().nvfp4_fold_segments(_c_vp(w.scales.data_ptr()), w.rows, w.cols, segs, len(segments),
                                     _c_vp(gs_out.data_ptr()), _stream(stream)), "nvfp4_fold_segments")
    return gs_out


def fp8_scale(x, out=None, stream=None):
    """Calibrated FP8 scale max|x| / 448 of a 2-D BF16 CUDA tensor (float32 [1] device tensor)."""
    import torch
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=x.device)
    _check(lib().nvfp4_fp8_scale(_c_vp(x.data_ptr()), x.shape[0], x.shape[1], x.stride(0), _c_vp(out.data_ptr()),
                                 _stream(stream)), "nvfp4_fp8_scale")
    return out


def kv_cache_fp8(k, v, k_scale, v_scale, slots, k_cache, v_cache, stream=None):
    """Write K / V token rows (BF16 [tokens, width]) into FP8 caches ([num_slots, width]
    uint8) at ``slots`` (int64 [tokens], negative = skip) with static scales."""
    import torch
    assert k.shape == v.shape and k.stride() == v.stride() and k.dtype == torch.bfloat16
    assert slots.dtype == torch.int64 and k_cache.shape == v_cache.shape
    _check(lib().nvfp4_kv_cache_fp8(_c_vp(k.data_ptr()), _c_vp(v.data_ptr()), k.shape[0], k.shape[1], k.stride(0),
                                    _c_vp(k_scale.data_ptr()), _c_vp(v_scale.data_ptr()), _c_vp(slots.data_ptr()),
                                    _c_vp(k_cache.data_ptr()), _c_vp(v_cache.data_ptr()), k_cache.shape[0],
                                    _stream(stream)), "nvfp4_kv_cache_fp8")


def gdn_recurrence(q, k, v, g, beta, cu_seqlens, state, *, initial_state=True, out=None, out_dtype="bf16",
                   stream=None):
    """Gated delta-rule recurrence of the GDN layers over packed sequences.

    q, k: BF16 [tokens, H_k * 128] (row-strided views allowed, e.g. column ranges of the
    fused in-projection output); v: BF16 [tokens, H_v * 128]; g, beta: FP32 [tokens, H_v]
    (row-strided, as the gate epilogue writes them); cu_seqlens: int32 [n_seqs + 1];
    state: FP32 [n_seqs, H_v, 128, 128] with state[s, h, j, i] = S[i, j], read as the
    initial state when ``initial_state`` and overwritten with the final one.  Returns
    out [tokens, H_v * 128] (BF16 or FP32), out[t, h*128 + j] = (S_t^T q_t)_j."""
    import torch
    tokens = q.shape[0]
    hk, hv = q.shape[1] // 128, v.shape[1] // 128
    assert q.dtype == k.dtype == v.dtype == torch.bfloat16 and q.shape == k.shape and q.stride() == k.stride()
    assert q.stride(1) == 1 and v.stride(1) == 1 and v.shape[0] == tokens
    assert g.dtype == beta.dtype == torch.float32 and g.stride() == beta.stride() and g.shape[1] >= hv
    assert cu_seqlens.dtype == torch.int32 and state.dtype == torch.float32 and state.is_contiguous()
    n_seqs = cu_seqlens.shape[0] - 1
    assert state.shape == (n_seqs, hv, 128, 128)
    if out_dtype not in ("bf16", "f32"):
        raise ValueError(f"out_dtype must be 'bf16' or 'f32', not {out_dtype!r}")
    kind = OUT_KINDS[out_dtype]
    if out is None:
        out = torch.empty((tokens, hv * 128), device=q.device,
                          dtype=torch.bfloat16 if out_dtype == "bf16" else torch.float32)
    _check(lib().nvfp4_gdn_recurrence(_c_vp(q.data_ptr()), _c_vp(k.data_ptr()), q.stride(0), _c_vp(v.data_ptr()),
                                      v.stride(0), _c_vp(g.data_ptr()), _c_vp(beta.data_ptr()), g.stride(0),
                                      _c_vp(cu_seqlens.data_ptr()), n_seqs, tokens, hk, hv, 128,
                                      _c_vp(state.data_ptr()), int(bool(initial_state)), _c_vp(out.data_ptr()),
                                      out.stride(0), kind, _stream(stream)), "nvfp4_gdn_recurrence")
    return out


def device_status() -> int:
    """Read and clear the device status word (synchronises the device)."""
    code = ctypes.c_int(0)
    _check(lib().nvfp4_get_device_status(ctypes.byref(code)), "nvfp4_get_device_status")
    return code.value


def selftest_stalled_linear(a: NVFP4Tensor, w: NVFP4Tensor, stall_stage: int, stream=None):
    """Run the failure-detection self-test (``nvfp4_selftest_stalled_linear``): the 1-CTA
    GEMM with K tile ``stall_stage`` never loaded and short wait limits.  Returns the
    (meaningless) FP32 output; the timeout shows in ``device_status()``."""
    import torch
    out = torch.zeros((a.rows, w.rows), dtype=torch.float32, device=a.codes.device)
    segs = (Segment * 1)(Segment(0, w.rows, w.gs.data_ptr()))
    A = Operand(a.codes.data_ptr(), a.scales.data_ptr(), a.rows, a.cols)
    W = Operand(w.codes.data_ptr(), w.scales.data_ptr(), w.rows, w.cols)
    _check(lib().nvfp4_selftest_stalled_linear(ctypes.byref(A), _c_vp(a.gs.data_ptr()), ctypes.byref(W), segs, 1,
                                               _c_vp(out.data_ptr()), out.stride(0), int(stall_stage),
                                               _stream(stream)), "nvfp4_selftest_stalled_linear")
    return out
