"""Seeded synthetic inputs for the NVFP4 W4A4 linear workloads.

This module is shared by the CPU oracle (``oracle/``) and the CUDA path (tests and
bench feed the same arrays to both).  It holds NONE of the method's arithmetic:
no global scale, no block scale, no E2M1/E4M3 encoding, no GEMM.  It only draws
random numbers and rounds them to BF16, the storage type of activations and
weights.

Every generator returns BF16 *bit patterns* as ``np.uint16`` arrays.  ``bf16_to_f32``
widens them to float32 exactly (a BF16 value is a float32 with 16 zero low bits),
which is what the oracle consumes; the GPU side reinterprets the same bits as a
``torch.bfloat16`` tensor.

Distributions follow the workloads the method is measured on:

* activations with sparse huge outliers (0.1 % of entries x50) for the small linear
  and the GDN in-projection;
* heavy-tailed residual-stream activations: Student-t (nu=3) plus 8 fixed hot
  channels x100, standing in for the max/RMS ~ 63.5, hot-channel ~ 100x median
  statistics the blog reports in its block-scaling mechanism section
  ("27BハイブリッドLLMを4ビットで動かす", section 機構①);
* weights ~ N(0, 0.02), with per-segment multipliers where a fused module's
  segments must carry global scales that differ (up to 16x);
* GDN recurrence inputs: unit-norm q / k heads, N(0,1) values, log-decays g <= 0 whose
  per-head rates span the short to the very long memory horizons the blog's recurrence
  section mentions (tens of thousands of tokens), write strengths beta in (0, 1).
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "f32_to_bf16_bits", "bf16_to_f32", "outlier_activations", "student_t_activations",
    "gaussian_weights", "segmented_weights", "gdn_gate_params", "gdn_recurrence_inputs",
    "GDN_INPROJ_SEGMENTS", "GDN_INPROJ_MULTIPLIERS",
]


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (round-to-nearest-even) and return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    if not np.all(np.isfinite(x)):
        raise ValueError("synthetic inputs must be finite")
    u = x.view(np.uint32).astype(np.uint64)
    lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = (u + np.uint64(0x7FFF) + lsb) >> np.uint64(16)
    return u.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen BF16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_activations(rows: int, cols: int, seed: int = 0, frac: float = 1e-3,
                        factor: float = 50.0) -> np.ndarray:
    """N(0,1) activations with ``round(frac*rows*cols)`` entries (a seeded permutation) scaled by ``factor``."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols), dtype=np.float32)
    n_out = int(round(frac * rows * cols))
    if n_out:
        idx = rng.permutation(rows * cols)[:n_out]
        x.reshape(-1)[idx] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def student_t_activations(rows: int, cols: int, seed: int = 0, nu: float = 3.0,
                          scale: float = 1.0, hot_channels: int = 8,
                          hot_factor: float = 100.0) -> np.ndarray:
    """Student-t(nu) activations times ``scale``; ``hot_channels`` seeded columns times ``hot_factor``."""
    rng = np.random.default_rng(seed)
    hot = rng.choice(cols, size=hot_channels, replace=False) if hot_channels else []
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, (1 << 24) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = (rng.standard_t(nu, size=(r1 - r0, cols)) * scale).astype(np.float32)
        if hot_channels:
            x[:, hot] *= np.float32(hot_factor)
        out[r0:r1] = f32_to_bf16_bits(x)
    return out


def gaussian_weights(rows: int, cols: int, seed: int = 1, std: float = 0.02) -> np.ndarray:
    """Weights ~ N(0, std) as BF16 bits, ``[rows, cols]`` (out_features x in_features)."""
    rng = np.random.default_rng(seed)
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, (1 << 24) // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        w = rng.standard_normal((r1 - r0, cols), dtype=np.float32) * np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(w)
    return out


# GDN fused in-projection: q | k | v | z | beta | alpha rows (out features) and the
# multipliers that make the segments' amaxes (hence global scales) differ by up to 16x.
GDN_INPROJ_SEGMENTS = (("q", 2048), ("k", 2048), ("v", 4096), ("z", 4096), ("beta", 32), ("alpha", 32))
GDN_INPROJ_MULTIPLIERS = {"q": 1.0, "k": 2.0, "v": 4.0, "z": 8.0, "beta": 16.0, "alpha": 1.0}


def segmented_weights(segments, cols: int, seed: int = 1, std: float = 0.02,
                      multipliers=None) -> list:
    """One BF16 weight per segment ``(name, rows)``; segment i is drawn with seed ``seed + i``.

    Returns a list of ``(name, bits[rows, cols])``.
    """
    multipliers = multipliers or {}
    out = []
    for i, (name, rows) in enumerate(segments):
        m = float(multipliers.get(name, 1.0))
        out.append((name, gaussian_weights(rows, cols, seed=seed + i, std=std * m)))
    return out


def gdn_gate_params(n_heads: int = 32, seed: int = 7):
    """``A_log`` and ``dt_bias`` ~ N(0,1), one float32 per head."""
    rng = np.random.default_rng(seed)
    a_log = rng.standard_normal(n_heads).astype(np.float32)
    dt_bias = rng.standard_normal(n_heads).astype(np.float32)
    return a_log, dt_bias


def gdn_recurrence_inputs(seq_lens, n_key_heads: int = 16, n_value_heads: int = 32, seed: int = 11,
                          ld: int | None = None, head_dim: int = 128):
    """Packed sequences of GDN recurrence inputs laid out like the fused in-projection's
    output rows: q at column 0, k at n_key_heads * head_dim, v after k; row width ``ld``
    (default: just q | k | v).

    q, k: each head an i.i.d. Gaussian vector scaled to unit length, then rounded to
    BF16; v ~ N(0, 1) in BF16; g[t, h] = -c_h * U(0.5, 1.5) with per-head rates c_h
    log-uniform in [2e-5, 0.5] (float32); beta ~ U(0.05, 1) (float32).
    Returns dict(rows=uint16 [T, ld], q_col, k_col, v_col, g, beta, cu_seqlens=int32)."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(seq_lens, np.int64)
    T = int(lens.sum())
    wk, wv = n_key_heads * head_dim, n_value_heads * head_dim
    ld = 2 * wk + wv if ld is None else ld
    assert ld >= 2 * wk + wv
    rows = np.zeros((T, ld), np.uint16)
    for col in (0, wk):
        x = rng.standard_normal((T, n_key_heads, head_dim))
        x /= np.linalg.norm(x, axis=-1, keepdims=True)
        rows[:, col:col + wk] = f32_to_bf16_bits(x.reshape(T, wk).astype(np.float32))
    rows[:, 2 * wk:2 * wk + wv] = f32_to_bf16_bits(rng.standard_normal((T, wv)).astype(np.float32))
    rate = np.exp(rng.uniform(np.log(2e-5), np.log(0.5), n_value_heads))
    g = (-rate[None, :] * rng.uniform(0.5, 1.5, (T, n_value_heads))).astype(np.float32)
    beta = rng.uniform(0.05, 1.0, (T, n_value_heads)).astype(np.float32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return dict(rows=rows, q_col=0, k_col=wk, v_col=2 * wk, g=g, beta=beta, cu_seqlens=cu)
