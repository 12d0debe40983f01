"""CPU oracle for the NVFP4 W4A4 linear.  TEST INFRASTRUCTURE, NOT PRODUCT CODE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference arm may import anything from ``oracle/``.  The library under
``nvfp4_w4a4_quantized_02_b200/`` never imports it and shares no code with it.

It is a plain, slow, obviously correct restatement of what the W4A4 linear
computes, written from these pages:

* Blog "27BハイブリッドLLMを4ビットで動かす——Gated DeltaNetはなぜ量子化に耐えるのか"
  (gotosocial), section 機構① (NVFP4 = E2M1 4-bit values plus one E4M3 scale per
  16 elements; the block maximum sets the scale), section 機構② (the gates
  g = -exp(A_log) * softplus(a + dt_bias) and beta = sigmoid(b)), section 罠①
  (per-module global scales clash when modules are fused into one GEMM), FAQ
  (W4A4 needs 4-bit tensor cores).
* Abstract page "Why Gated DeltaNet Survives 4-Bit Quantization" (fugumt,
  arXiv 2609.04098): 16-element block scaling; the global-scale mismatch of fused
  GEMMs.

The pages fix neither a rounding mode, nor an operation order, nor a global-scale
formula.  The readings taken here are:

R1  global scale gs = fl32(2688 / amax(|x|)), 2688 = 448 (E4M3 max) * 6 (E2M1 max);
    dequantisation divides by gs; amax == 0 gives gs = 1.
R2  per 16-element block: s = fl32(fl32(amax_b / 6) * gs); sf = E4M3(s) rounded to
    nearest, ties to even, saturating at 448; inv = 0 if sf == 0 else fl32(gs / dec(sf));
    v = fl32(x * inv); code = E2M1(v) rounded to nearest, ties to even, saturating
    at 6, sign bit copied from v (so a negative value that rounds to zero is -0).
R3  the linear: Y[m, n] = alpha(n) * sum_k Ahat[m, k] * What[n, k] with
    Ahat = e2m1(code) * dec(sf) (no global scale) and alpha(n) = 1 / (gs_A * gs_W[seg(n)]),
    the per-segment correction of a fused GEMM; accumulated in FP64.
R4  epilogues in FP64: SiLU(gate) * up; beta = sigmoid; g = -exp(A_log) * softplus(a + dt_bias)
    with softplus(x) = max(x, 0) + log1p(exp(-|x|)).
R5  re-quantising an output for the next layer first rounds it to BF16 (nearest even).
R13 FP8 KV cache (blog section "KVキャッシュはFP8で十分？": static FP8 scales, one per
    K and one per V tensor of each attention layer, calibrated and shipped with the
    checkpoint): the reciprocal of the shipped scale is taken once, inv = fl32(1 /
    scale), and a cached value is E4M3(fl32(x * inv)), nearest even, saturating at
    +-448, sign kept; it decodes to e4m3 * scale.  A calibrated scale is
    fl32(amax / 448) (amax 0 gives 1).  Token t is written to cache row slots[t]; a
    negative slot skips the token.
R12 fused-group repair (blog section 罠①: the fused group is rewritten to a common
    global scale and the ratio is folded into the block scales, re-rounding error
    <= 6.2 %): the common scale is the smallest segment scale, gs_c = min gs_seg, so
    every ratio is <= 1 and no block scale saturates; each block scale becomes
    sf' = E4M3(fl32(dec(sf) * fl32(gs_c / gs_seg))), nearest even; codes are kept.
R14 GDN recurrence (blog section "Gated DeltaNetの仕組み"): per value head, a state
    S in R^{d_k x d_v} evolves as S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T
    with alpha_t = exp(g_t), g and beta the gate outputs of the in-projection's
    epilogue (R4).  The pages give no read-out: o_t = S_t^T q_t (the state read with the
    query, after the update).  q and k are taken as given (the model's short
    convolution and normalisation are neither linears nor on the pages); value head h
    reads key head h // (H_v / H_k).

Float32 steps (R1, R2) use numpy float32 scalars/arrays, whose +, *, / are IEEE-754
single precision, round to nearest even: the same operations a correct kernel
performs.  Encoding decisions (nearest E4M3 / E2M1 value) are taken on those exact
float32 values by nearest-neighbour search over the format's value table.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "E2M1_MAX", "E4M3_MAX", "GS_NUMERATOR",
    "e2m1_decode", "e2m1_encode", "e4m3_decode", "e4m3_encode",
    "global_scale", "quantize", "dequantize", "block_scaled_matmul", "linear",
    "silu", "sigmoid", "softplus", "silu_mul", "gdn_gates", "round_to_bf16",
    "fold_segments", "e4m3_encode_signed", "fp8_scale", "kv_cache_fp8", "gdn_recurrence",
]

E2M1_MAX = 6.0
E4M3_MAX = 448.0
GS_NUMERATOR = np.float32(E4M3_MAX * E2M1_MAX)  # 2688, reading R1
BLOCK = 16


# --------------------------------------------------------------------------- E2M1
def e2m1_decode(code) -> np.ndarray:
    """Value of a 4-bit E2M1 code: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.

    Exponent 0 is subnormal: value = mantissa * 0.5.  Otherwise 2**(e-1) * (1 + m/2).
    """
    c = np.asarray(code, dtype=np.int64)
    s = (c >> 3) & 1
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, m * 0.5, np.ldexp(1.0 + m * 0.5, (e - 1).astype(np.int64)))
    return np.where(s == 1, -mag, mag).astype(np.float64)


# magnitude of code 0..7, ascending with the code
_E2M1_MAGS = e2m1_decode(np.arange(8))


def _nearest_even(a: np.ndarray, table: np.ndarray) -> np.ndarray:
    """Index of the entry of the ascending ``table`` nearest to each ``a`` (a >= 0).

    Ties between the two neighbours go to the even index (the code whose mantissa
    LSB is 0); values above the last entry go to the last entry (saturation).
    """
    a = np.asarray(a, dtype=np.float64)
    hi = np.searchsorted(table, a, side="left")
    hi = np.minimum(hi, len(table) - 1)
    lo = np.maximum(hi - 1, 0)
    d_lo = np.abs(a - table[lo])
    d_hi = np.abs(table[hi] - a)
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    # at or beyond the largest entry the result saturates to it (decided by comparison,
    # not by distances, which stop being distinguishable in FP64 for huge inputs)
    idx = np.where(a >= table[-1], len(table) - 1, idx)
    return idx.astype(np.int64)


def e2m1_encode(v) -> np.ndarray:
    """E2M1 code of each value: nearest magnitude, ties to even code, saturating at 6.

    The sign bit is copied from the input (reading R2), so -0.0 and negative values
    that round to zero encode as 0x8.
    """
    v = np.asarray(v, dtype=np.float64)
    if not np.all(np.isfinite(v)):
        raise ValueError("e2m1_encode: non-finite input")
    idx = _nearest_even(np.abs(v), _E2M1_MAGS)
    return (idx | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


# --------------------------------------------------------------------------- E4M3
def e4m3_decode(byte) -> np.ndarray:
    """Value of an 8-bit E4M3 pattern: sign bit 7, exponent bits 6..3 (bias 7), mantissa 2..0.

    Exponent 0 is subnormal (m/8 * 2**-6); S.1111.111 is NaN; no infinities.
    """
    b = np.asarray(byte, dtype=np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 15
    m = b & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return np.where(s == 1, -mag, mag).astype(np.float64)


# finite non-negative E4M3 values, code 0x00..0x7E, ascending with the code
_E4M3_POS = e4m3_decode(np.arange(0x7F))


def e4m3_encode(s) -> np.ndarray:
    """Unsigned E4M3 scale byte: nearest finite value, ties to even code, saturating at 448."""
    s = np.asarray(s, dtype=np.float64)
    if not np.all(np.isfinite(s)) or np.any(s < 0):
        raise ValueError("e4m3_encode: scale must be finite and >= 0")
    return _nearest_even(s, _E4M3_POS).astype(np.uint8)


# ----------------------------------------------------------------- quantisation
def global_scale(x) -> np.float32:
    """Per-tensor FP32 global scale gs = fl32(2688 / amax|x|); amax 0 gives 1 (reading R1)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(GS_NUMERATOR / amax)


def quantize(x, gs):
    """NVFP4 block quantisation of a float32 matrix ``x [rows, cols]`` (cols % 16 == 0).

    Returns ``(codes uint8 [rows, cols], sf uint8 [rows, cols/16])``: one E2M1 code
    per element (not packed) and one E4M3 scale per 16-element row block (logical
    order, not swizzled).  Steps follow reading R2.
    """
    x = np.asarray(x, dtype=np.float32)
    gs = np.float32(gs)
    rows, cols = x.shape
    if cols % BLOCK:
        raise ValueError("cols must be a multiple of 16")
    if not np.all(np.isfinite(x)):
        raise ValueError("quantize: non-finite input")
    xb = x.reshape(rows, cols // BLOCK, BLOCK)
    amax_b = np.max(np.abs(xb), axis=2)                               # exact
    s = (amax_b / np.float32(E2M1_MAX)).astype(np.float32) * gs       # two fl32 roundings
    s = s.astype(np.float32)
    sf = e4m3_encode(s)
    dec = e4m3_decode(sf).astype(np.float32)                          # exact in fp32
    with np.errstate(divide="ignore"):
        inv = np.where(dec == 0, np.float32(0), gs / np.where(dec == 0, np.float32(1), dec))
    inv = inv.astype(np.float32)
    v = (xb * inv[:, :, None]).astype(np.float32)
    codes = e2m1_encode(v).reshape(rows, cols)
    return codes, sf


def dequantize(codes, sf, gs=1.0) -> np.ndarray:
    """FP64 value of quantised data: e2m1(code) * dec(sf) / gs."""
    codes = np.asarray(codes)
    sf = np.asarray(sf)
    rows, cols = codes.shape
    scale = np.repeat(e4m3_decode(sf), BLOCK, axis=1)[:, :cols]
    return e2m1_decode(codes) * scale / np.float64(gs)


def block_scaled_matmul(a_codes, a_sf, w_codes, w_sf) -> np.ndarray:
    """acc[m, n] = sum_k e2m1(A)[m,k] dec(sfA)[m,k/16] e2m1(W)[n,k] dec(sfW)[n,k/16], in FP64."""
    A = dequantize(a_codes, a_sf)
    W = dequantize(w_codes, w_sf)
    return A @ W.T


def linear(a_codes, a_sf, gs_a, w_codes, w_sf, segments) -> np.ndarray:
    """Fused W4A4 linear with per-segment global-scale correction (reading R3).

    ``segments`` is a list of ``(n_begin, n_end, gs_w)`` covering the output columns;
    column n of the result is ``acc[:, n] / (gs_a * gs_w(seg(n)))``.
    """
    acc = block_scaled_matmul(a_codes, a_sf, w_codes, w_sf)
    n = acc.shape[1]
    alpha = np.full(n, np.nan)
    for n0, n1, gs_w in segments:
        alpha[n0:n1] = 1.0 / (np.float64(gs_a) * np.float64(gs_w))
    if np.any(np.isnan(alpha)):
        raise ValueError("segments do not cover every output column")
    return acc * alpha[None, :]


# -------------------------------------------------------------------- epilogues
def sigmoid(x):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-x))


def softplus(x):
    """Stable softplus: max(x, 0) + log1p(exp(-|x|))."""
    x = np.asarray(x, dtype=np.float64)
    return np.maximum(x, 0.0) + np.log1p(np.exp(-np.abs(x)))


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x * sigmoid(x)


def silu_mul(gate, up):
    """MLP activation h = SiLU(gate) * up."""
    return silu(gate) * np.asarray(up, dtype=np.float64)


def gdn_gates(b, a, a_log, dt_bias):
    """Gated DeltaNet gates from the b/a projections (blog section 機構②).

    beta = sigmoid(b); g = -exp(A_log[h]) * softplus(a + dt_bias[h]); h = column (head).
    """
    b = np.asarray(b, dtype=np.float64)
    a = np.asarray(a, dtype=np.float64)
    a_log = np.asarray(a_log, dtype=np.float64)
    dt_bias = np.asarray(dt_bias, dtype=np.float64)
    beta = sigmoid(b)
    g = -np.exp(a_log)[None, :] * softplus(a + dt_bias[None, :])
    return beta, g


def round_to_bf16(x) -> np.ndarray:
    """Round FP64 values to the nearest BF16 value (8 significant bits), ties to even.

    Direct from the exact value (no intermediate float32 rounding).  Normal range only.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                    # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


# ------------------------------------------------------------ fused-group repair
def fold_segments(sf_segments, gs_segments):
    """Re-express the modules of a fused weight with one global scale (reading R12).

    ``sf_segments``: list of logical block-scale arrays (uint8 [rows_i, cols/16]), one per
    module; ``gs_segments``: the modules' global scales.  Returns ``(sf_folded_list, gs_c)``.
    The value a block decodes to, e2m1 * dec(sf') / gs_c, then differs from
    e2m1 * dec(sf) / gs_seg only by the re-rounding of the E4M3 scale.
    """
    gs = [np.float32(g) for g in gs_segments]
    gs_c = np.float32(min(gs))
    out = []
    for sf, g in zip(sf_segments, gs):
        ratio = np.float32(gs_c / g)                      # one fl32 division
        s = (e4m3_decode(sf).astype(np.float32) * ratio).astype(np.float32)
        out.append(e4m3_encode(s))
    return out, gs_c


# ------------------------------------------------------------------ FP8 KV cache
def e4m3_encode_signed(v) -> np.ndarray:
    """Signed E4M3 byte: nearest finite magnitude, ties to even code, saturating at 448,
    sign bit 7 copied from the input (so -0.0 -> 0x80)."""
    v = np.asarray(v, dtype=np.float64)
    if not np.all(np.isfinite(v)):
        raise ValueError("e4m3_encode_signed: non-finite input")
    mag = _nearest_even(np.abs(v), _E4M3_POS)
    return (mag | (np.signbit(v).astype(np.int64) << 7)).astype(np.uint8)


def fp8_scale(x) -> np.float32:
    """Calibrated per-tensor FP8 scale fl32(amax|x| / 448); 1 for an all-zero tensor (R13)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x))) if x.size else np.float32(0)
    return np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(E4M3_MAX))


def kv_cache_fp8(x, scale, slots, num_slots, cache=None) -> np.ndarray:
    """Write token rows of ``x [tokens, width]`` into an FP8 cache ``[num_slots, width]``
    (uint8): row slots[t] = E4M3(fl32(x[t] * fl32(1 / scale))); slots < 0 are skipped (R13)."""
    x = np.asarray(x, dtype=np.float32)
    tokens, width = x.shape
    out = np.zeros((num_slots, width), np.uint8) if cache is None else np.array(cache, dtype=np.uint8)
    inv = np.float32(np.float32(1.0) / np.float32(scale))
    q = e4m3_encode_signed((x * inv).astype(np.float32))
    for t in range(tokens):
        if slots[t] >= 0:
            out[slots[t]] = q[t]
    return out


# ---------------------------------------------------------------- GDN recurrence
def gdn_recurrence(q, k, v, g, beta, state=None):
    """Gated delta-rule recurrence of one sequence, in FP64 (reading R14).

    q, k: [T, H_k, d_k]; v: [T, H_v, d_v]; g, beta: [T, H_v]; state: [H_v, d_k, d_v] or
    None (zeros).  Returns (o [T, H_v, d_v], final state).  Token by token, as written:
    S <- exp(g) S + beta k (v - S^T k)^T ;  o = S^T q.
    """
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    g = np.asarray(g, np.float64)
    beta = np.asarray(beta, np.float64)
    T, hk, dk = k.shape
    hv, dv = v.shape[1], v.shape[2]
    if hv % hk:
        raise ValueError("value heads must be a multiple of key heads")
    rep = hv // hk
    S = np.zeros((hv, dk, dv)) if state is None else np.array(state, np.float64)
    o = np.empty((T, hv, dv))
    for t in range(T):
        kt = np.repeat(k[t], rep, axis=0)                  # [H_v, d_k]
        qt = np.repeat(q[t], rep, axis=0)
        pred = np.einsum("hij,hi->hj", S, kt)              # S^T k
        upd = beta[t][:, None] * (v[t] - pred)             # beta (v - S^T k)
        S = np.exp(g[t])[:, None, None] * S + kt[:, :, None] * upd[:, None, :]
        o[t] = np.einsum("hij,hi->hj", S, qt)              # S^T q
    return o, S
