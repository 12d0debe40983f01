"""Pins for the CPU oracle: format facts, brute force, closed forms and invariants.

Nothing here re-types the oracle's formulas: every expectation comes from the
format definition (golden file), an exhaustive search, an exact special case or
a mathematical identity, chosen so that a dropped term, a wrong sign, a wrong
index or a transposed operand in the oracle fails at least one test.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import layout
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_format_facts.json")


@pytest.fixture(scope="module")
def facts():
    with open(GOLDEN) as f:
        return json.load(f)


# ------------------------------------------------------------------ E2M1 pins
def test_e2m1_decode_matches_value_set(facts):
    vals = oracle.e2m1_decode(np.arange(16))
    want = np.array(facts["e2m1_values_by_code"])
    assert np.array_equal(vals, want)
    assert np.array_equal(np.signbit(vals), np.signbit(want))


def _brute_e2m1(v):
    """Nearest of the 8 magnitudes by exhaustive search in exact rational arithmetic;
    ties to the even code."""
    mags = [Fraction(abs(x)) for x in json.load(open(GOLDEN))["e2m1_values_by_code"][:8]]
    best = None
    for code, m in enumerate(mags):
        d = abs(abs(Fraction(v)) - m)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    code = best[1]
    if math.copysign(1.0, v) < 0:
        code |= 8
    return code


def test_e2m1_encode_brute_force_sweep():
    # dense sweep over [-8, 8] including every midpoint and every representable value
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    grid = np.unique(np.concatenate([np.linspace(-8, 8, 4097), mids, -mids,
                                     [6.0, 7.0, 1e6, -1e6, 0.2499999, 0.2500001,
                                      1e18, -2.7e18, 3e38, -3e38, 1e300]]))
    got = oracle.e2m1_encode(grid)
    want = np.array([_brute_e2m1(float(v)) for v in grid], dtype=np.uint8)
    assert np.array_equal(got, want)


def test_e2m1_threshold_table(facts):
    rules = facts["e2m1_round_to_nearest_even_thresholds"]["rules"]
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(0, 8, 20000),
                        np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])])
    got = np.abs(oracle.e2m1_decode(oracle.e2m1_encode(v)))
    for x, g in zip(v, got):
        for op, t, mag in rules:
            if op == "else" or (op == "<=" and x <= t) or (op == "<" and x < t):
                assert g == mag, (x, g, mag)
                break


def test_e2m1_sign_of_zero():
    assert oracle.e2m1_encode(np.array([-0.0]))[0] == 0x8
    assert oracle.e2m1_encode(np.array([-0.1]))[0] == 0x8
    assert oracle.e2m1_encode(np.array([0.1]))[0] == 0x0
    assert oracle.e2m1_encode(np.array([-0.3]))[0] == 0x9


# ------------------------------------------------------------------ E4M3 pins
def test_e4m3_known_values(facts):
    for hexs, val in facts["e4m3_known"]:
        d = oracle.e4m3_decode(int(hexs, 16))
        assert d == val and np.signbit(d) == np.signbit(val), hexs
    for hexs in facts["e4m3_nan"]:
        assert np.isnan(oracle.e4m3_decode(int(hexs, 16)))
    pos = oracle.e4m3_decode(np.arange(1, 128))
    assert np.sum(np.isfinite(pos) & (pos > 0)) == facts["e4m3_finite_positive_count"]
    # strictly increasing with the code over the finite non-negative range
    fin = oracle.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(fin) > 0)


_E4M3_TABLE = [Fraction(float(oracle.e4m3_decode(c))) for c in range(0x7F)]


def _brute_e4m3(s):
    """Nearest finite E4M3 by exhaustive search in exact rational arithmetic; ties to even."""
    best = None
    s = Fraction(s)
    for code, val in enumerate(_E4M3_TABLE):
        d = abs(s - val)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0):
            best = (d, code)
    return best[1]


def test_e4m3_encode_brute_force():
    rng = np.random.default_rng(5)
    fin = oracle.e4m3_decode(np.arange(0x7F))
    mids = (fin[1:] + fin[:-1]) / 2
    s = np.concatenate([rng.uniform(0, 500, 3000), np.exp(rng.uniform(-14, 6.5, 3000)),
                        mids, fin, [448.0, 449.0, 464.0, 480.0, 1e9, 0.0, 2.0 ** -10, 2.0 ** -11,
                                    2.0e20, 3.0e38]])
    s = s.astype(np.float32).astype(np.float64)
    got = oracle.e4m3_encode(s)
    want = np.array([_brute_e4m3(float(x)) for x in s], dtype=np.uint8)
    assert np.array_equal(got, want)
    assert oracle.e4m3_encode(np.array([1e30]))[0] == 0x7E


# ---------------------------------------------------------------- quantiser pins
def _random_block_matrix(rng, rows, cols, spread=True):
    x = rng.standard_normal((rows, cols)).astype(np.float32)
    if spread:
        x *= np.exp(rng.uniform(-6, 6, (rows, cols // 16, 1))).repeat(16, axis=2).reshape(rows, cols).astype(np.float32)
    return synth.bf16_to_f32(synth.f32_to_bf16_bits(x))


def test_global_scale_definition():
    x = np.array([[0.5, -2688.0] + [0.0] * 14], dtype=np.float32)
    assert oracle.global_scale(x) == np.float32(1.0)
    assert oracle.global_scale(np.zeros((2, 16), np.float32)) == np.float32(1.0)
    x = np.array([[3.0] * 16], dtype=np.float32)
    assert oracle.global_scale(x) == np.float32(896.0)


def test_roundtrip_of_representable_blocks():
    """A block of E2M1 values times 2**e containing +-6*2**e quantises back to itself (gs = 1)."""
    rng = np.random.default_rng(11)
    vals = oracle.e2m1_decode(np.arange(16))
    rows, cols = 64, 64
    codes = rng.integers(0, 16, (rows, cols)).astype(np.uint8)
    codes[:, ::16] = np.where(rng.random((rows, cols // 16)) < 0.5, 7, 15)  # each block has +-6
    e = rng.integers(-5, 7, (rows, cols // 16))
    x = (vals[codes] * np.ldexp(1.0, e).repeat(16, axis=1)).astype(np.float32)
    qc, sf = oracle.quantize(x, np.float32(1.0))
    # +0 / -0 both decode to 0: compare values and signs of non-zero codes
    assert np.array_equal(oracle.e2m1_decode(qc), vals[codes])
    assert np.array_equal(qc[vals[codes] != 0], codes[vals[codes] != 0])
    assert np.array_equal(oracle.e4m3_decode(sf), np.ldexp(1.0, e))


def test_block_amax_maps_to_six_and_largest_block_to_448():
    rng = np.random.default_rng(12)
    x = _random_block_matrix(rng, 48, 256)
    gs = oracle.global_scale(x)
    codes, sf = oracle.quantize(x, gs)
    xb = np.abs(x.reshape(48, 16, 16))
    arg = xb.argmax(axis=2)
    cb = codes.reshape(48, 16, 16)
    top = np.take_along_axis(cb, arg[:, :, None], axis=2)[:, :, 0]
    normal = sf >= 0x08
    assert np.all((top[normal] & 7) == 7)
    # the block holding the tensor amax gets the largest scale, 448
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert sf[r, c // 16] == 0x7E
    assert sf.max() == 0x7E


def test_zero_block():
    x = np.zeros((2, 32), np.float32)
    x[1, 16:] = -0.0
    x[0, 16:] = np.linspace(-1, 1, 16)
    codes, sf = oracle.quantize(x, np.float32(3.0))
    assert sf[0, 0] == 0 and sf[1, 0] == 0 and sf[1, 1] == 0
    assert np.all(codes[0, :16] == 0)
    assert np.all(codes[1, 16:] == 8)  # -0 keeps its sign bit (reading R2)


def test_quantize_elementwise_optimal_given_scale():
    """Brute force: sf is the nearest E4M3 of s, and every code is the nearest of all 16 codes to x*gs/dec(sf)."""
    rng = np.random.default_rng(13)
    x = _random_block_matrix(rng, 6, 64)
    gs = oracle.global_scale(x)
    codes, sf = oracle.quantize(x, gs)
    allv = oracle.e2m1_decode(np.arange(16))
    for r in range(6):
        for j in range(4):
            blk = x[r, 16 * j:16 * j + 16]
            amax = np.float32(np.max(np.abs(blk)))
            s = np.float32(np.float32(amax / np.float32(6)) * gs)
            assert sf[r, j] == _brute_e4m3(float(s))
            dec = float(oracle.e4m3_decode(sf[r, j]))
            inv = np.float32(0) if dec == 0 else np.float32(gs / np.float32(dec))
            for i in range(16):
                v = float(np.float32(blk[i] * inv))
                d = np.abs(allv - v)
                best = d.min()
                cand = [c for c in range(16) if d[c] == best]
                assert codes[r, 16 * j + i] in cand
                c = int(codes[r, 16 * j + i])
                if len({c & 7 for c in cand}) > 1:   # tie: even mantissa wins
                    assert c % 2 == 0


def test_dequant_error_sanity_band():
    """Not a pin: relative round-trip error on outlier activations lands near the blog's 7.5-9.2 %."""
    x = synth.bf16_to_f32(synth.outlier_activations(64, 1024, seed=0))
    gs = oracle.global_scale(x)
    codes, sf = oracle.quantize(x, gs)
    xh = oracle.dequantize(codes, sf, gs)
    rel = np.linalg.norm(xh - x) / np.linalg.norm(x)
    assert 0.03 < rel < 0.2


# ------------------------------------------------------------------ GEMM pins
def test_linear_textbook_triple_loop():
    rng = np.random.default_rng(21)
    M, N, K = 3, 5, 32
    a = _random_block_matrix(rng, M, K)
    w = _random_block_matrix(rng, N, K)
    gs_a = oracle.global_scale(a)
    ca, sa = oracle.quantize(a, gs_a)
    gsw = [np.float32(7.0), np.float32(0.25)]
    cw, sw = oracle.quantize(w, np.float32(1.0))
    segs = [(0, 2, gsw[0]), (2, 5, gsw[1])]
    y = oracle.linear(ca, sa, gs_a, cw, sw, segs)
    vals = json.load(open(GOLDEN))["e2m1_values_by_code"]
    e4 = dict((int(h, 16), v) for h, v in json.load(open(GOLDEN))["e4m3_known"])
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += (vals[ca[m, k]] * float(oracle.e4m3_decode(sa[m, k // 16]))
                        * vals[cw[n, k]] * float(oracle.e4m3_decode(sw[n, k // 16])))
            g = gsw[0] if n < 2 else gsw[1]
            assert math.isclose(y[m, n], acc / (float(gs_a) * float(g)), rel_tol=1e-12, abs_tol=1e-300)
    assert e4[0x38] == 1.0


def test_linear_exact_small_integer_case():
    """gs = 1 and every scale = 1.0 (0x38): 2*Y is an integer matrix product."""
    rng = np.random.default_rng(22)
    M, N, K = 17, 9, 128
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    twice = np.array([0, 1, 2, 3, 4, 6, 8, 12, 0, -1, -2, -3, -4, -6, -8, -12], dtype=np.int64)
    want = (twice[ca] @ twice[cw].T) / 4.0
    y = oracle.linear(ca, sa, np.float32(1), cw, sw, [(0, N, np.float32(1))])
    assert np.array_equal(y, want)


def test_fused_equals_separate_modules():
    """One GEMM over concatenated segments with per-segment alpha == the per-module GEMMs."""
    rng = np.random.default_rng(23)
    K = 64
    x = _random_block_matrix(rng, 10, K)
    gs_a = oracle.global_scale(x)
    ca, sa = oracle.quantize(x, gs_a)
    mods = [(_random_block_matrix(rng, 16, K) * s).astype(np.float32) for s in (1, 8, 16)]
    sep, codes, scales, segs, n0 = [], [], [], [], 0
    for w in mods:
        gw = oracle.global_scale(w)
        cw, sw = oracle.quantize(w, gw)
        sep.append(oracle.linear(ca, sa, gs_a, cw, sw, [(0, 16, gw)]))
        codes.append(cw), scales.append(sw), segs.append((n0, n0 + 16, gw))
        n0 += 16
    fused = oracle.linear(ca, sa, gs_a, np.concatenate(codes), np.concatenate(scales), segs)
    assert np.array_equal(fused, np.concatenate(sep, axis=1))
    # one shared scale (the mismatch the pages describe) is measurably wrong
    wrong = oracle.linear(ca, sa, gs_a, np.concatenate(codes), np.concatenate(scales),
                          [(0, 48, segs[0][2])])
    assert not np.allclose(wrong, fused, rtol=1e-2)


# ---------------------------------------------------------------- epilogue pins
def test_gate_closed_forms(facts):
    cf = facts["gate_closed_forms"]
    assert oracle.sigmoid(0.0) == cf["sigmoid_at_0"]
    assert math.isclose(oracle.softplus(0.0), cf["softplus_at_0"], rel_tol=1e-15)
    a_log = np.array([0.3, -1.2])
    dt = np.array([0.5, -0.25])
    beta, g = oracle.gdn_gates(np.zeros((1, 2)), -dt[None, :], a_log, dt)
    assert np.allclose(beta, 0.5)
    assert np.allclose(g, -np.exp(a_log) * cf["softplus_at_0"], rtol=1e-15)
    x = np.linspace(-30, 30, 601)
    assert np.allclose(oracle.sigmoid(x) + oracle.sigmoid(-x), 1.0, atol=1e-15)
    assert np.allclose(oracle.softplus(x) - oracle.softplus(-x), x, atol=1e-12)
    assert np.allclose(oracle.silu(x) - oracle.silu(-x), x, atol=1e-12)
    assert np.all(np.diff(oracle.softplus(x)) > 0) and np.all(oracle.softplus(x) > 0)
    # decay gate is negative and decreasing in a
    _, g = oracle.gdn_gates(np.zeros((601, 1)), x[:, None], np.array([0.0]), np.array([0.0]))
    assert np.all(g < 0) and np.all(np.diff(g[:, 0]) < 0)
    assert np.allclose(oracle.silu_mul(np.array([0.0, 2.0]), np.array([5.0, 3.0])),
                       [0.0, 6.0 / (1.0 + math.exp(-2.0))])


def test_round_to_bf16_agrees_with_independent_rounders():
    import torch
    rng = np.random.default_rng(31)
    x32 = (rng.standard_normal(20000) * np.exp(rng.uniform(-20, 20, 20000))).astype(np.float32)
    ours = oracle.round_to_bf16(x32.astype(np.float64))
    via_synth = synth.bf16_to_f32(synth.f32_to_bf16_bits(x32)).astype(np.float64)
    via_torch = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ours, via_synth)
    assert np.array_equal(ours, via_torch)
    # exact ties in FP64 go to even
    assert oracle.round_to_bf16(1.0 + 2.0 ** -8) == 1.0
    assert oracle.round_to_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6


# ------------------------------------------------------------------- layout
def test_scale_layout_reading():
    cols = 512  # 32 blocks -> 8 atoms per 128-row group
    assert layout.scale_offset(0, 0, cols) == 0
    assert layout.scale_offset(0, 1, cols) == 1
    assert layout.scale_offset(1, 0, cols) == 16
    assert layout.scale_offset(32, 0, cols) == 4
    assert layout.scale_offset(96, 3, cols) == 15
    assert layout.scale_offset(0, 4, cols) == 512
    assert layout.scale_offset(128, 0, cols) == 8 * 512
    rng = np.random.default_rng(41)
    for rows, c in [(1, 16), (130, 80), (300, 512)]:
        sf = rng.integers(0, 255, (rows, c // 16)).astype(np.uint8)
        buf = layout.swizzle_scales(sf, rows, c)
        assert buf.size == layout.scale_bytes(rows, c)
        assert np.array_equal(layout.unswizzle_scales(buf, rows, c), sf)
        # offsets are a bijection onto the non-padding bytes
        r, j = np.meshgrid(np.arange(rows), np.arange(c // 16), indexing="ij")
        offs = layout.scale_offset(r, j, c).ravel()
        assert len(np.unique(offs)) == offs.size


def test_nibble_packing_reading():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    p = layout.pack_nibbles(codes)
    assert p.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(layout.unpack_nibbles(p), codes)


def test_synth_is_seeded_and_bf16():
    a = synth.outlier_activations(8, 64, seed=0)
    b = synth.outlier_activations(8, 64, seed=0)
    assert a.dtype == np.uint16 and np.array_equal(a, b)
    t = synth.student_t_activations(16, 128, seed=0)
    x = synth.bf16_to_f32(t)
    assert np.all(np.isfinite(x))


# ------------------------------------------------------------ fused-group repair
def _rand_sf(rng, shape, lo=0x08, hi=0x7E):
    return rng.integers(lo, hi + 1, shape).astype(np.uint8)


def test_fold_equal_scales_is_identity():
    rng = np.random.default_rng(100)
    sfs = [_rand_sf(rng, (8, 4)), _rand_sf(rng, (16, 4))]
    out, gs_c = oracle.fold_segments(sfs, [3.5, 3.5])
    assert gs_c == np.float32(3.5)
    for a, b in zip(sfs, out):
        assert np.array_equal(a, b)


def test_fold_power_of_two_ratio_is_exact():
    """gs_seg = 4 * gs_c: every normal scale that stays normal is divided by 4 exactly."""
    rng = np.random.default_rng(101)
    sf = _rand_sf(rng, (32, 8), lo=0x20, hi=0x7E)   # >= 2**-3: /4 stays >= 2**-5, normal
    out, gs_c = oracle.fold_segments([sf, sf], [2.0, 8.0])
    assert gs_c == np.float32(2.0)
    assert np.array_equal(out[0], sf)
    assert np.array_equal(oracle.e4m3_decode(out[1]), oracle.e4m3_decode(sf) / 4.0)


def test_fold_rerounding_bound_matches_the_pages():
    """Each folded scale is the ratio-scaled scale up to one E4M3 rounding: relative error
    <= 2**-4 (the pages' <= 6.2 %) while the result is normal (>= 2**-6), and <= half a
    subnormal step (2**-10) below that."""
    rng = np.random.default_rng(102)
    sf = _rand_sf(rng, (256, 16), lo=0x01)
    gss = [1.0, 1.82, 2.75, 7.3, 16.0]
    outs, gs_c = oracle.fold_segments([sf] * len(gss), gss)
    for g, o in zip(gss, outs):
        exact = oracle.e4m3_decode(sf) * np.float64(np.float32(gs_c / np.float32(g)))
        got = oracle.e4m3_decode(o)
        normal = exact >= 2.0 ** -6
        assert np.all(np.abs(got - exact)[normal] <= 2.0 ** -4 * exact[normal] + 1e-30)
        assert np.all(np.abs(got - exact)[~normal] <= 2.0 ** -10)
        assert np.all(got <= 448.0)


def test_fold_dequantised_weights_within_bound():
    """Folding changes each decoded weight by at most 2**-4 of itself (normal scales)."""
    rng = np.random.default_rng(103)
    segs = [rng.standard_normal((32, 64)).astype(np.float32) * m for m in (0.02, 0.1, 0.32)]
    q = [oracle.quantize(w, oracle.global_scale(w)) + (oracle.global_scale(w),) for w in segs]
    outs, gs_c = oracle.fold_segments([sf for _, sf, _ in q], [g for _, _, g in q])
    for (codes, sf, g), sf2 in zip(q, outs):
        before = oracle.dequantize(codes, sf, g)
        after = oracle.dequantize(codes, sf2, gs_c)
        assert np.all(np.abs(after - before) <= 2.0 ** -4 * np.abs(before) + 1e-12)


def test_fold_repairs_the_shared_scale_mismatch():
    """A fused GEMM run with one global scale: wrong by the scale ratios before folding,
    close to the per-module result after it (blog section 罠①)."""
    rng = np.random.default_rng(104)
    x = rng.standard_normal((16, 256)).astype(np.float32)
    ws = [rng.standard_normal((32, 256)).astype(np.float32) * m for m in (0.02, 0.0364, 0.055)]
    gx = oracle.global_scale(x)
    cx, sx = oracle.quantize(x, gx)
    qs = [oracle.quantize(w, oracle.global_scale(w)) + (oracle.global_scale(w),) for w in ws]
    codes = np.concatenate([c for c, _, _ in qs])
    segs, n0 = [], 0
    for _, _, g in qs:
        segs.append((n0, n0 + 32, g))
        n0 += 32
    ref = oracle.linear(cx, sx, gx, codes, np.concatenate([s for _, s, _ in qs]), segs)
    wrong = oracle.linear(cx, sx, gx, codes, np.concatenate([s for _, s, _ in qs]), [(0, 96, qs[0][2])])
    folded, gs_c = oracle.fold_segments([s for _, s, _ in qs], [g for _, _, g in qs])
    fixed = oracle.linear(cx, sx, gx, codes, np.concatenate(folded), [(0, 96, gs_c)])
    err = lambda y: np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert err(wrong) > 0.2
    assert err(fixed) < 0.05


# ------------------------------------------------------------------ FP8 KV cache
def test_e4m3_signed_encode_facts():
    vals = oracle.e4m3_decode(np.arange(0x7F))                     # all finite magnitudes
    assert np.array_equal(oracle.e4m3_encode_signed(vals), np.arange(0x7F))
    assert np.array_equal(oracle.e4m3_encode_signed(-vals[1:]), np.arange(1, 0x7F) | 0x80)
    assert oracle.e4m3_encode_signed(-0.0) == 0x80 and oracle.e4m3_encode_signed(0.0) == 0x00
    assert oracle.e4m3_encode_signed(1e6) == 0x7E and oracle.e4m3_encode_signed(-1e6) == 0xFE
    # ties between 1.0 (0x38) and 1.125 (0x39) go to the even code; just above goes up
    assert oracle.e4m3_encode_signed(1.0625) == 0x38
    assert oracle.e4m3_encode_signed(np.nextafter(1.0625, 2.0)) == 0x39
    assert oracle.e4m3_encode_signed(-1.0625) == 0xB8


def test_fp8_scale_and_roundtrip():
    rng = np.random.default_rng(120)
    x = rng.standard_normal((64, 128)).astype(np.float32) * 3
    s = oracle.fp8_scale(x)
    assert s == np.float32(np.max(np.abs(x)) / np.float32(448))
    assert oracle.fp8_scale(np.zeros((2, 16))) == 1.0
    cache = oracle.kv_cache_fp8(x, s, np.arange(64), 64)
    back = oracle.e4m3_decode(cache & 0x7F) * np.where(cache & 0x80, -1, 1) * np.float64(s)
    # the tensor amax maps to 448 (up to the fl32 division), every value within one E4M3
    # rounding: relative 2**-4 in the normal range, half the subnormal step below it
    r, c = np.unravel_index(np.argmax(np.abs(x)), x.shape)
    assert (cache[r, c] & 0x7F) == 0x7E
    normal = np.abs(x / s) >= 2.0 ** -6
    err = np.abs(back - x)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(x[normal]))
    assert np.all(err[~normal] <= 2.0 ** -10 * np.float64(s))
    # exactly representable values come back exactly (power-of-two scale: exact reciprocal)
    vals = oracle.e4m3_decode(np.arange(0x7F)).astype(np.float32)[None, :] * np.float32(0.5)
    c2 = oracle.kv_cache_fp8(vals, np.float32(0.5), [0], 1)
    assert np.array_equal(c2[0], np.arange(0x7F))



def test_kv_cache_slot_scatter():
    x = np.arange(4 * 16, dtype=np.float32).reshape(4, 16) - 20
    cache = np.full((6, 16), 0x55, np.uint8)
    out = oracle.kv_cache_fp8(x, np.float32(1.0), [5, -1, 0, 2], 6, cache=cache)
    assert np.array_equal(out[5], oracle.e4m3_encode_signed(x[0]))
    assert np.array_equal(out[0], oracle.e4m3_encode_signed(x[2]))
    assert np.array_equal(out[2], oracle.e4m3_encode_signed(x[3]))
    for r in (1, 3, 4):  # untouched rows (slot -1 wrote nothing)
        assert np.all(out[r] == 0x55)


# ---------------------------------------------------------------- GDN recurrence
def _unit(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_gdn_no_write_no_decay_keeps_state():
    rng = np.random.default_rng(140)
    T, hk, hv, d = 5, 2, 4, 8
    q, k = _unit(rng, (T, hk, d)), _unit(rng, (T, hk, d))
    v = rng.standard_normal((T, hv, d))
    S0 = rng.standard_normal((hv, d, d))
    o, S = oracle.gdn_recurrence(q, k, v, np.zeros((T, hv)), np.zeros((T, hv)), S0)
    assert np.array_equal(S, S0)
    qq = np.repeat(q, 2, axis=1)
    assert np.allclose(o, np.einsum("hij,thi->thj", S0, qq), rtol=1e-14, atol=1e-14)
    # pure decay: beta = 0 scales the state by prod(alpha)
    g = -rng.uniform(0, 0.1, (T, hv))
    _, S2 = oracle.gdn_recurrence(q, k, v, g, np.zeros((T, hv)), S0)
    assert np.allclose(S2, np.exp(g.sum(0))[:, None, None] * S0, rtol=1e-13)


def test_gdn_delta_rule_overwrites_along_the_key():
    """alpha = 1, beta = 1, |k| = 1: after a write the state maps k_t exactly to v_t
    (the write replaces what the state predicted along k_t; blog mechanism ③)."""
    rng = np.random.default_rng(141)
    T, hk, hv, d = 6, 1, 2, 16
    q, k = _unit(rng, (T, hk, d)), _unit(rng, (T, hk, d))
    v = rng.standard_normal((T, hv, d))
    S0 = rng.standard_normal((hv, d, d))
    for t in range(1, T + 1):
        _, S = oracle.gdn_recurrence(q[:t], k[:t], v[:t], np.zeros((t, hv)), np.ones((t, hv)), S0)
        assert np.allclose(np.einsum("hij,i->hj", S, k[t - 1, 0]), v[t - 1], rtol=1e-12, atol=1e-12)
    # and directions orthogonal to k_t are left as they were
    _, S1 = oracle.gdn_recurrence(q[:1], k[:1], v[:1], np.zeros((1, hv)), np.ones((1, hv)), S0)
    w = rng.standard_normal(d)
    w -= (w @ k[0, 0]) * k[0, 0]
    assert np.allclose(np.einsum("hij,i->hj", S1, w), np.einsum("hij,i->hj", S0, w), atol=1e-12)


def test_gdn_single_step_by_hand():
    """d = 2, one head: S0 = [[1, 2], [3, 4]], k = (1, 0), v = (10, 20), alpha = 0.5,
    beta = 0.25, q = (0, 1).  S0^T k = (1, 2); beta (v - S0^T k) = (2.25, 4.5);
    S1 = 0.5 S0 + k (2.25, 4.5) = [[2.75, 5.5], [1.5, 2]]; o = S1^T q = (1.5, 2)."""
    S0 = np.array([[[1.0, 2.0], [3.0, 4.0]]])
    o, S = oracle.gdn_recurrence(np.array([[[0.0, 1.0]]]), np.array([[[1.0, 0.0]]]),
                                 np.array([[[10.0, 20.0]]]), np.log([[0.5]]), np.array([[0.25]]), S0)
    assert np.allclose(S[0], [[2.75, 5.5], [1.5, 2.0]], rtol=1e-15)
    assert np.allclose(o[0, 0], [1.5, 2.0], rtol=1e-15)


def test_gdn_linear_in_values_from_zero_state():
    rng = np.random.default_rng(142)
    T, hk, hv, d = 7, 2, 4, 8
    q, k = _unit(rng, (T, hk, d)), _unit(rng, (T, hk, d))
    v = rng.standard_normal((T, hv, d))
    g, b = -rng.uniform(0, 2, (T, hv)), rng.uniform(0, 1, (T, hv))
    o1, _ = oracle.gdn_recurrence(q, k, v, g, b)
    o2, _ = oracle.gdn_recurrence(q, k, 3.0 * v, g, b)
    assert np.allclose(o2, 3.0 * o1, rtol=1e-12, atol=1e-12)
    # value head h reads key head h // 2
    o3, _ = oracle.gdn_recurrence(q[:, :1], k[:, :1], v[:, :2], g[:, :2], b[:, :2])
    assert np.allclose(o3, o1[:, :2], rtol=1e-13)


def _chunked_recurrence(q, k, v, g, beta, S0, C):
    """The recurrence regrouped in chunks of C tokens (the form the prefill kernel
    evaluates), written out independently of the oracle in FP64.  One value head:
    q, k [T, d]; v [T, d]; g, beta [T]; S0 [d, d].  Per chunk, with the chunk-local
    cumulative decays G_t = g_1 + .. + g_t (G_0 = 0):
        (I + L) U = diag(beta) (V - diag(e^{G_{t-1}}) K S0),
            L[t, s] = beta_t e^{G_{t-1} - G_s} k_t.k_s  (s < t),
        O = diag(e^{G_t}) Q S0 + P U,  P[t, s] = e^{G_t - G_s} q_t.k_s  (s <= t),
        S = e^{G_C} S0 + K^T diag(e^{G_C - G_s}) U."""
    T = q.shape[0]
    S = S0.copy()
    out = np.empty((T, S0.shape[1]))
    for c0 in range(0, T, C):
        Q, K, V = q[c0:c0 + C], k[c0:c0 + C], v[c0:c0 + C]
        n = Q.shape[0]
        G = np.cumsum(g[c0:c0 + C])
        Gm = np.concatenate([[0.0], G[:-1]])
        b = beta[c0:c0 + C]
        L = np.tril(b[:, None] * np.exp(Gm[:, None] - G[None, :]) * (K @ K.T), -1)
        R = b[:, None] * (V - np.exp(Gm)[:, None] * (K @ S))
        U = np.linalg.solve(np.eye(n) + L, R)
        P = np.tril(np.exp(G[:, None] - G[None, :]) * (Q @ K.T))
        out[c0:c0 + n] = np.exp(G)[:, None] * (Q @ S) + P @ U
        S = np.exp(G[-1]) * S + K.T @ (np.exp(G[-1] - G)[:, None] * U)
    return out, S


@pytest.mark.parametrize("T,C", [(150, 64), (64, 64), (7, 4), (33, 16)])
def test_gdn_chunked_form_equals_the_token_recurrence(T, C):
    """The chunked regrouping used for long sequences reproduces the token-by-token
    recurrence (FP64): ragged last chunks, strong and zero decays, a carried state."""
    rng = np.random.default_rng(143 + T)
    d = 16
    q, k = _unit(rng, (T, 1, d)), _unit(rng, (T, 1, d))
    v = rng.standard_normal((T, 1, d))
    g = -rng.uniform(0.0, 0.5, (T, 1))
    g[T // 3] = -30.0    # a near-total forget
    g[T // 2] = 0.0      # no decay
    b = rng.uniform(0.05, 1.0, (T, 1))
    S0 = rng.standard_normal((1, d, d))
    o_ref, S_ref = oracle.gdn_recurrence(q, k, v, g, b, S0)
    o, S = _chunked_recurrence(q[:, 0], k[:, 0], v[:, 0], g[:, 0], b[:, 0], S0[0], C)
    assert np.allclose(o, o_ref[:, 0], rtol=1e-10, atol=1e-10)
    assert np.allclose(S, S_ref[0], rtol=1e-10, atol=1e-10)
