"""GPU parity of the block-scaled GEMM and its epilogues against the oracle."""
import numpy as np
import pytest

import oracle
import synth
from oracle import layout
from nvfp4_testutil import (assert_gemm_close, bf16_to_f64, logical, make_operand, oracle_quant,
                            rel_fro, to_dev_bf16, to_dev_f32)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _sync():
    import torch
    torch.cuda.synchronize()


# ------------------------------------------------------------- exact probes
def test_exact_integer_codes_pin_operand_layout(nv):
    """All scales 1.0 and gs = 1: FP32 accumulation is exact, so the output is
    bit-exact; a wrong nibble order or smem descriptor changes it."""
    rng = np.random.default_rng(1)
    M, N, K = 256, 512, 1024
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    ref = oracle.linear(ca, sa, 1.0, cw, sw, [(0, N, 1.0)])
    out = nv.linear(make_operand(ca, sa, 1.0), make_operand(cw, sw, 1.0), out_dtype="f32")
    _sync()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} mismatches"


def test_exact_power_of_two_scales_pin_scale_layout(nv):
    """Per-block scales in {1/2, 1, 2, 4}: still exact in FP32; pins which TMEM
    scale column / lane feeds which row and K block, for A and W."""
    rng = np.random.default_rng(2)
    M, N, K = 384, 768, 768
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    choices = np.array([0x30, 0x38, 0x40, 0x48], np.uint8)
    sa = choices[rng.integers(0, 4, (M, K // 16))]
    sw = choices[rng.integers(0, 4, (N, K // 16))]
    ref = oracle.linear(ca, sa, 1.0, cw, sw, [(0, N, 1.0)])
    out = nv.linear(make_operand(ca, sa, 1.0), make_operand(cw, sw, 1.0), out_dtype="f32")
    _sync()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} mismatches"


@pytest.mark.parametrize("M,N", [(100, 80), (256, 16), (256, 48), (256, 336), (300, 464), (512, 272), (128, 208),
                                 (257, 272), (511, 48)])
def test_exact_narrow_last_n_tile(nv, M, N):
    """The last N-tile narrower than 256 runs an MMA of N = its width rounded up to 32;
    in the CTA pair the second CTA then holds B rows [N/2, N) of the tile.  Integer codes
    and unit scales keep the FP32 result exact, so any misplaced B row shows."""
    rng = np.random.default_rng(M * 1000 + N)
    K = 512
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    ref = oracle.linear(ca, sa, 1.0, cw, sw, [(0, N, 1.0)])
    out = nv.linear(make_operand(ca, sa, 1.0), make_operand(cw, sw, 1.0), out_dtype="f32")
    _sync()
    got = out.cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} mismatches"
    assert nv.device_status() == 0


def test_repeat_launches_bit_identical(nv):
    """Race check: the CTA-pair kernel (SiLU*mul + NVFP4 requant, and BF16 out), the
    1-CTA kernel and the decode-size split-K path, each launched four times back to back
    on the same inputs, write the same bytes every time.  A stage or scale set reused
    before its consumers finished, or an accumulator read before its MMAs completed,
    would make launches differ."""
    import torch
    K = 2048
    xb = synth.student_t_activations(1024, K, seed=95)
    gu, gsegs = nv.quantize_fused([to_dev_bf16(synth.gaussian_weights(2048, K, seed=96)),
                                   to_dev_bf16(synth.gaussian_weights(2048, K, seed=97, std=0.04))])
    a = _quant_dev(nv, xb)
    a100 = _quant_dev(nv, xb[:100])
    a32 = _quant_dev(nv, xb[:32])
    h16 = nv.linear(a, gu, segments=gsegs, epilogue="silu_mul", out_dtype="bf16")
    gs_h = nv.global_scale(h16)
    runs = {"pair_nvfp4": [], "pair_bf16": [], "one_cta": [], "decode": []}
    for _ in range(4):
        q = nv.linear(a, gu, segments=gsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h)
        runs["pair_nvfp4"].append(torch.cat([q.codes.flatten(), q.scales]))
        runs["pair_bf16"].append(nv.linear(a, gu, segments=gsegs, out_dtype="bf16"))
        runs["one_cta"].append(nv.linear(a100, gu, segments=gsegs, out_dtype="f32"))
        runs["decode"].append(nv.linear_splitk(a32, gu, segments=gsegs, out_dtype="bf16", split_k=2))
    _sync()
    for k, outs in runs.items():
        for o in outs[1:]:
            assert torch.equal(o, outs[0]), k
    assert nv.device_status() == 0


@pytest.mark.parametrize("M", [100, 256])
def test_outputs_only_16_byte_aligned(nv, M):
    """The epilogue stores 32 bytes per lane when every output row starts 32-byte
    aligned, else 16: a row stride of N + 8 BF16 / N + 4 FP32 elements, or a base 16
    bytes past a 32-byte boundary, takes the 16-byte path and gives the same values
    (and the NVFP4 output the same bytes)."""
    import torch
    K, N = 512, 384
    xb = synth.student_t_activations(M, K, seed=90)
    wb = synth.gaussian_weights(N, K, seed=91)
    a = _quant_dev(nv, xb)
    w = _quant_dev(nv, wb)
    y16 = nv.linear(a, w, out_dtype="bf16")
    y32 = nv.linear(a, w, out_dtype="f32")
    b16 = torch.zeros((M, N + 8), dtype=torch.bfloat16, device="cuda")
    b32 = torch.zeros((M, N + 4), dtype=torch.float32, device="cuda")
    nv.linear(a, w, out_dtype="bf16", out=b16[:, :N])
    nv.linear(a, w, out_dtype="f32", out=b32[:, :N])
    flat16 = torch.zeros(M * N + 8, dtype=torch.bfloat16, device="cuda")
    o16 = flat16[8:].view(M, N)  # base 16 bytes past a 32-byte boundary
    nv.linear(a, w, out_dtype="bf16", out=o16)
    gs_h = nv.global_scale(y16)
    q_ref = nv.linear(a, w, out_dtype="nvfp4", gs_out=gs_h)
    flat8 = torch.zeros(M * N // 2 + 16, dtype=torch.uint8, device="cuda")
    q = nv.linear(a, w, out_dtype="nvfp4", gs_out=gs_h, out=flat8[16:].view(M, N // 2))
    _sync()
    assert torch.equal(b16[:, :N], y16) and torch.equal(o16, y16) and torch.equal(b32[:, :N], y32)
    assert (b16[:, N:] == 0).all() and (b32[:, N:] == 0).all()
    assert torch.equal(q.codes, q_ref.codes) and torch.equal(q.scales, q_ref.scales)
    assert nv.device_status() == 0


@pytest.mark.parametrize("M", [128, 256])
def test_single_nonzero_probes(nv, M):
    """One non-zero code / scale at a time lands in exactly one output element.
    M = 128 runs the one-CTA kernel, M = 256 the CTA-pair kernel (rows 128..255 and
    B rows 128..255 come from the second CTA of the pair)."""
    N, K = 256, 256
    probes = [(0, 0, 0), (5, 7, 1), (37, 130, 77), (127, 255, 255), (64, 200, 128), (96, 31, 200)]
    if M > 128:
        probes += [(128, 0, 0), (200, 129, 63), (255, 255, 255), (131, 3, 250)]
    for (m, n, k) in probes:
        ca = np.zeros((M, K), np.uint8)
        cw = np.zeros((N, K), np.uint8)
        ca[m, k] = 7      # 6.0
        cw[n, k] = 2      # 1.0
        sa = np.full((M, K // 16), 0x38, np.uint8)
        sw = np.full((N, K // 16), 0x38, np.uint8)
        sa[m, k // 16] = 0x40   # 2.0
        out = nv.linear(make_operand(ca, sa, 1.0), make_operand(cw, sw, 1.0), out_dtype="f32")
        _sync()
        got = out.cpu().numpy()
        want = np.zeros((M, N), np.float32)
        want[m, n] = 12.0
        assert np.array_equal(got, want), (m, n, k, np.argwhere(got != 0)[:4], got[got != 0][:4])


# ------------------------------------------------------- realistic parity
def test_raster_groups_of_32_with_a_ragged_group(nv):
    """A wide weight (64 N-tiles or more) whose group of A rows fits a quarter of L2 is
    rastered in groups of 32 pair M-tiles; 33 M-tiles leave a last group of one.  Exact
    integer case (all scales 1, gs 1: FP32 accumulation is exact).  One row in every
    256-row pair tile, plus rows at tile and group boundaries, are compared with the
    oracle over all columns, so every (M-tile, N-tile) pair of the launch is checked."""
    rng = np.random.default_rng(7)
    M, N, K = 33 * 256, 64 * 256, 256
    ca = rng.integers(0, 16, (M, K)).astype(np.uint8)
    cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    rows = sorted({256 * t + (37 * t) % 256 for t in range(33)} | {0, 127, 128, 255, 256, 8191, 8192, M - 1})
    ref = oracle.linear(ca[rows], sa[rows], 1.0, cw, sw, [(0, N, 1.0)])
    out = nv.linear(make_operand(ca, sa, 1.0), make_operand(cw, sw, 1.0), out_dtype="f32")
    _sync()
    got = out[rows].cpu().numpy().astype(np.float64)
    assert np.array_equal(got, ref), f"{np.sum(got != ref)} mismatches"


def _quant_dev(nv, bits, gs=None):
    x = to_dev_bf16(bits)
    return nv.quantize(x, None if gs is None else to_dev_f32([gs]))


def test_config1_linear(nv):
    """Single W4A4 linear: X 128x1024 (N(0,1), 0.1% outliers x50), W 1024x1024 N(0,0.02)."""
    xb = synth.outlier_activations(128, 1024, seed=0)
    wb = synth.gaussian_weights(1024, 1024, seed=1)
    ca, sa, gsa = oracle_quant(xb)
    cw, sw, gsw = oracle_quant(wb)
    ref = oracle.linear(ca, sa, gsa, cw, sw, [(0, 1024, gsw)])
    a = _quant_dev(nv, xb)
    w = _quant_dev(nv, wb)
    y32 = nv.linear(a, w, out_dtype="f32")
    y16 = nv.linear(a, w, out_dtype="bf16")
    _sync()
    assert rel_fro(y32.cpu().numpy(), ref) <= 1e-3
    assert_gemm_close(y16, ref)


def test_ragged_multi_segment(nv):
    """M and N not multiples of the tile; three segments with different global scales."""
    M, K = 300, 768
    segs = [("s0", 128), ("s1", 176), ("s2", 96)]
    ws = synth.segmented_weights(segs, K, seed=11, multipliers={"s0": 1.0, "s1": 5.0, "s2": 0.25})
    xb = synth.outlier_activations(M, K, seed=10)
    ca, sa, gsa = oracle_quant(xb)
    codes, scales, oseg, dseg, n0 = [], [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        codes.append(c), scales.append(s)
        oseg.append((n0, n0 + wb.shape[0], g))
        n0 += wb.shape[0]
    N = n0
    ref = oracle.linear(ca, sa, gsa, np.concatenate(codes), np.concatenate(scales), oseg)
    w, dsegs = _fused_weight(nv, [wb for _, wb in ws])
    a = _quant_dev(nv, xb)
    y32 = nv.linear(a, w, segments=dsegs, out_dtype="f32")
    y16 = nv.linear(a, w, segments=dsegs, out_dtype="bf16")
    _sync()
    assert rel_fro(y32.cpu().numpy(), ref) <= 1e-3
    assert_gemm_close(y16, ref)
    # one shared global scale (the mismatch the pages describe) is far outside tolerance
    y_wrong = nv.linear(a, w, segments=[(0, N, dsegs[0][2])], out_dtype="f32")
    _sync()
    assert rel_fro(y_wrong.cpu().numpy(), ref) > 0.1


def _fused_weight(nv, segs_bits):
    """Per-segment quantisation on the device, each with its own global scale, packed
    into one fused weight (nvfp4_quantize_rows)."""
    return nv.quantize_fused([to_dev_bf16(wb) for wb in segs_bits])


def test_gdn_gates_epilogue(nv):
    """Fused GDN-style projection: two wide segments + beta (16 heads) + alpha (16 heads)."""
    M, K, H = 200, 512, 16
    names = [("q", 256), ("z", 256), ("beta", H), ("alpha", H)]
    ws = synth.segmented_weights(names, K, seed=21, multipliers={"q": 1, "z": 8, "beta": 16, "alpha": 1})
    xb = synth.outlier_activations(M, K, seed=20)
    a_log, dt_bias = synth.gdn_gate_params(H, seed=22)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + wb.shape[0], g))
        n0 += wb.shape[0]
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    beta_ref, g_ref = oracle.gdn_gates(y[:, 512:512 + H], y[:, 528:528 + H], a_log, dt_bias)
    w, dsegs = _fused_weight(nv, [wb for _, wb in ws])
    a = _quant_dev(nv, xb)
    import torch
    beta = torch.empty((M, H), dtype=torch.float32, device="cuda")
    g = torch.empty((M, H), dtype=torch.float32, device="cuda")
    gates = dict(beta_begin=512, alpha_begin=528, n_heads=H, A_log=to_dev_f32(a_log),
                 dt_bias=to_dev_f32(dt_bias), beta_out=beta, g_out=g)
    out = nv.linear(a, w, segments=dsegs, epilogue="gdn_gates", gates=gates, out_dtype="bf16")
    _sync()
    assert np.max(np.abs(beta.cpu().numpy() - beta_ref)) <= 1e-3
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= 1e-3
    o = bf16_to_f64(out)
    assert_gemm_close(out[:, :512], y[:, :512])
    # gated columns of the BF16 output hold the gate values: within the gates' 1e-3
    # absolute tolerance plus one BF16 rounding step of the value
    for got, ref in ((o[:, 512:528], beta_ref), (o[:, 528:544], g_ref)):
        ulp = np.ldexp(1.0, np.frexp(np.abs(ref))[1] - 8)
        err = np.abs(got - ref)
        bad = err > 1e-3 + ulp
        assert not bad.any(), (np.argwhere(bad)[:4], got[bad][:4], ref[bad][:4])


@pytest.mark.parametrize("M", [256, 300])
def test_silu_mul_epilogue_and_requant(nv, M):
    """MLP gate|up with SiLU*mul: BF16 output vs oracle, and the fused NVFP4
    re-quantisation equal (bit for bit) to BF16 output + the standalone quantiser and
    to the oracle's quantiser applied to that BF16 output.
    M = 300: the last CTA pair covers rows 256..511, of which 300..383 are scale
    padding (written as zero) and 384..511 lie outside the output."""
    import torch
    K, Nh = 512, 256
    ws = synth.segmented_weights([("gate", Nh), ("up", Nh)], K, seed=31, multipliers={"gate": 1, "up": 2})
    xb = synth.student_t_activations(M, K, seed=30)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + Nh, g))
        n0 += Nh
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    h_ref = oracle.silu_mul(y[:, :Nh], y[:, Nh:])
    w, dsegs = _fused_weight(nv, [wb for _, wb in ws])
    a = _quant_dev(nv, xb)
    h16 = nv.linear(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="bf16")
    _sync()
    assert_gemm_close(h16, h_ref)
    # fused requant == unfused BF16 output quantised by the standalone kernel
    gs_h = nv.global_scale(h16)
    out_scales = torch.full((nv.scale_bytes(M, Nh),), 0xAB, dtype=torch.uint8, device="cuda")
    hq = nv.linear(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h,
                   out_scales=out_scales)
    hq2 = nv.quantize(h16, gs_h)
    _sync()
    assert torch.equal(hq.codes, hq2.codes)
    assert torch.equal(hq.scales, hq2.scales)
    gc, gsf = logical(hq)
    # bit-exact against the oracle's quantiser applied to the kernel's own BF16 h
    kc, ks = oracle.quantize(h16.float().cpu().numpy(), np.float32(gs_h.item()))
    assert np.array_equal(gc, kc) and np.array_equal(gsf, ks)
    # and end to end: codes of the oracle's FP64 h rounded to BF16, with the same gs
    rc, rsf = oracle.quantize(oracle.round_to_bf16(h_ref).astype(np.float32), np.float32(gs_h.item()))
    assert np.mean(gsf == rsf) > 0.995
    assert np.mean(gc == rc) > 0.995
    deq_g = oracle.dequantize(gc, gsf, gs_h.item())
    deq_r = oracle.dequantize(rc, rsf, gs_h.item())
    assert rel_fro(deq_g, deq_r) < 1e-2


def test_device_status_clean(nv):
    assert nv.device_status() == 0
