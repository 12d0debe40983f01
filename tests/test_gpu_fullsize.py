"""GPU parity at the full workload sizes (the launch configurations bench.py times),
checked on sampled output rows that the oracle computes one by one.

* GDN fused input projection: X [8192 x 5120] (N(0,1), 0.1 % outliers x50), one fused
  weight q|k|v|z|beta|alpha = 2048|2048|4096|4096|32|32 rows, each segment with its
  own global scale (multipliers 1|2|4|8|16|1), gate epilogue.
* MLP block: X [32768 x 5120] (Student-t(3), 8 hot channels x100), gate|up
  [2 x 17408 x 5120] with SiLU*mul and NVFP4 re-quantisation, down [5120 x 17408].
* The other linears of the 496-linear sweep at M = 4096: GDN output projection,
  fused attention q|k|v (three modules, three global scales), attention output.
"""
import numpy as np
import pytest

import oracle
import synth
from nvfp4_testutil import assert_gemm_close, logical, oracle_quant, rel_fro, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _sample_rows(M, n_random, seed):
    """Tile-boundary rows (first / last of the first and last 256-row CTA pair, both
    halves of a pair) plus seeded random rows."""
    fixed = [0, 1, 127, 128, 255, 256, M // 2, M - 257, M - 256, M - 129, M - 128, M - 1]
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([fixed, rng.choice(M, n_random, replace=False)]))
    return rows[(rows >= 0) & (rows < M)]


def _oracle_rows(bits, rows, gs):
    """Oracle quantisation of selected rows of x with the tensor's global scale."""
    x = synth.bf16_to_f32(bits[rows])
    return oracle.quantize(x, np.float32(gs))


def test_gdn_inproj_full_size_sampled_rows(nv):
    import torch
    M, K = 8192, 5120
    xb = synth.outlier_activations(M, K, seed=0)
    ws = synth.segmented_weights(synth.GDN_INPROJ_SEGMENTS, K, seed=1,
                                 multipliers=synth.GDN_INPROJ_MULTIPLIERS)
    a_log, dt_bias = synth.gdn_gate_params(32, seed=7)
    N = sum(w.shape[0] for _, w in ws)
    rows = _sample_rows(M, 40, seed=3)

    gsa = oracle.global_scale(synth.bf16_to_f32(xb))
    ca, sa = _oracle_rows(xb, rows, gsa)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + wb.shape[0], g))
        n0 += wb.shape[0]
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    beta_ref, g_ref = oracle.gdn_gates(y[:, N - 64:N - 32], y[:, N - 32:], a_log, dt_bias)

    a = nv.quantize(to_dev_bf16(xb))
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    beta = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    g = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    gates = dict(beta_begin=N - 64, alpha_begin=N - 32, n_heads=32, A_log=to_dev_f32(a_log),
                 dt_bias=to_dev_f32(dt_bias), beta_out=beta, g_out=g)
    out = nv.linear(a, w, segments=dsegs, epilogue="gdn_gates", gates=gates, out_dtype="bf16")
    torch.cuda.synchronize()
    assert float(a.gs.item()) == float(gsa)
    assert np.max(np.abs(beta.cpu().numpy()[rows] - beta_ref)) <= 1e-3
    assert np.max(np.abs(g.cpu().numpy()[rows] - g_ref)) <= 1e-3
    got = out[torch.from_numpy(rows).cuda()]
    assert_gemm_close(got[:, :N - 64], y[:, :N - 64])
    assert nv.device_status() == 0


def test_mlp_block_full_size_sampled_rows(nv):
    """Each step of the MLP block at full size, on sampled rows:
    (a) X's global scale and codes (bit-exact);
    (b) gate|up GEMM + SiLU*mul to BF16 against the oracle's FP64 h;
    (c) the fused NVFP4 re-quantisation: bit-equal to the standalone quantiser of (b)'s
        BF16 output on the whole tensor, bit-equal on the sampled rows to the oracle's
        quantiser applied to that same BF16 output, and equal to the oracle's codes of
        its own FP64 h except where the FP32-vs-FP64 accumulation difference moves h
        across a rounding midpoint;
    (d) the down projection at full size (M = 32768, K = 17408) fed with the oracle's
        own re-quantised rows (zero rows elsewhere), against the oracle."""
    import torch
    from nvfp4_testutil import make_operand
    M, H, I = 32768, 5120, 17408
    xb = synth.student_t_activations(M, H, seed=0)
    wg = synth.gaussian_weights(I, H, seed=1, std=0.02)
    wu = synth.gaussian_weights(I, H, seed=2, std=0.04)
    wd = synth.gaussian_weights(H, I, seed=3, std=0.02)
    rows = _sample_rows(M, 20, seed=4)
    rows_t = torch.from_numpy(rows).cuda()

    gsx = oracle.global_scale(synth.bf16_to_f32(xb))
    cx, sx = _oracle_rows(xb, rows, gsx)
    cg, sg, gsg = oracle_quant(wg)
    cu, su, gsu = oracle_quant(wu)
    cd, sd, gsd = oracle_quant(wd)
    y = oracle.linear(cx, sx, gsx, np.concatenate([cg, cu]), np.concatenate([sg, su]),
                      [(0, I, gsg), (I, 2 * I, gsu)])
    h_ref = oracle.silu_mul(y[:, :I], y[:, I:])
    h = oracle.round_to_bf16(h_ref).astype(np.float32)
    gsh = oracle.global_scale(h)  # static scale of H, calibrated on the sampled rows
    ch, sh = oracle.quantize(h, gsh)
    out_ref = oracle.linear(ch, sh, gsh, cd, sd, [(0, H, gsd)])

    # (a)
    xq = nv.quantize(to_dev_bf16(xb))
    w_gu, seg_gu = nv.quantize_fused([to_dev_bf16(wg), to_dev_bf16(wu)])
    w_d = nv.quantize(to_dev_bf16(wd))
    torch.cuda.synchronize()
    assert float(xq.gs.item()) == float(gsx)
    gcx, gsfx = logical(xq)
    assert np.array_equal(gcx[rows], cx) and np.array_equal(gsfx[rows], sx)
    # (b)
    h16 = nv.linear(xq, w_gu, segments=seg_gu, epilogue="silu_mul", out_dtype="bf16")
    torch.cuda.synchronize()
    assert_gemm_close(h16[rows_t], h_ref)
    # (c)
    gs_h = to_dev_f32([gsh])
    hq = nv.linear(xq, w_gu, segments=seg_gu, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h)
    hq2 = nv.quantize(h16, gs_h)
    torch.cuda.synchronize()
    assert torch.equal(hq.codes, hq2.codes) and torch.equal(hq.scales, hq2.scales)
    codes, sf = logical(hq)
    gc, gsf = codes[rows], sf[rows]
    # bit-exact against the oracle's quantiser applied to the kernel's own BF16 h (the
    # block format of the next layer's input): every sampled row, codes and scales
    kc, ks = oracle.quantize(h16[rows_t].float().cpu().numpy(), np.float32(gsh))
    assert np.array_equal(gc, kc) and np.array_equal(gsf, ks)
    # end to end against the FP64 h: equal except where the FP32-vs-FP64 accumulation
    # moves h across a BF16 or E2M1 rounding midpoint
    assert np.mean(gsf == sh) > 0.999
    assert np.mean(gc == ch) > 0.999
    assert rel_fro(oracle.dequantize(gc, gsf, gsh), oracle.dequantize(ch, sh, gsh)) < 1e-2
    del h16, hq2
    # (d)
    full_c = np.zeros((M, I), np.uint8)
    full_s = np.zeros((M, I // 16), np.uint8)
    full_c[rows], full_s[rows] = ch, sh
    h_op = make_operand(full_c, full_s, gsh)
    del full_c, full_s
    out = nv.linear(h_op, w_d, out_dtype="bf16")
    torch.cuda.synchronize()
    assert_gemm_close(out[rows_t], out_ref)
    assert nv.device_status() == 0


# The remaining linear shapes of the 496-linear sweep, at its M = 4096 prefill size
# (the CTA-pair kernel, as the sweep launches them): the GDN output projection
# (4096 -> 5120), the attention q|k|v projection fused as one GEMM of three modules
# with their own global scales (5120 -> 6144 | 1024 | 1024), and the attention output
# projection (6144 -> 5120).  Inputs: Student-t(3) activations standing in for the
# layer input / mixer output, N(0, 0.02) weights (k and v modules x2 and x4 so that
# the three global scales differ).
SWEEP_SHAPES = [
    ("gdn_out", 4096, [("o", 5120, 1.0)]),
    ("attn_qkv", 5120, [("q", 6144, 1.0), ("k", 1024, 2.0), ("v", 1024, 4.0)]),
    ("attn_o", 6144, [("o", 5120, 1.0)]),
]


def _sample_cols(n, n_random, seed):
    """Tile-boundary weight rows (output columns) of a module plus seeded random ones."""
    fixed = [0, 1, 127, 128, 255, 256, n // 2, n - 257, n - 256, n - 129, n - 128, n - 1]
    rng = np.random.default_rng(seed)
    cols = np.unique(np.concatenate([fixed, rng.choice(n, n_random, replace=False)]))
    return cols[(cols >= 0) & (cols < n)]


@pytest.mark.parametrize("name,K,mods", SWEEP_SHAPES, ids=[s[0] for s in SWEEP_SHAPES])
def test_sweep_linear_shapes_sampled_rows(nv, name, K, mods):
    """Sampled rows x sampled output columns of each module (every module's global
    scale taken over its whole weight), against the oracle."""
    import torch
    M = 4096
    xb = synth.student_t_activations(M, K, seed=20)
    wbs = [synth.gaussian_weights(n, K, seed=21 + i, std=0.02 * m) for i, (_, n, m) in enumerate(mods)]
    rows = _sample_rows(M, 24, seed=5)

    gsa = oracle.global_scale(synth.bf16_to_f32(xb))
    ca, sa = _oracle_rows(xb, rows, gsa)
    oc, os_, oseg, cols, n0, off = [], [], [], [], 0, 0
    for i, wb in enumerate(wbs):
        gw = oracle.global_scale(synth.bf16_to_f32(wb))
        cm = _sample_cols(wb.shape[0], 40, seed=30 + i)
        c, s_ = oracle.quantize(synth.bf16_to_f32(wb[cm]), np.float32(gw))
        oc.append(c), os_.append(s_), oseg.append((n0, n0 + len(cm), np.float32(gw)))
        cols.append(off + cm)
        n0 += len(cm)
        off += wb.shape[0]
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    cols = np.concatenate(cols)

    a = nv.quantize(to_dev_bf16(xb))
    if len(wbs) == 1:
        w = nv.quantize(to_dev_bf16(wbs[0]))
        out = nv.linear(a, w, out_dtype="bf16")
    else:
        w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for wb in wbs])
        out = nv.linear(a, w, segments=dsegs, out_dtype="bf16")
    torch.cuda.synchronize()
    assert float(a.gs.item()) == float(gsa)
    got = out[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()]
    assert_gemm_close(got, y)
    assert nv.device_status() == 0
