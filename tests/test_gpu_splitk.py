"""GPU parity of the split-K linear (decode regime: few token rows, K split over
several work units per output tile) against the oracle and against nvfp4_linear."""
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


def _sync():
    import torch
    torch.cuda.synchronize()


def test_down_proj_decode_full_size(nv):
    """32 decode tokens through the MLP down projection (5120 x 17408): FP32 and BF16
    outputs against the oracle, with the library's split count and with splits 1, 5
    and 10."""
    import torch
    M, N, K = 32, 5120, 17408
    xb = synth.student_t_activations(M, K, seed=40)
    wb = synth.gaussian_weights(N, K, seed=41)
    ca, sa, gsa = oracle_quant(xb)
    cw, sw, gsw = oracle_quant(wb)
    ref = oracle.linear(ca, sa, gsa, cw, sw, [(0, N, gsw)])
    a = nv.quantize(to_dev_bf16(xb))
    w = nv.quantize(to_dev_bf16(wb))
    s_def = nv.splitk_default(M, N, K)
    assert 1 < s_def <= K // 256  # 20 output tiles, 68 K tiles: the split pays here
    # the rule: SMs // tiles splits (one wave of work units), with >= 4 K tiles per split;
    # up to 64 rows a tile is 128 weight rows (all tokens), else 128 x 256 outputs
    sms = torch.cuda.get_device_properties(0).multi_processor_count

    def rule(m, n, k):
        tiles = -(-n // 128) if m <= 64 else -(-m // 128) * -(-n // 256)
        return max(1, min(k // 256 // 4, sms // tiles))
    for shape in [(M, N, K), (M, 34816, 5120), (M, 5120, 4096), (M, 12352, 5120), (4096, 5120, 4096),
                  (M, 1024, 512), (64, 5120, 5120), (65, 5120, 5120)]:
        assert nv.splitk_default(*shape) == rule(*shape), shape
    for s in (s_def, 1, 5, 10):
        y32 = nv.linear_splitk(a, w, out_dtype="f32", split_k=s)
        y16 = nv.linear_splitk(a, w, out_dtype="bf16", split_k=s)
        _sync()
        assert rel_fro(y32.cpu().numpy(), ref) <= 1e-3, s
        assert_gemm_close(y16, ref)
    # same sums as the one-unit-per-tile kernel up to the order of FP32 additions
    y_ref = nv.linear(a, w, out_dtype="f32")
    y_split = nv.linear_splitk(a, w, out_dtype="f32", split_k=s_def)
    _sync()
    assert rel_fro(y_split.cpu().numpy(), y_ref.cpu().numpy()) <= 1e-6
    assert nv.device_status() == 0


@pytest.mark.parametrize("M", [1, 7, 32, 33, 64, 65, 100, 129, 200])
def test_ragged_rows_and_splits(nv, M):
    """Rows that fill part of a 128-row tile, or span two; every split count.  Up to
    64 rows the decode kernel runs (32 or 64 token columns per MMA), above it the
    128 x 256 tile kernel; 400 weight rows end in a ragged 128-row weight tile."""
    K, segs = 768, [("s0", 128), ("s1", 176), ("s2", 96)]
    ws = synth.segmented_weights(segs, K, seed=50, multipliers={"s0": 1.0, "s1": 5.0, "s2": 0.25})
    xb = synth.outlier_activations(M, K, seed=51)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + wb.shape[0], g))
        n0 += wb.shape[0]
    ref = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    a = nv.quantize(to_dev_bf16(xb))
    for s in (1, 2, 3):
        y = nv.linear_splitk(a, w, segments=dsegs, out_dtype="f32", split_k=s)
        _sync()
        assert rel_fro(y.cpu().numpy(), ref) <= 1e-3, (M, s)


@pytest.mark.parametrize("split_k", [None, 3])
def test_gdn_inproj_decode_full_size(nv, split_k):
    """32 decode tokens through the fused GDN in-projection (12352 x 5120, six
    segments) with the gate epilogue: the library's split count and 3 splits."""
    import torch
    M, K = 32, 5120
    xb = synth.outlier_activations(M, K, seed=60)
    ws = synth.segmented_weights(synth.GDN_INPROJ_SEGMENTS, K, seed=61,
                                 multipliers=synth.GDN_INPROJ_MULTIPLIERS)
    a_log, dt_bias = synth.gdn_gate_params(32, seed=62)
    N = sum(wb.shape[0] for _, wb in ws)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + wb.shape[0], g))
        n0 += wb.shape[0]
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    beta_ref, g_ref = oracle.gdn_gates(y[:, N - 64:N - 32], y[:, N - 32:], a_log, dt_bias)
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    a = nv.quantize(to_dev_bf16(xb))
    beta = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    g = torch.empty((M, 32), dtype=torch.float32, device="cuda")
    gates = dict(beta_begin=N - 64, alpha_begin=N - 32, n_heads=32, A_log=to_dev_f32(a_log),
                 dt_bias=to_dev_f32(dt_bias), beta_out=beta, g_out=g)
    out = nv.linear_splitk(a, w, segments=dsegs, epilogue="gdn_gates", gates=gates, out_dtype="bf16",
                           split_k=split_k)
    _sync()
    assert np.max(np.abs(beta.cpu().numpy() - beta_ref)) <= 1e-3
    assert np.max(np.abs(g.cpu().numpy() - g_ref)) <= 1e-3
    assert_gemm_close(out[:, :N - 64], y[:, :N - 64])


@pytest.mark.parametrize("split_k", [1, 3, 4])
def test_silu_mul_requant_decode(nv, split_k):
    """Gate|up with SiLU*mul and NVFP4 re-quantisation: BF16 output against the oracle;
    the NVFP4 output equals the standalone quantiser applied to the BF16 output, and
    the oracle's quantiser applied to it.  With
    4 K tiles, splits 1, 3 (two K ranges of 2, so 2 splits) and 4."""
    import torch
    M, K, Nh = 32, 1024, 2048
    ws = synth.segmented_weights([("gate", Nh), ("up", Nh)], K, seed=70, multipliers={"gate": 1, "up": 2})
    xb = synth.student_t_activations(M, K, seed=71)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + Nh, g))
        n0 += Nh
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    h_ref = oracle.silu_mul(y[:, :Nh], y[:, Nh:])
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    a = nv.quantize(to_dev_bf16(xb))
    h16 = nv.linear_splitk(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="bf16", split_k=split_k)
    _sync()
    assert_gemm_close(h16, h_ref)
    gs_h = nv.global_scale(h16)
    scales = torch.full((nv.scale_bytes(M, Nh),), 0xAB, dtype=torch.uint8, device="cuda")
    hq = nv.linear_splitk(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h,
                          out_scales=scales, split_k=split_k)
    hq2 = nv.quantize(h16, gs_h)
    _sync()
    assert torch.equal(hq.codes, hq2.codes) and torch.equal(hq.scales, hq2.scales)
    gc, gsf = logical(hq)
    # bit-exact against the oracle's quantiser applied to the kernel's own BF16 h
    kc, ks = oracle.quantize(h16.float().cpu().numpy(), np.float32(gs_h.item()))
    assert np.array_equal(gc, kc) and np.array_equal(gsf, ks)
    rc, rsf = oracle.quantize(oracle.round_to_bf16(h_ref).astype(np.float32), np.float32(gs_h.item()))
    assert np.mean(gc == rc) > 0.995 and np.mean(gsf == rsf) > 0.995


@pytest.mark.parametrize("M", [1, 20, 33, 64])
def test_silu_mul_unsplit_decode(nv, M):
    """One split at decode size: SiLU*mul (and the NVFP4 requant) over the gate and up
    halves of the fused weight.  Token counts on both sides of the 32-row MMA width;
    BF16 and FP32 against the oracle, the NVFP4 output (scale buffer pre-filled with
    0xAB, so padding rows must be zeroed) equal to the standalone quantiser of the BF16
    output and to the oracle's quantiser of it."""
    import torch
    K, Nh = 768, 384
    ws = synth.segmented_weights([("gate", Nh), ("up", Nh)], K, seed=72, multipliers={"gate": 1, "up": 3})
    xb = synth.student_t_activations(M, K, seed=73)
    ca, sa, gsa = oracle_quant(xb)
    oc, os_, oseg, n0 = [], [], [], 0
    for _, wb in ws:
        c, s, g = oracle_quant(wb)
        oc.append(c), os_.append(s), oseg.append((n0, n0 + Nh, g))
        n0 += Nh
    y = oracle.linear(ca, sa, gsa, np.concatenate(oc), np.concatenate(os_), oseg)
    h_ref = oracle.silu_mul(y[:, :Nh], y[:, Nh:])
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    a = nv.quantize(to_dev_bf16(xb))
    h16 = nv.linear_splitk(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="bf16", split_k=1)
    h32 = nv.linear_splitk(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="f32", split_k=1)
    _sync()
    assert_gemm_close(h16, h_ref)
    assert rel_fro(h32.cpu().numpy(), h_ref) <= 1e-3
    assert torch.equal(h32.to(torch.bfloat16), h16)
    gs_h = nv.global_scale(h16)
    scales = torch.full((nv.scale_bytes(M, Nh),), 0xAB, dtype=torch.uint8, device="cuda")
    hq = nv.linear_splitk(a, w, segments=dsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h,
                          out_scales=scales, split_k=1)
    hq2 = nv.quantize(h16, gs_h)
    _sync()
    assert torch.equal(hq.codes, hq2.codes) and torch.equal(hq.scales, hq2.scales)
    gc, gsf = logical(hq)
    kc, ks = oracle.quantize(h16.float().cpu().numpy(), np.float32(gs_h.item()))
    assert np.array_equal(gc, kc) and np.array_equal(gsf, ks)
    assert nv.device_status() == 0


def test_bad_split_and_workspace_rejected(nv):
    import torch
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Error
    M, N, K = 8, 256, 512
    a = nv.quantize(to_dev_bf16(synth.outlier_activations(M, K, seed=80)))
    w = nv.quantize(to_dev_bf16(synth.gaussian_weights(N, K, seed=81)))
    for s in (0, 3):  # K / 256 = 2 K tiles
        with pytest.raises(NVFP4Error):
            nv.linear_splitk(a, w, out_dtype="f32", split_k=s)
    small = torch.empty(nv.splitk_workspace_bytes(M, N, 2) - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(NVFP4Error):
        nv.linear_splitk(a, w, out_dtype="f32", split_k=2, workspace=small)
    assert nv.splitk_workspace_bytes(M, N, 2) == 2 * M * N * 4
