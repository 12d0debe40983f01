"""GPU parity of the quantiser against the oracle: bit-exact codes and scales."""
import numpy as np
import pytest

import oracle
import synth
from oracle import layout
from nvfp4_testutil import logical, oracle_quant, to_dev_bf16, to_dev_f32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _check_exact(nv, bits, gs=None, ld_pad=0):
    import torch
    rows, cols = bits.shape
    if ld_pad:
        wide = np.zeros((rows, cols + ld_pad), np.uint16)
        wide[:, :cols] = bits
        x = to_dev_bf16(wide)[:, :cols]
    else:
        x = to_dev_bf16(bits)
    ref_codes, ref_sf, ref_gs = oracle_quant(bits, gs)
    gs_dev = nv.global_scale(x) if gs is None else to_dev_f32([gs])
    torch.cuda.synchronize()
    assert np.float32(gs_dev.item()) == ref_gs, (gs_dev.item(), ref_gs)
    scales = torch.full((nv.scale_bytes(rows, cols),), 0xAB, dtype=torch.uint8, device="cuda")
    qt = nv.quantize(x, gs_dev, scales=scales)
    codes, sf = logical(qt)
    assert np.array_equal(sf, ref_sf), f"{np.sum(sf != ref_sf)} scale mismatches"
    assert np.array_equal(codes, ref_codes), f"{np.sum(codes != ref_codes)} code mismatches"
    # padding bytes of the scale buffer are written as zero
    full = qt.scales.cpu().numpy()
    mask = np.ones(full.size, bool)
    r, j = np.meshgrid(np.arange(rows), np.arange(cols // 16), indexing="ij")
    mask[layout.scale_offset(r, j, cols).ravel()] = False
    assert np.all(full[mask] == 0)
    return qt


def test_config1_activation_and_weight_bit_exact(nv):
    _check_exact(nv, synth.outlier_activations(128, 1024, seed=0))
    _check_exact(nv, synth.gaussian_weights(1024, 1024, seed=1))


def test_ragged_rows_cols_and_leading_dim(nv):
    _check_exact(nv, synth.outlier_activations(300, 80, seed=3), ld_pad=16)
    _check_exact(nv, synth.student_t_activations(129, 1040, seed=4, hot_channels=3))
    _check_exact(nv, synth.gaussian_weights(1, 16, seed=5))


@pytest.mark.parametrize("rows,cols,ld_pad", [(32, 5120, 0), (64, 4096, 0), (33, 80, 8), (7, 1040, 24)])
def test_decode_size_rows(nv, rows, cols, ld_pad):
    """Up to 64 rows (one thread per block, no tile staging): bit-exact codes and scales,
    padding rows and the blocks past the last column written as zero."""
    _check_exact(nv, synth.student_t_activations(rows, cols, seed=7 + rows), ld_pad=ld_pad)


def test_special_values_pin_rounding_and_sign(nv):
    """Ties, saturation, -0, tiny negatives, zero blocks, exact E2M1 multiples."""
    vals = oracle.e2m1_decode(np.arange(16))
    rows = []
    rows.append(np.zeros(64))
    rows.append(-np.zeros(64))
    rows.append(np.concatenate([[-1e-30] * 15 + [6.0], [-0.0] * 15 + [3.0], np.linspace(-6, 6, 32)]))
    rows.append(np.tile(vals, 4))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0])
    rows.append(np.concatenate([mids, -mids, mids * 2, -mids * 2, mids * 0.5, -mids * 0.5, mids * 64, -mids * 64]))
    rng = np.random.default_rng(9)
    rows.append(rng.standard_normal(64) * 1e-6)
    rows.append(np.exp(rng.uniform(-60, 60, 64)) * np.sign(rng.standard_normal(64)))
    x = np.array(rows, dtype=np.float32)
    bits = synth.f32_to_bf16_bits(x)
    _check_exact(nv, bits)
    _check_exact(nv, bits, gs=np.float32(1.0))
    _check_exact(nv, bits, gs=np.float32(1e-3))   # scales underflow to E4M3 subnormals / zero
    _check_exact(nv, bits, gs=np.float32(1e9))    # scales saturate at 448


def test_config2_full_size_all_rows(nv):
    """Activation-quantise workload at full size (32768 x 5120 Student-t with hot
    channels), every row bit-exact against the oracle, and three launches identical
    (a race between tiles of the staged kernel would show up as a difference)."""
    import torch
    rows, cols = 32768, 5120
    bits = synth.student_t_activations(rows, cols, seed=0)
    x = to_dev_bf16(bits)
    gs = nv.global_scale(x)
    ref_gs = oracle.global_scale(synth.bf16_to_f32(bits))
    torch.cuda.synchronize()
    assert np.float32(gs.item()) == ref_gs
    qts = [nv.quantize(x, gs) for _ in range(3)]
    torch.cuda.synchronize()
    for qt in qts[1:]:
        assert torch.equal(qt.codes, qts[0].codes) and torch.equal(qt.scales, qts[0].scales)
    codes_all = qts[0].codes.cpu().numpy()
    scales_all = qts[0].scales.cpu().numpy()
    j = np.arange(cols // 16)
    for r0 in range(0, rows, 2048):
        rr = np.arange(r0, r0 + 2048)
        ref_codes, ref_sf = oracle.quantize(synth.bf16_to_f32(bits[rr]), ref_gs)
        got_sf = scales_all[layout.scale_offset(rr[:, None], j[None, :], cols)]
        assert np.array_equal(got_sf, ref_sf), f"scales differ in rows {r0}..{r0 + 2047}"
        assert np.array_equal(layout.unpack_nibbles(codes_all[rr]), ref_codes), f"codes differ in rows {r0}.."
    # the block holding the tensor amax carries the largest scale
    r, c = np.unravel_index(np.argmax(np.abs(synth.bf16_to_f32(bits))), bits.shape)
    assert scales_all[layout.scale_offset(r, c // 16, cols)] == 0x7E
    assert nv.device_status() == 0


def test_fused_pack_equals_separate_quantisation(nv):
    """quantize_rows packs modules with their own global scales at any row offset."""
    import torch
    parts = [synth.gaussian_weights(r, 256, seed=40 + i, std=0.02 * m)
             for i, (r, m) in enumerate([(48, 1.0), (100, 16.0), (32, 0.5), (16, 2.0)])]
    w, segs = nv.quantize_fused([to_dev_bf16(p) for p in parts])
    torch.cuda.synchronize()
    codes, sf = logical(w)
    n0 = 0
    for p, (b, e, gs) in zip(parts, segs):
        rc, rsf, rgs = oracle_quant(p)
        assert (b, e) == (n0, n0 + p.shape[0])
        assert np.float32(gs.item()) == rgs
        assert np.array_equal(codes[b:e], rc) and np.array_equal(sf[b:e], rsf)
        n0 = e
    full = w.scales.cpu().numpy()
    r, j = np.meshgrid(np.arange(n0), np.arange(256 // 16), indexing="ij")
    mask = np.ones(full.size, bool)
    mask[layout.scale_offset(r, j, 256).ravel()] = False
    assert np.all(full[mask] == 0)


def test_amax_exact(nv):
    """nvfp4_amax: max|x| exactly (a maximum of BF16 magnitudes), over a ragged matrix
    read through a leading dimension wider than its columns, with the maximum on a
    negative entry; an all-zero tensor gives 0, and global_scale is 2688 / amax."""
    import torch
    rows, cols, ld = 333, 496, 512
    xb = synth.student_t_activations(rows, ld, seed=77)
    x = synth.bf16_to_f32(xb)[:, :cols].copy()
    r, c = 201, 417
    x[r, c] = -4.0 * float(np.max(np.abs(x)))
    # columns past `cols` hold a larger magnitude that the kernel must not read
    bits = synth.f32_to_bf16_bits(np.pad(x, ((0, 0), (0, ld - cols)), constant_values=1.0e4))
    dev = to_dev_bf16(bits)
    view = dev[:, :cols]
    got = nv.amax(view)
    gs = nv.global_scale(view)
    z = nv.amax(torch.zeros((4, 32), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    ref = float(np.max(np.abs(synth.bf16_to_f32(bits)[:, :cols])))
    assert float(got.item()) == ref
    assert float(gs.item()) == float(oracle.global_scale(synth.bf16_to_f32(bits)[:, :cols]))
    assert float(z.item()) == 0.0
    assert nv.device_status() == 0
