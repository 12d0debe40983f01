"""GPU checks of the layout entry points against the oracle's layout reading:
nvfp4_unswizzle_scales (swizzled block scales back in logical order) and
nvfp4_pack_weight (separately quantised modules packed into one fused weight, blog
section 罠①: each module keeps its own global scale)."""
import numpy as np
import pytest

import oracle
import synth
from oracle import layout
from nvfp4_testutil import oracle_quant, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


@pytest.mark.parametrize("rows,cols", [(1, 16), (37, 80), (300, 512), (1024, 5120)])
def test_unswizzle_scales_equals_oracle(nv, rows, cols):
    """Logical scales of a quantised tensor: equal to the oracle's quantiser's scales and
    to the oracle's reading of the swizzled buffer; a ragged last 4-block word (cols = 80:
    five blocks) and a strided output leave the bytes past each row untouched."""
    import torch
    xb = synth.student_t_activations(rows, cols, seed=rows + cols)
    _, sf_ref, gs = oracle_quant(xb)
    t = nv.quantize(to_dev_bf16(xb))
    ld = cols // 16 + 3
    out = torch.full((rows, ld), 0xCD, dtype=torch.uint8, device="cuda")
    nv.unswizzle_scales(t, out=out)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.array_equal(got[:, :cols // 16], sf_ref)
    assert np.array_equal(got[:, :cols // 16], layout.unswizzle_scales(t.scales.cpu().numpy(), rows, cols))
    assert (got[:, cols // 16:] == 0xCD).all()
    assert nv.device_status() == 0


def test_pack_weight_equals_fused_quantisation(nv):
    """Three modules quantised one by one, packed at row offsets that split the 128-row
    scale atoms, with padding to 512 rows: byte-identical to quantising them straight into the fused
    buffer (nvfp4_quantize_rows), padding rows zero, and equal to the oracle's per-module
    codes and scales in logical form; the fused linear is the same bit for bit."""
    import torch
    K = 1024
    sizes, mults = [176, 48, 96], [1.0, 4.0, 0.5]  # offsets 0, 176, 224: unaligned to the 128-row atoms
    wbs = [synth.gaussian_weights(n, K, seed=50 + i, std=0.02 * m) for i, (n, m) in enumerate(zip(sizes, mults))]
    total = sum(sizes)
    rows_out = 512
    parts = [nv.quantize(to_dev_bf16(wb)) for wb in wbs]
    packed, segs = nv.pack_weight(parts, rows_out=rows_out)
    fused, fsegs = nv.quantize_fused([to_dev_bf16(wb) for wb in wbs])
    torch.cuda.synchronize()
    pc = packed.codes.cpu().numpy()
    ps = packed.scales.cpu().numpy()
    assert np.array_equal(pc[:total], fused.codes.cpu().numpy())
    assert (pc[total:] == 0).all()
    psf = layout.unswizzle_scales(ps, rows_out, K)
    assert np.array_equal(psf[:total], layout.unswizzle_scales(fused.scales.cpu().numpy(), total, K))
    assert (psf[total:] == 0).all()
    # the scale buffer's own padding (rows 512.. none here; blocks: K % 64 == 0) is zero
    live = np.zeros_like(ps, dtype=bool)
    r, j = np.meshgrid(np.arange(rows_out), np.arange(K // 16), indexing="ij")
    live[layout.scale_offset(r, j, K)] = True
    assert (ps[~live] == 0).all()
    # against the oracle, module by module
    codes_l = layout.unpack_nibbles(pc)
    for (n0, n1, gs), wb in zip(segs, wbs):
        c, s, g = oracle_quant(wb)
        assert float(gs.item()) == float(g)
        assert np.array_equal(codes_l[n0:n1], c) and np.array_equal(psf[n0:n1], s)
    # the fused linear over the packed weight (padding rows give zero columns)
    xb = synth.student_t_activations(256, K, seed=60)
    a = nv.quantize(to_dev_bf16(xb))
    y_packed = nv.linear(a, packed, segments=segs + [(total, rows_out, parts[0].gs)], out_dtype="f32")
    y_fused = nv.linear(a, fused, segments=fsegs, out_dtype="f32")
    torch.cuda.synchronize()
    assert torch.equal(y_packed[:, :total], y_fused)
    assert (y_packed[:, total:] == 0).all()
    assert nv.device_status() == 0
