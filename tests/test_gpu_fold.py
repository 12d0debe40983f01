"""GPU parity of the fused-group scale repair (nvfp4_fold_segments) against the oracle,
and the repaired fused GEMM with one global scale."""
import numpy as np
import pytest

import oracle
import synth
from nvfp4_testutil import logical, oracle_quant, rel_fro, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


@pytest.mark.parametrize("K", [5120, 80 * 16])
def test_fold_gdn_inproj_bit_exact_and_gemm(nv, K):
    """The six GDN in-projection modules (segment amaxes up to 16x apart): folded block
    scales bit-exact against the oracle, padding untouched; the one-scale GEMM on the
    folded weight against the oracle's folded linear, and the repair against the
    mismatch it fixes."""
    import torch
    names = synth.GDN_INPROJ_SEGMENTS if K == 5120 else (("q", 256), ("k", 128), ("beta", 32), ("alpha", 32))
    ws = synth.segmented_weights(names, K, seed=110, multipliers=synth.GDN_INPROJ_MULTIPLIERS)
    N = sum(w.shape[0] for _, w in ws)
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    before = w.scales.clone()
    gs_c = nv.fold_segments(w, dsegs)
    torch.cuda.synchronize()
    oq = [oracle_quant(wb) for _, wb in ws]
    folded, ref_gc = oracle.fold_segments([sf for _, sf, _ in oq], [g for _, _, g in oq])
    assert np.float32(gs_c.item()) == ref_gc
    _, got_sf = logical(w)
    assert np.array_equal(got_sf, np.concatenate(folded))
    # the padding bytes (rows past N, blocks past K/16) are unchanged
    from oracle import layout
    mask = np.ones(before.numel(), bool)
    r, j = np.meshgrid(np.arange(N), np.arange(K // 16), indexing="ij")
    mask[layout.scale_offset(r.ravel(), j.ravel(), K)] = False
    assert torch.equal(w.scales.cpu()[torch.from_numpy(mask)], before.cpu()[torch.from_numpy(mask)])
    # GEMM with the single common scale
    M = 64
    xb = synth.outlier_activations(M, K, seed=111)
    ca, sa, gsa = oracle_quant(xb)
    codes = np.concatenate([c for c, _, _ in oq])
    y_fold = oracle.linear(ca, sa, gsa, codes, np.concatenate(folded), [(0, N, ref_gc)])
    a = nv.quantize(to_dev_bf16(xb))
    y = nv.linear(a, w, segments=[(0, N, gs_c)], out_dtype="f32")
    torch.cuda.synchronize()
    assert rel_fro(y.cpu().numpy(), y_fold) <= 1e-3
    # against the per-module linear: the repair removes the mismatch up to re-rounding
    segs, n0 = [], 0
    for c, s, g in oq:
        segs.append((n0, n0 + c.shape[0], g))
        n0 += c.shape[0]
    y_mod = oracle.linear(ca, sa, gsa, codes, np.concatenate([s for _, s, _ in oq]), segs)
    y_shared = oracle.linear(ca, sa, gsa, codes, np.concatenate([s for _, s, _ in oq]), [(0, N, oq[0][2])])
    assert rel_fro(y_shared, y_mod) > 0.5
    assert rel_fro(y.cpu().numpy(), y_mod) < 0.05


def test_fold_rejects_aliased_output(nv):
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Error
    ws = synth.segmented_weights((("a", 32), ("b", 32)), 256, seed=112)
    w, dsegs = nv.quantize_fused([to_dev_bf16(wb) for _, wb in ws])
    with pytest.raises(NVFP4Error):
        nv.fold_segments(w, dsegs, gs_out=dsegs[1][2])
