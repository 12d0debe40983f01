"""The split-K linear entry point that allocates nothing (nvfp4_linear_splitk_noalloc).

Some callers cannot allocate device memory for a workspace: a plugin or custom-op
hook that is handed only inputs and outputs, or a serving path that must not call
cudaMalloc (it can synchronise the device).  For them the library keeps the split-K
partial sums in a fixed scratch array of its own.  This test calls that entry point
through the C ABI twice in a row, on two different problems, and checks each result
against the entry point that takes a caller workspace: the same kernels on the same
inputs, so the results must be equal bit for bit.  It lives in a file of its own that
pytest collects last.
"""
import numpy as np
import pytest

import synth
from nvfp4_testutil import rel_fro, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _problem(nv, M, N, K, seed):
    a = nv.quantize(to_dev_bf16(synth.student_t_activations(M, K, seed=seed)))
    w = nv.quantize(to_dev_bf16(synth.gaussian_weights(N, K, seed=seed + 1)))
    return a, w


def test_noalloc_matches_workspace_entry_point_twice(nv):
    import torch
    # call 1: 32 decode tokens through the down projection (5120 outputs in 40 weight
    #         tiles, K = 17408: the one-wave rule picks 3 splits, 3 x 32 x 5120 x 4 = 2 MB
    #         of partials)
    # call 2: a different shape and split count, so stale scratch from call 1 would show
    # Both entry points run the same kernels in the same order on the same inputs, so the
    # results are equal bit for bit.
    for (M, N, K, seed) in [(32, 5120, 17408, 90), (17, 1024, 2048, 92)]:
        a, w = _problem(nv, M, N, K, seed)
        s = nv.splitk_default(M, N, K)
        assert nv.splitk_workspace_bytes(M, N, s) <= nv.NOALLOC_SCRATCH_BYTES
        ref = nv.linear_splitk(a, w, out_dtype="f32", split_k=s)
        ref16 = nv.linear_splitk(a, w, out_dtype="bf16", split_k=s)
        got = nv.linear_splitk_noalloc(a, w, out_dtype="f32", split_k=s)
        got16 = nv.linear_splitk_noalloc(a, w, out_dtype="bf16", split_k=s)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (M, N, K)
        assert torch.equal(got16, ref16), (M, N, K)
        # and the pair agrees with itself across precisions (the BF16 store of the sums)
        assert rel_fro(got16.float().cpu().numpy(), ref.to(torch.bfloat16).float().cpu().numpy()) == 0.0
    assert nv.device_status() == 0


def test_noalloc_default_split_fits_the_scratch(nv):
    """With no split count given, the wrapper lowers the library's default to the largest
    count whose partials fit the fixed array; one split above decode size needs no
    scratch at all and runs the plain kernel."""
    import torch
    # 32 output tiles of 128 x 256, 16 K tiles: the one-wave rule picks 4 splits, whose
    # partials (16 MB) exceed the 8 MB array; 2 splits (8 MB) fit
    M, N, K = 128, 8192, 4096
    a, w = _problem(nv, M, N, K, 96)
    assert nv.splitk_workspace_bytes(M, N, nv.splitk_default(M, N, K)) > nv.NOALLOC_SCRATCH_BYTES
    s = nv.noalloc_default_splits(M, N, K)
    assert 1 <= s <= nv.splitk_default(M, N, K)
    assert s == 1 or nv.splitk_workspace_bytes(M, N, s) <= nv.NOALLOC_SCRATCH_BYTES
    ref = nv.linear_splitk(a, w, out_dtype="f32", split_k=s)
    got = nv.linear_splitk_noalloc(a, w, out_dtype="f32")
    # 384 rows x 8192 outputs at one split: 12 MB of partials would not fit, but one
    # split above decode size runs the plain kernel without partials
    a2, w2 = _problem(nv, 384, 8192, 1024, 98)
    ref2 = nv.linear(a2, w2, out_dtype="f32")
    got2 = nv.linear_splitk_noalloc(a2, w2, out_dtype="f32", split_k=1)
    torch.cuda.synchronize()
    assert torch.equal(got, ref)
    assert torch.equal(got2, ref2)
    assert nv.device_status() == 0


def test_noalloc_rejects_partials_beyond_the_scratch(nv):
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Error
    M, N, K = 128, 4096, 2048  # 8 splits: 128 * 4096 * 8 * 4 = 16 MB > the 8 MB scratch
    a, w = _problem(nv, M, N, K, 94)
    assert nv.splitk_workspace_bytes(M, N, 8) > nv.NOALLOC_SCRATCH_BYTES
    with pytest.raises(NVFP4Error) as e:
        nv.linear_splitk_noalloc(a, w, out_dtype="f32", split_k=8)
    assert e.value.status == 2  # NVFP4_ERR_UNSUPPORTED_SHAPE
