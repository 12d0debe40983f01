"""The split-K linear entry point that allocates nothing (nvfp4_linear_splitk_noalloc).

Some callers cannot allocate device memory for a workspace: a plugin or custom-op
hook that is handed only inputs and outputs, or a serving path that must not call
cudaMalloc (it can synchronise the device).  For them the library keeps the split-K
partial sums in a fixed scratch array of its own.  This test calls that entry point
through the C ABI twice in a row, on two different problems, and checks each result
against the entry point that takes a caller workspace, within the tolerance the other
linear tests use.  It lives in a file of its own that pytest collects last.
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
    # call 1: 32 decode tokens through the down projection (partials: 7 x 32 x 5120 x 4 = 4.6 MB)
    # call 2: a different shape and split count, so stale scratch from call 1 would show
    for (M, N, K, seed) in [(32, 5120, 17408, 90), (17, 1024, 2048, 92)]:
        a, w = _problem(nv, M, N, K, seed)
        s = nv.splitk_default(M, N, K)
        assert nv.splitk_workspace_bytes(M, N, s) <= nv.NOALLOC_SCRATCH_BYTES
        ref = nv.linear_splitk(a, w, out_dtype="f32", split_k=s)
        got = nv.linear_splitk_noalloc(a, w, out_dtype="f32", split_k=s)
        got16 = nv.linear_splitk_noalloc(a, w, out_dtype="bf16", split_k=s)
        torch.cuda.synchronize()
        r = ref.cpu().numpy()
        assert rel_fro(got.cpu().numpy(), r) <= 1e-3, (M, N, K)
        r16 = ref.to(torch.bfloat16).float().cpu().numpy()
        assert rel_fro(got16.float().cpu().numpy(), r16) <= 1e-3, (M, N, K)
    assert nv.device_status() == 0


def test_noalloc_rejects_partials_beyond_the_scratch(nv):
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Error
    M, N, K = 128, 4096, 2048  # 8 splits: 128 * 4096 * 8 * 4 = 16 MB > the 8 MB scratch
    a, w = _problem(nv, M, N, K, 94)
    assert nv.splitk_workspace_bytes(M, N, 8) > nv.NOALLOC_SCRATCH_BYTES
    with pytest.raises(NVFP4Error) as e:
        nv.linear_splitk_noalloc(a, w, out_dtype="f32", split_k=8)
    assert e.value.status == 2  # NVFP4_ERR_UNSUPPORTED_SHAPE
