"""Failure detection on the GPU without a fault: every mbarrier wait in the library's
kernels has a time limit (0.5 s, read from the GPU's global timer), after which the kernel records NVFP4_ERR_DEVICE_TIMEOUT
in the device status word, waits for its own work in flight, frees its TMEM and
returns.  nvfp4_selftest_stalled_linear makes such a wait run out on purpose: the
producer of the 1-CTA GEMM never loads one pipeline stage, and that instantiation's
waits give up after 1 ms.  The test checks the status read-back, that the read
clears it, and that the context then runs a normal linear to parity."""
import numpy as np
import pytest

import oracle
import synth
from nvfp4_testutil import oracle_quant, rel_fro, to_dev_bf16

pytestmark = pytest.mark.gpu

TIMEOUT = 5  # NVFP4_ERR_DEVICE_TIMEOUT


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


@pytest.mark.parametrize("stall_stage", [0, 1, 3])
def test_stalled_pipeline_reports_timeout_and_context_survives(nv, stall_stage):
    import torch
    M, N, K = 128, 256, 1024  # one tile, 4 K tiles (the 4-stage ring never wraps)
    xb = synth.outlier_activations(M, K, seed=40)
    wb = synth.gaussian_weights(N, K, seed=41)
    a = nv.quantize(to_dev_bf16(xb))
    w = nv.quantize(to_dev_bf16(wb))
    assert nv.device_status() == 0
    nv.selftest_stalled_linear(a, w, stall_stage)
    assert nv.device_status() == TIMEOUT
    assert nv.device_status() == 0  # the read cleared it
    # the same context runs the product path to parity afterwards
    out = nv.linear(a, w, out_dtype="f32")
    torch.cuda.synchronize()
    ca, sa, gsa = oracle_quant(xb)
    cw, sw, gsw = oracle_quant(wb)
    ref = oracle.linear(ca, sa, gsa, cw, sw, [(0, N, gsw)])
    assert rel_fro(out.cpu().numpy(), ref) <= 1e-3
    assert nv.device_status() == 0


def test_selftest_rejects_bad_arguments(nv):
    from nvfp4_w4a4_quantized_02_b200 import NVFP4Error
    K = 512
    a = nv.quantize(to_dev_bf16(synth.outlier_activations(128, K, seed=42)))
    w = nv.quantize(to_dev_bf16(synth.gaussian_weights(256, K, seed=43)))
    for bad in (-1, 2):  # 2 K tiles
        with pytest.raises(NVFP4Error) as e:
            nv.selftest_stalled_linear(a, w, bad)
        assert e.value.status == 1
    w2 = nv.quantize(to_dev_bf16(synth.gaussian_weights(512, K, seed=44)))
    with pytest.raises(NVFP4Error) as e:
        nv.selftest_stalled_linear(a, w2, 0)  # two output tiles
    assert e.value.status == 2
    assert nv.device_status() == 0
