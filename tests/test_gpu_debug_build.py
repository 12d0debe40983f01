"""The bounds-checking build (libnvfp4_w4a4_debug.so, selected by NVFP4_DEBUG=1): the
same kernels with an index check before every GEMM and quantiser global store, which
records NVFP4_ERR_DEVICE_INDEX and skips the store when it fails.  A child process
runs a spread of entry points on it (quantiser at TMA and decode sizes, the 1-CTA and
CTA-pair GEMMs with segments, SiLU*mul with NVFP4 requant at prefill and decode size,
split-K and the unsplit decode epilogue with GDN gates); every output must equal the product build's bit for
bit and the status word must stay clean."""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CASES = r'''
import numpy as np, torch, synth
import nvfp4_w4a4_quantized_02_b200 as nv

def dev(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()

def run():
    out = {}
    x = dev(synth.student_t_activations(300, 512, seed=5))
    q = nv.quantize(x)
    out["q_codes"], out["q_scales"] = q.codes, q.scales
    qs = nv.quantize(dev(synth.student_t_activations(20, 512, seed=6)))
    out["qs_codes"], out["qs_scales"] = qs.codes, qs.scales
    parts = [dev(synth.gaussian_weights(n, 512, seed=7 + i)) for i, n in enumerate((176, 48, 240))]
    w, segs = nv.quantize_fused(parts)
    out["pair"] = nv.linear(q, w, segments=segs, out_dtype="bf16")
    a100 = nv.quantize(x[:100])
    out["one"] = nv.linear(a100, w, segments=segs, out_dtype="f32")
    gu, gsegs = nv.quantize_fused([dev(synth.gaussian_weights(256, 512, seed=20)),
                                   dev(synth.gaussian_weights(256, 512, seed=21))])
    h16 = nv.linear(q, gu, segments=gsegs, epilogue="silu_mul", out_dtype="bf16")
    gs_h = nv.global_scale(h16)
    hq = nv.linear(q, gu, segments=gsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h)
    out["h16"], out["hq_codes"], out["hq_scales"] = h16, hq.codes, hq.scales
    a32 = nv.quantize(x[:32])
    out["splitk2"] = nv.linear_splitk(a32, w, segments=segs, out_dtype="bf16", split_k=2)
    gq = nv.linear_splitk(a32, gu, segments=gsegs, epilogue="silu_mul", out_dtype="nvfp4", gs_out=gs_h, split_k=1)
    out["gu_dec_codes"], out["gu_dec_scales"] = gq.codes, gq.scales
    beta = torch.zeros((32, 16), dtype=torch.float32, device="cuda")
    g = torch.zeros((32, 16), dtype=torch.float32, device="cuda")
    gates = dict(beta_begin=432, alpha_begin=448, n_heads=16,
                 A_log=torch.linspace(-1, 1, 16, device="cuda"), dt_bias=torch.linspace(-2, 2, 16, device="cuda"),
                 beta_out=beta, g_out=g)
    out["direct"] = nv.linear_splitk(a32, w, segments=segs, epilogue="gdn_gates", gates=gates, out_dtype="bf16",
                                     split_k=1)
    out["beta"], out["g"] = beta, g
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() if v.dtype != torch.bfloat16 else v.view(torch.int16).cpu().numpy()
           for k, v in out.items()}
    res["status"] = np.array([nv.device_status()])
    return res
'''


def test_debug_build_matches_product_build(tmp_path):
    import torch
    import nvfp4_w4a4_quantized_02_b200 as nv
    if nv.DEBUG:
        pytest.skip("compares the debug build with the product build, which this process (NVFP4_DEBUG=1) "
                    "does not load")
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    build.build(debug=True)
    assert torch.cuda.is_available()
    child = tmp_path / "child.py"
    dst = tmp_path / "debug.npz"
    child.write_text(f"import sys\nsys.path.insert(0, {ROOT!r})\nsys.path.insert(0, {os.path.join(ROOT, 'tests')!r})\n"
                     + CASES + f"\nnp.savez({str(dst)!r}, **run())\n")
    env = dict(os.environ, NVFP4_DEBUG="1")
    r = subprocess.run([sys.executable, str(child)], env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    dbg = dict(np.load(dst))
    ns = {}
    exec(CASES, ns)
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert not nv.DEBUG  # this process runs the product build
    rel = ns["run"]()
    assert int(dbg["status"][0]) == 0 and int(rel["status"][0]) == 0
    for k in rel:
        assert np.array_equal(dbg[k], rel[k]), k
