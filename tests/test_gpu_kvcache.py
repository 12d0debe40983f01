"""GPU parity of the FP8 KV-cache codec (static per-tensor scales, slot scatter)."""
import numpy as np
import pytest

import oracle
import synth
from nvfp4_testutil import to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _paged_slots(tokens, num_slots, seed, page=16, skip_every=0):
    """Token t -> slot in a shuffled page of `page` slots (a paged cache); every
    `skip_every`-th token gets -1 (a padding token)."""
    rng = np.random.default_rng(seed)
    pages = rng.permutation(num_slots // page)
    t = np.arange(tokens)
    slots = pages[t // page] * page + t % page
    if skip_every:
        slots[::skip_every] = -1
    return slots.astype(np.int64)


@pytest.mark.parametrize("tokens,width,ld", [(300, 1024, 1024), (77, 128, 136), (32768, 1024, 1024)])
def test_kv_cache_bit_exact(nv, tokens, width, ld):
    import torch
    kb = synth.student_t_activations(tokens, ld, seed=130, hot_channels=4)
    vb = synth.student_t_activations(tokens, ld, seed=131, hot_channels=0)
    k = to_dev_bf16(kb)[:, :width]
    v = to_dev_bf16(vb)[:, :width]
    kx, vx = synth.bf16_to_f32(kb)[:, :width], synth.bf16_to_f32(vb)[:, :width]
    ks, vs = nv.fp8_scale(k), nv.fp8_scale(v)
    torch.cuda.synchronize()
    assert np.float32(ks.item()) == oracle.fp8_scale(kx) and np.float32(vs.item()) == oracle.fp8_scale(vx)
    num_slots = ((tokens + 15) // 16) * 16 * 2
    slots = _paged_slots(tokens, num_slots, seed=132, skip_every=7)
    kc = torch.full((num_slots, width), 0x55, dtype=torch.uint8, device="cuda")
    vc = torch.full((num_slots, width), 0x55, dtype=torch.uint8, device="cuda")
    nv.kv_cache_fp8(k, v, ks, vs, torch.from_numpy(slots).cuda(), kc, vc)
    torch.cuda.synchronize()
    init = np.full((num_slots, width), 0x55, np.uint8)
    ref_k = oracle.kv_cache_fp8(kx, np.float32(ks.item()), slots, num_slots, cache=init)
    ref_v = oracle.kv_cache_fp8(vx, np.float32(vs.item()), slots, num_slots, cache=init)
    assert np.array_equal(kc.cpu().numpy(), ref_k)
    assert np.array_equal(vc.cpu().numpy(), ref_v)
    assert nv.device_status() == 0


def test_kv_cache_signs_ties_and_saturation(nv):
    import torch
    vals = oracle.e4m3_decode(np.arange(0x7F))
    mids = (vals[:-1] + vals[1:]) / 2  # exact ties in binary
    row = np.concatenate([vals, -vals, mids[:112], [1e4, -1e4, -0.0, 0.0]])[:448].astype(np.float32)
    row = row[: (len(row) // 16) * 16]
    x = np.stack([row, row * 0.5]).astype(np.float32)
    bits = synth.f32_to_bf16_bits(x)
    xf = synth.bf16_to_f32(bits)
    xd = to_dev_bf16(bits)
    one = torch.ones(1, dtype=torch.float32, device="cuda")
    kc = torch.zeros((2, x.shape[1]), dtype=torch.uint8, device="cuda")
    vc = torch.zeros_like(kc)
    nv.kv_cache_fp8(xd, xd, one, one, torch.tensor([1, 0], dtype=torch.int64, device="cuda"), kc, vc)
    torch.cuda.synchronize()
    ref = oracle.kv_cache_fp8(xf, np.float32(1.0), [1, 0], 2)
    assert np.array_equal(kc.cpu().numpy(), ref)


def test_kv_cache_out_of_range_slot_reported_not_written(nv):
    import torch
    tokens, width = 8, 64
    x = to_dev_bf16(synth.outlier_activations(tokens, width, seed=133))
    s = torch.ones(1, dtype=torch.float32, device="cuda")
    slots = torch.tensor([0, 1, 2, 99, 3, -1, 4, 5], dtype=torch.int64, device="cuda")
    kc = torch.full((6, width), 0x55, dtype=torch.uint8, device="cuda")
    vc = torch.full((6, width), 0x55, dtype=torch.uint8, device="cuda")
    guard = torch.full((4096,), 0x33, dtype=torch.uint8, device="cuda")
    nv.kv_cache_fp8(x, x, s, s, slots, kc, vc)
    assert nv.device_status() == 7  # NVFP4_ERR_DEVICE_INDEX, read and cleared
    assert nv.device_status() == 0
    assert torch.all(guard == 0x33)
    assert not torch.any(kc == 0x55)  # all six slots written by the six valid tokens
