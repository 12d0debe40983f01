"""GPU parity of the gated delta-rule recurrence (GDN layers) against the FP64 oracle.

Tolerance (FP32 state and arithmetic against FP64): the state stays O(1) because every
write is a contraction along a unit key (beta |k|^2 <= 1) and alpha <= 1, so FP32
rounding (2^-24 per operation, 128-term dot products) cannot grow without bound;
outputs and final states must agree to 1e-4 of their largest magnitude.  A BF16 output
adds its own rounding, at most 2^-9 of the value (bounded here by 2^-8 |ref|).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

ABS = 1e-4


@pytest.fixture(scope="module")
def nv():
    import torch
    from nvfp4_w4a4_quantized_02_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_02_b200 as nv
    assert torch.cuda.is_available()
    return nv


def _split(d, hk, hv):
    """FP64 q, k [T, hk, 128] and v [T, hv, 128] from the synthetic rows."""
    T = d["rows"].shape[0]
    f = lambda c, h: synth.bf16_to_f32(d["rows"][:, c:c + h * 128]).astype(np.float64).reshape(T, h, 128)
    return f(d["q_col"], hk), f(d["k_col"], hk), f(d["v_col"], hv)


def _dev_inputs(d, hk, hv, gate_ld=None):
    import torch
    rows = torch.from_numpy(d["rows"].view(np.int16)).cuda().view(torch.bfloat16)
    q = rows[:, d["q_col"]:d["q_col"] + hk * 128]
    k = rows[:, d["k_col"]:d["k_col"] + hk * 128]
    v = rows[:, d["v_col"]:d["v_col"] + hv * 128]
    T = rows.shape[0]
    gl = gate_ld or hv
    g = torch.zeros((T, gl), dtype=torch.float32, device="cuda")
    b = torch.zeros((T, gl), dtype=torch.float32, device="cuda")
    g[:, :hv] = torch.from_numpy(d["g"]).cuda()
    b[:, :hv] = torch.from_numpy(d["beta"]).cuda()
    cu = torch.from_numpy(d["cu_seqlens"]).cuda()
    return q, k, v, g[:, :hv], b[:, :hv], cu


def _oracle(d, hk, hv, S0, heads=None):
    """Per sequence oracle outputs [T, hv, 128] and final states [n, hv, 128, 128]
    (oracle layout S[i, j]); S0 in the library layout [n, hv, j, i] or None.
    `heads` restricts the value heads computed (the others are left NaN)."""
    q, k, v = _split(d, hk, hv)
    cu = d["cu_seqlens"]
    n = len(cu) - 1
    rep = hv // hk
    heads = list(range(hv)) if heads is None else list(heads)
    out = np.full((q.shape[0], hv, 128), np.nan)
    fin = np.full((n, hv, 128, 128), np.nan)
    for s in range(n):
        a, e = cu[s], cu[s + 1]
        for h in heads:
            st = None if S0 is None else S0[s, h].T[None]
            kh = h // rep
            o, S = oracle.gdn_recurrence(q[a:e, kh:kh + 1], k[a:e, kh:kh + 1], v[a:e, h:h + 1],
                                         d["g"][a:e, h:h + 1], d["beta"][a:e, h:h + 1], st)
            out[a:e, h] = o[:, 0]
            fin[s, h] = S[0]
    return out, fin


def _check(got, ref, bf16):
    got = np.asarray(got, np.float64)
    scale = max(1.0, float(np.max(np.abs(ref)))) if ref.size else 1.0
    err = np.abs(got - ref)
    bound = ABS * scale + (2.0 ** -8 * np.abs(ref) if bf16 else 0.0)
    assert np.all(err <= bound), float(np.max(err / np.maximum(bound, 1e-30)))


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("initial", [False, True])
def test_gdn_ragged_sequences(nv, out_dtype, initial):
    """Empty, one-token and ragged sequences across the 32-token staging chunks, strided
    q/k/v rows and strided gate rows, with and without an initial state."""
    import torch
    hk, hv = 2, 4
    lens = [0, 1, 37, 70, 33, 8, 64]
    d = synth.gdn_recurrence_inputs(lens, hk, hv, seed=150, ld=2 * hk * 128 + hv * 128 + 72)
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv, gate_ld=hv + 3)
    rng = np.random.default_rng(151)
    S0 = (0.3 * rng.standard_normal((len(lens), hv, 128, 128))).astype(np.float32)
    state = torch.from_numpy(S0).cuda() if initial else torch.full(S0.shape, np.nan, device="cuda")
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, initial_state=initial, out_dtype=out_dtype)
    torch.cuda.synchronize()
    o_ref, s_ref = _oracle(d, hk, hv, S0 if initial else None)
    T = sum(lens)
    _check(out.float().cpu().numpy().reshape(T, hv, 128), o_ref, out_dtype == "bf16")
    _check(state.cpu().numpy().transpose(0, 1, 3, 2), s_ref, False)
    assert nv.device_status() == 0


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
@pytest.mark.parametrize("initial", [False, True])
def test_gdn_long_ragged_sequences(nv, out_dtype, initial):
    """Long sequences (64 tokens or more per sequence on average, the prefill launch):
    empty, one token, 63, 64 and ragged multi-chunk sequences across the 32-token
    staging chunks, with strided rows and gates, with and without an initial state."""
    import torch
    hk, hv = 2, 4
    lens = [0, 1, 63, 64, 130, 200]
    assert sum(lens) >= 64 * len(lens)
    d = synth.gdn_recurrence_inputs(lens, hk, hv, seed=160, ld=2 * hk * 128 + hv * 128 + 40)
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv, gate_ld=hv + 5)
    rng = np.random.default_rng(161)
    S0 = (0.3 * rng.standard_normal((len(lens), hv, 128, 128))).astype(np.float32)
    state = torch.from_numpy(S0).cuda() if initial else torch.full(S0.shape, np.nan, device="cuda")
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, initial_state=initial, out_dtype=out_dtype)
    torch.cuda.synchronize()
    o_ref, s_ref = _oracle(d, hk, hv, S0 if initial else None)
    T = sum(lens)
    _check(out.float().cpu().numpy().reshape(T, hv, 128), o_ref, out_dtype == "bf16")
    _check(state.cpu().numpy().transpose(0, 1, 3, 2), s_ref, False)
    assert nv.device_status() == 0


def test_gdn_decode_batch(nv):
    """Decode: 32 sequences of one token each over a carried state (one warp per state
    column), all 32 value heads over 16 key heads."""
    import torch
    hk, hv, n = 16, 32, 32
    d = synth.gdn_recurrence_inputs([1] * n, hk, hv, seed=152)
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv)
    rng = np.random.default_rng(153)
    S0 = (0.3 * rng.standard_normal((n, hv, 128, 128))).astype(np.float32)
    state = torch.from_numpy(S0).cuda()
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, out_dtype="f32")
    torch.cuda.synchronize()
    o_ref, s_ref = _oracle(d, hk, hv, S0)
    _check(out.cpu().numpy().reshape(n, hv, 128), o_ref, False)
    _check(state.cpu().numpy().transpose(0, 1, 3, 2), s_ref, False)


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_gdn_decode_few_tokens(nv, out_dtype):
    """Under 4 tokens per sequence on average (the one-warp-per-column path): sequences
    of 3, 1, 0 and 2 tokens, strided rows, a carried state, BF16 and FP32 outputs."""
    import torch
    hk, hv = 2, 4
    lens = [3, 1, 0, 2, 1, 1]
    d = synth.gdn_recurrence_inputs(lens, hk, hv, seed=159, ld=2 * hk * 128 + hv * 128 + 24)
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv, gate_ld=hv + 1)
    rng = np.random.default_rng(160)
    S0 = (0.3 * rng.standard_normal((len(lens), hv, 128, 128))).astype(np.float32)
    state = torch.from_numpy(S0).cuda()
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, out_dtype=out_dtype)
    torch.cuda.synchronize()
    o_ref, s_ref = _oracle(d, hk, hv, S0)
    _check(out.float().cpu().numpy().reshape(sum(lens), hv, 128), o_ref, out_dtype == "bf16")
    _check(state.cpu().numpy().transpose(0, 1, 3, 2), s_ref, False)
    assert nv.device_status() == 0


def test_gdn_resuming_from_the_final_state(nv):
    """Running tokens [0, a) then [a, T) from the first call's final state agrees with one
    call over [0, T) to FP32 rounding: the kernel carries S as A S' with a running decay
    product A, and a split only adds the rounding of the stored A S' (not bit-exact)."""
    import torch
    hk, hv, T, a = 2, 4, 200, 77
    d = synth.gdn_recurrence_inputs([T], hk, hv, seed=154)
    q, k, v, g, b, _ = _dev_inputs(d, hk, hv)
    one = torch.tensor([0, T], dtype=torch.int32, device="cuda")
    s_full = torch.zeros((1, hv, 128, 128), device="cuda")
    o_full = nv.gdn_recurrence(q, k, v, g, b, one, s_full, initial_state=False, out_dtype="f32")
    s_part = torch.zeros((1, hv, 128, 128), device="cuda")
    c1 = torch.tensor([0, a], dtype=torch.int32, device="cuda")
    c2 = torch.tensor([0, T - a], dtype=torch.int32, device="cuda")
    o1 = nv.gdn_recurrence(q[:a], k[:a], v[:a], g[:a], b[:a], c1, s_part, initial_state=False, out_dtype="f32")
    o2 = nv.gdn_recurrence(q[a:], k[a:], v[a:], g[a:], b[a:], c2, s_part, initial_state=True, out_dtype="f32")
    torch.cuda.synchronize()
    for got, ref in ((torch.cat([o1, o2]), o_full), (s_part, s_full)):
        ref = ref.cpu().double()
        assert torch.max(torch.abs(got.cpu().double() - ref)) <= 1e-5 * max(1.0, float(ref.abs().max()))


def test_gdn_full_size_sampled_heads(nv):
    """The prefill workload: 2 sequences x 4096 tokens, 16 key / 32 value heads, read
    straight from in-projection-shaped rows (width 12352: q | k | v | z | beta | alpha),
    BF16 output; the oracle runs the sampled value heads (each its own recurrence)."""
    import torch
    hk, hv = 16, 32
    d = synth.gdn_recurrence_inputs([4096, 4096], hk, hv, seed=155, ld=12352)
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv)
    state = torch.empty((2, hv, 128, 128), device="cuda")
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, initial_state=False)
    torch.cuda.synchronize()
    heads = [0, 1, 14, 31]
    o_ref, s_ref = _oracle(d, hk, hv, None, heads=heads)
    got = out.float().cpu().numpy().reshape(-1, hv, 128)
    fin = state.cpu().numpy().transpose(0, 1, 3, 2)
    for h in heads:
        _check(got[:, h], o_ref[:, h], True)
        _check(fin[:, h], s_ref[:, h], False)
    assert np.all(np.isfinite(got)) and np.all(np.isfinite(fin))
    assert nv.device_status() == 0


@pytest.mark.parametrize("lens,cu_list", [([1, 2, 1], [0, 1, 0, 4]),         # one warp per column
                                          ([5, 3], [0, 5, 3, 8]),            # token-by-token kernel
                                          ([100, 60, 80], [0, 100, 40, 240])])  # chunked kernel
def test_gdn_bad_sequence_bounds_are_skipped_and_reported(nv, lens, cu_list):
    """Sequence 1 runs backwards: it is skipped (its state untouched) and reported; the
    other sequences still run and write their rows."""
    import torch
    hk, hv = 1, 2
    T = sum(lens)
    d = synth.gdn_recurrence_inputs(lens, hk, hv, seed=156)
    q, k, v, g, b, _ = _dev_inputs(d, hk, hv)
    cu = torch.tensor(cu_list, dtype=torch.int32, device="cuda")
    S0 = torch.randn((3, hv, 128, 128), device="cuda")
    state = S0.clone()
    out = torch.full((T, hv * 128), 7.0, device="cuda")
    nv.gdn_recurrence(q, k, v, g, b, cu, state, out=out, out_dtype="f32")
    assert nv.device_status() == 7
    assert torch.equal(state[1], S0[1])
    assert not torch.equal(state[0], S0[0]) and not torch.equal(state[2], S0[2])
    assert torch.all(out[:cu_list[1]] != 7.0) and torch.all(out[cu_list[2]:T] != 7.0)


def test_gdn_strong_decay_and_zero_alpha(nv):
    """Gates that drive the running decay product below 2^-60 within a few tokens (and
    alpha = exp(-200), which is 0 in FP32): the kernel's scaled-state bookkeeping must
    fold the scale back in and still match the recurrence as written."""
    import torch
    hk, hv, T = 1, 2, 100
    d = synth.gdn_recurrence_inputs([T], hk, hv, seed=157)
    d["g"][10] = -200.0
    d["g"][20:60] = -3.0
    d["g"][70:, 1] = -40.0
    q, k, v, g, b, cu = _dev_inputs(d, hk, hv)
    rng = np.random.default_rng(158)
    S0 = rng.standard_normal((1, hv, 128, 128)).astype(np.float32)
    state = torch.from_numpy(S0).cuda()
    out = nv.gdn_recurrence(q, k, v, g, b, cu, state, out_dtype="f32")
    torch.cuda.synchronize()
    o_ref, s_ref = _oracle(d, hk, hv, S0)
    _check(out.cpu().numpy().reshape(T, hv, 128), o_ref, False)
    _check(state.cpu().numpy().transpose(0, 1, 3, 2), s_ref, False)
