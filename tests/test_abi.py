"""CPU checks of the C-ABI boundary: the library loads, exports every declared entry
point, and rejects bad arguments before touching a device."""
import ctypes
import os
import re

import pytest

import nvfp4_w4a4_quantized_02_b200 as nv
from nvfp4_w4a4_quantized_02_b200 import build as nvbuild
from oracle import layout

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nvfp4.h")


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def declared_symbols():
    src = open(HEADER).read()
    return re.findall(r"NVFP4_API\s+[\w\s\*]+?\b(nvfp4_\w+)\s*\(", src)


def test_header_declares_the_boundary():
    syms = declared_symbols()
    assert set(syms) == set(nv.SYMBOLS), syms


def test_library_exports_every_declared_symbol(L):
    for s in declared_symbols():
        assert hasattr(L, s), s
    out = os.popen(f"nm -D --defined-only {nv.LIB_PATH}").read()
    exported = set(re.findall(r" T (\w+)", out))
    assert set(declared_symbols()) <= exported
    # nothing else of ours leaks out of the library
    assert {s for s in exported if s.startswith("nvfp4")} == set(declared_symbols())


def test_scale_bytes_matches_layout_reading(L):
    for rows, cols in [(1, 16), (128, 64), (129, 80), (300, 512), (32768, 5120), (8192, 17408)]:
        assert nv.scale_bytes(rows, cols) == layout.scale_bytes(rows, cols)
    assert nv.scale_bytes(0, 64) == 0 and nv.scale_bytes(4, 8) == 0 and nv.scale_bytes(4, 24) == 0


def test_status_strings(L):
    names = [L.nvfp4_status_string(i).decode() for i in range(8)]
    assert names[0] == "NVFP4_OK" and names[5] == "NVFP4_ERR_DEVICE_TIMEOUT"
    assert names[7] == "NVFP4_ERR_DEVICE_INDEX"
    assert L.nvfp4_status_string(99).decode() == "NVFP4_ERR_UNKNOWN"


def test_invalid_arguments_rejected_without_launch(L):
    vp = ctypes.c_void_p
    fake = vp(1 << 20)  # never dereferenced: validation fails first
    assert L.nvfp4_quantize(None, 4, 64, 64, fake, fake, fake, None) == 1
    assert L.nvfp4_quantize(fake, 4, 24, 24, fake, fake, fake, None) == 2      # cols % 16
    assert L.nvfp4_quantize(vp((1 << 20) + 2), 4, 64, 64, fake, fake, fake, None) == 3  # x misaligned
    assert L.nvfp4_quantize(fake, 4, 64, 60, fake, fake, fake, None) == 1      # ld < cols
    assert L.nvfp4_global_scale(fake, 4, 64, 64, None, None) == 1
    A = nv.Operand(1 << 20, 1 << 21, 128, 512)
    W = nv.Operand(1 << 22, 1 << 23, 256, 512)
    segs = (nv.Segment * 1)(nv.Segment(0, 256, 1 << 24))
    ep = nv.EpilogueParams()
    call = lambda A_, W_, s, n, epi, okind, ldo, out=fake: L.nvfp4_linear(
        ctypes.byref(A_), fake, ctypes.byref(W_), s, n, epi, ctypes.byref(ep), out, okind, ldo, None)
    A_badk = nv.Operand(1 << 20, 1 << 21, 128, 320)
    W_badk = nv.Operand(1 << 22, 1 << 23, 256, 320)
    assert call(A_badk, W_badk, segs, 1, 0, 0, 256) == 2               # K % 256
    assert call(A, W, segs, 0, 0, 0, 256) == 1                         # no segment
    assert call(A, W, segs, 1, 7, 0, 256) == 1                         # unknown epilogue
    assert call(A, W, segs, 1, 0, 9, 256) == 1                         # unknown output kind
    bad = (nv.Segment * 2)(nv.Segment(0, 128, 1 << 24), nv.Segment(144, 256, 1 << 24))
    assert call(A, W, bad, 2, 0, 0, 256) == 1                          # gap in segments
    odd = (nv.Segment * 2)(nv.Segment(0, 120, 1 << 24), nv.Segment(120, 256, 1 << 24))
    assert call(A, W, odd, 2, 0, 0, 256) == 2                          # bound % 16
    assert call(A, W, segs, 1, 0, 0, 100) == 1                         # ldo < N
    assert call(A, W, segs, 1, 0, 0, 256, out=vp((1 << 20) + 8)) == 3  # out misaligned
    assert call(A, W, segs, 1, 2, 0, 256) == 1                         # gates without params
    assert call(A, W, segs, 1, 0, 2, 0) == 1                           # nvfp4 out without gs_out
    W_odd = nv.Operand(1 << 22, 1 << 23, 384, 512)
    segs384 = (nv.Segment * 1)(nv.Segment(0, 384, 1 << 24))
    assert call(A, W_odd, segs384, 1, 1, 0, 192) == 2                  # silu_mul needs N % 256


def test_splitk_helpers_without_device(L):
    assert L.nvfp4_splitk_workspace_bytes(32, 5120, 7) == 32 * 5120 * 7 * 4
    assert L.nvfp4_splitk_workspace_bytes(0, 5120, 7) == 0
    assert L.nvfp4_splitk_workspace_bytes(32, 5120, 0) == 0
    # invalid sizes are rejected before any device query
    assert L.nvfp4_splitk_default(0, 256, 512) == 0
    assert L.nvfp4_splitk_default(8, 256, 300) == 0


def test_gdn_recurrence_rejects_bad_arguments_without_launch(L):
    vp = ctypes.c_void_p
    f = vp(1 << 20)  # never dereferenced: validation fails first

    def call(q=f, ld_qk=256, ld_v=512, ld_gate=4, n_seqs=1, tokens=8, hk=2, hv=4, d=128, state=f, out=f,
             ld_out=512, kind=0):
        return L.nvfp4_gdn_recurrence(q, f, ld_qk, f, ld_v, f, f, ld_gate, f, n_seqs, tokens, hk, hv, d, state, 1,
                                      out, ld_out, kind, None)
    assert call(q=None) == 1
    assert call(d=64) == 2                        # head_dim must be 128
    assert call(hk=3, hv=4) == 1                  # value heads not a multiple of key heads
    assert call(n_seqs=0) == 1
    assert call(n_seqs=70000) == 2
    assert call(kind=2) == 1                      # NVFP4 output not offered
    assert call(ld_qk=128) == 1                   # 2 key heads need 256 columns
    assert call(ld_v=256) == 1
    assert call(ld_gate=3) == 1
    assert call(ld_out=500) == 1
    assert call(q=vp((1 << 20) + 8)) == 3         # q not 16-byte aligned
    assert call(ld_qk=260) == 3                   # row stride not a multiple of 8 BF16
    assert call(state=vp((1 << 20) + 4)) == 3
    assert call(ld_out=516) == 3                  # BF16 out rows must stay 16-byte aligned


def test_splitk_rejects_bad_split_and_workspace_without_launch(L):
    """The split count and the workspace are checked before any device work: split 0 or
    above K / 256, no workspace, too small or misaligned a workspace; the no-alloc
    variant rejects partials beyond its fixed scratch array."""
    vp = ctypes.c_void_p
    fake = vp(1 << 20)
    A = nv.Operand(1 << 20, 1 << 21, 8, 512)        # 8 rows, K = 512: 2 K tiles
    W = nv.Operand(1 << 22, 1 << 23, 256, 512)
    segs = (nv.Segment * 1)(nv.Segment(0, 256, 1 << 24))
    ep = nv.EpilogueParams()
    need = L.nvfp4_splitk_workspace_bytes(8, 256, 2)

    def call(split, ws=fake, ws_bytes=need):
        return L.nvfp4_linear_splitk(ctypes.byref(A), fake, ctypes.byref(W), segs, 1, 0, ctypes.byref(ep), fake, 0,
                                     256, split, ws, ws_bytes, None)
    assert call(0) == 1                                 # split 0
    assert call(3) == 1                                 # more splits than K tiles
    assert call(2, ws=None) == 1                        # no workspace
    assert call(2, ws_bytes=need - 16) == 1             # workspace too small
    assert call(2, ws=vp((1 << 20) + 8)) == 3           # workspace not 16-byte aligned
    big_W = nv.Operand(1 << 22, 1 << 23, 65536, 512)
    big_segs = (nv.Segment * 1)(nv.Segment(0, 65536, 1 << 24))
    big_A = nv.Operand(1 << 20, 1 << 21, 64, 512)
    # 2 x 64 x 65536 FP32 partials (32 MiB) do not fit the 8 MiB no-alloc scratch
    assert L.nvfp4_linear_splitk_noalloc(ctypes.byref(big_A), fake, ctypes.byref(big_W), big_segs, 1, 0,
                                         ctypes.byref(ep), fake, 0, 65536, 2, None) == 2


def test_layout_and_selftest_entry_points_reject_bad_arguments_without_launch(L):
    vp = ctypes.c_void_p
    f = vp(1 << 20)  # never dereferenced: validation fails first
    # nvfp4_unswizzle_scales(scales, rows, cols, out, ld, stream)
    assert L.nvfp4_unswizzle_scales(None, 4, 64, f, 4, None) == 1
    assert L.nvfp4_unswizzle_scales(f, 0, 64, f, 4, None) == 1
    assert L.nvfp4_unswizzle_scales(f, 4, 64, f, 3, None) == 1          # ld < cols / 16
    assert L.nvfp4_unswizzle_scales(f, 4, 72, f, 8, None) == 2          # cols % 16
    assert L.nvfp4_unswizzle_scales(vp((1 << 20) + 4), 4, 64, f, 4, None) == 3
    # nvfp4_pack_weight(parts, nparts, codes, scales, rows_out, stream)
    parts = (nv.Operand * 2)(nv.Operand(1 << 20, 1 << 21, 100, 512), nv.Operand(1 << 22, 1 << 23, 28, 512))
    assert L.nvfp4_pack_weight(parts, 0, f, f, 128, None) == 1
    assert L.nvfp4_pack_weight(parts, 2, f, f, 127, None) == 1          # rows_out below the modules' rows
    assert L.nvfp4_pack_weight(parts, 2, None, f, 128, None) == 1
    assert L.nvfp4_pack_weight(parts, 2, vp((1 << 20) + 8), f, 128, None) == 3
    odd = (nv.Operand * 2)(nv.Operand(1 << 20, 1 << 21, 100, 544), nv.Operand(1 << 22, 1 << 23, 28, 544))
    assert L.nvfp4_pack_weight(odd, 2, f, f, 128, None) == 2            # K % 64
    mixed = (nv.Operand * 2)(nv.Operand(1 << 20, 1 << 21, 100, 512), nv.Operand(1 << 22, 1 << 23, 28, 1024))
    assert L.nvfp4_pack_weight(mixed, 2, f, f, 128, None) == 1          # modules of different K
    # nvfp4_selftest_stalled_linear: one tile only, stall stage inside the K tiles
    A = nv.Operand(1 << 20, 1 << 21, 128, 512)
    W = nv.Operand(1 << 22, 1 << 23, 256, 512)
    segs = (nv.Segment * 1)(nv.Segment(0, 256, 1 << 24))
    call = lambda A_, W_, s_, stall: L.nvfp4_selftest_stalled_linear(ctypes.byref(A_), f, ctypes.byref(W_), s_, 1,
                                                                     f, 512, stall, None)
    assert call(A, W, segs, -1) == 1
    assert call(A, W, segs, 2) == 1                                       # 2 K tiles
    W2 = nv.Operand(1 << 22, 1 << 23, 512, 512)
    segs2 = (nv.Segment * 1)(nv.Segment(0, 512, 1 << 24))
    assert call(A, W2, segs2, 0) == 2                                     # two output tiles


def test_debug_build_exports_the_same_boundary():
    """The bounds-checking build (-DNVFP4_DEBUG) compiles and exports exactly the
    declared entry points; it rejects bad arguments like the product build."""
    path = nvbuild.build(debug=True)
    out = os.popen(f"nm -D --defined-only {path}").read()
    exported = {s for s in re.findall(r" T (\w+)", out) if s.startswith("nvfp4")}
    assert exported == set(declared_symbols())
    D = ctypes.CDLL(path)
    fake = ctypes.c_void_p(1 << 20)
    assert D.nvfp4_quantize(None, 4, 64, 64, fake, fake, fake, None) == 1
    assert D.nvfp4_quantize(fake, 4, 24, 24, fake, fake, fake, None) == 2


def test_amax_rejects_bad_arguments_without_launch(L):
    vp = ctypes.c_void_p
    f = vp(1 << 20)
    assert L.nvfp4_amax(None, 4, 64, 64, f, None) == 1
    assert L.nvfp4_amax(f, 4, 64, 64, None, None) == 1
    assert L.nvfp4_amax(f, 4, 64, 60, f, None) == 1          # ld < cols
    assert L.nvfp4_amax(f, 4, 72, 72, f, None) == 2          # cols % 16
    assert L.nvfp4_amax(vp((1 << 20) + 2), 4, 64, 64, f, None) == 3
    assert L.nvfp4_amax(f, 4, 64, 68, f, None) == 3          # ld % 8
