// The per-block NVFP4 arithmetic shared by the standalone quantiser and the
// GEMM epilogue that re-quantises its output, so that both take every decision
// with the same FP32 operations:
//   s = (amax_b / 6) * gs ; sf = E4M3(s) ; inv = gs / e4m3(sf) (0 if sf == 0) ;
//   code = E2M1(x * inv)
// (blog "27BハイブリッドLLMを4ビットで動かす", section 機構①: 16-element blocks, the
// block maximum sets the E4M3 scale; order of operations is this library's reading).
#pragma once

#include "ptx.cuh"

namespace nvfp4 {

// E4M3 block-scale byte of a block whose maximum magnitude is `amax`.
__device__ __forceinline__ uint32_t block_scale_byte(float amax, float gs) {
  const float s = __fmul_rn(__fdiv_rn(amax, 6.0f), gs);
  return cvt_e4m3x2(0.0f, s) & 0xFFu;
}

// Block scale from the block's amax: returns the E4M3 byte and sets `inv`, the
// factor that maps the block onto the E2M1 grid (0 when the scale is 0).
__device__ __forceinline__ uint32_t block_scale(float amax, float gs, float &inv) {
  const uint32_t sf = block_scale_byte(amax, gs);
  inv = sf == 0 ? 0.0f : __fdiv_rn(gs, e4m3_to_f32(sf));
  return sf;
}

// Eight values -> eight E2M1 codes (element i in nibble i).  The products x * inv are
// IEEE round-to-nearest, two per packed instruction.
__device__ __forceinline__ uint32_t encode8(const float *x, float inv) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const float2 r = mul_f32x2(make_float2(x[i], x[i + 1]), make_float2(inv, inv));
    v[i] = r.x;
    v[i + 1] = r.y;
  }
  return cvt_e2m1x8(v);
}

// x[16] -> E4M3 scale byte (returned) and 16 E2M1 codes in two words (element i in
// nibble i%8 of word i/8).
__device__ __forceinline__ uint32_t quantize16(const float (&x)[16], float gs, uint32_t &c0, uint32_t &c1) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  float inv;
  const uint32_t sf = block_scale(amax, gs, inv);
  c0 = encode8(x, inv);
  c1 = encode8(x + 8, inv);
  return sf;
}

// Swizzled byte offset of the 32-bit scale word holding blocks [4*ka, 4*ka+4) of row r
// (128-row x 4-block atoms of 512 bytes, block index fastest).
__device__ __forceinline__ int64_t scale_word_offset(int64_t r, int64_t ka, int64_t kb_atoms) {
  return ((r >> 7) * kb_atoms + ka) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}

}  // namespace nvfp4
