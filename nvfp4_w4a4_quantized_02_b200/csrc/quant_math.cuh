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

// x[16] -> E4M3 scale byte (returned) and 16 E2M1 codes in two words (element i in
// nibble i%8 of word i/8).
__device__ __forceinline__ uint32_t quantize16(const float (&x)[16], float gs, uint32_t &c0, uint32_t &c1) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  const float s = __fmul_rn(__fdiv_rn(amax, 6.0f), gs);
  const uint32_t sf = cvt_e4m3x2(0.0f, s) & 0xFFu;
  const float inv = sf == 0 ? 0.0f : __fdiv_rn(gs, e4m3_to_f32(sf));
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(x[i], inv);
  c0 = cvt_e2m1x8(v);
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __fmul_rn(x[8 + i], inv);
  c1 = cvt_e2m1x8(v);
  return sf;
}

// Swizzled byte offset of the 32-bit scale word holding blocks [4*ka, 4*ka+4) of row r
// (128-row x 4-block atoms of 512 bytes, block index fastest).
__device__ __forceinline__ int64_t scale_word_offset(int64_t r, int64_t ka, int64_t kb_atoms) {
  return ((r >> 7) * kb_atoms + ka) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
}

}  // namespace nvfp4
