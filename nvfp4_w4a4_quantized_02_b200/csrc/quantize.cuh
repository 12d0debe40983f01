// NVFP4 quantiser kernels: per-tensor amax -> global scale, and the block
// quantiser (BF16 -> packed E2M1 codes + swizzled E4M3 block scales).
//
// Method: blog "27BハイブリッドLLMを4ビットで動かす", section 機構① (E2M1 values, one
// E4M3 scale per 16 elements, the block maximum sets the scale) and section 罠①
// (a per-tensor global scale per module).  Operation order (all FP32, IEEE round
// to nearest even, no contraction):
//   gs = 2688 / amax_t ;  s = (amax_b / 6) * gs ;  sf = E4M3(s) ;
//   inv = gs / e4m3(sf) (0 when sf == 0) ;  code = E2M1(x * inv).
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kQuantThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- amax pass
struct AmaxArgs {
  const uint16_t *x;
  int64_t rows, cols, ld;
  int64_t chunks_per_row;  // ceil(cols / 64)
  unsigned int *amax_bits; // float bits of max|x|, pre-zeroed
};

__global__ void __launch_bounds__(kQuantThreads) amax_kernel(AmaxArgs a) {
  const int64_t n_chunks = a.rows * a.chunks_per_row;
  uint32_t m = 0;  // max of |bf16| bit patterns (order-preserving for non-negative values)
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < n_chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = c / a.chunks_per_row;
    const int64_t col0 = (c - r * a.chunks_per_row) * 64;
    const int nvec = (int)((a.cols - col0) / 8 < 8 ? (a.cols - col0) / 8 : 8);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x + r * a.ld + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < nvec) {
        uint4 v = __ldg(src + i);
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          m = max(m, w[j] & 0x7FFFu);
          m = max(m, (w[j] >> 16) & 0x7FFFu);
        }
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[kQuantThreads / 32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kQuantThreads / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0 && m) atomicMax(a.amax_bits, m << 16);
  }
}

// gs = fl32(2688 / amax); amax == 0 -> 1.  In place: amax bits in, gs out.
__global__ void global_scale_finalize_kernel(float *gs) {
  const float amax = *gs;
  *gs = amax == 0.0f ? 1.0f : __fdiv_rn(2688.0f, amax);
}

// ------------------------------------------------------------- block quantiser
struct QuantArgs {
  const uint16_t *x;
  int64_t rows, cols, ld;
  const float *gs;
  uint8_t *codes;      // codes of the whole destination tensor (row 0)
  uint8_t *scales;     // scale buffer of the whole destination tensor
  int64_t row_offset;  // destination row of x's row 0
  int64_t rows_cover;  // rows of the destination this call writes scale words for
  int64_t kb_atoms;    // ceil(cols / 64): 4-block scale words per row
};

// One thread per 64-column chunk of a row (4 blocks = one 32-bit scale word).
// Chunks are numbered row-major so a warp streams 4 KB of one row.  Chunks of the
// rows [rows, rows_cover) (padding up to a multiple of 128 after the last rows of
// the destination) only write their (zero) scale word.
__global__ void __launch_bounds__(kQuantThreads) quantize_kernel(QuantArgs a) {
  const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= a.rows_cover * a.kb_atoms) return;
  const int64_t rl = c / a.kb_atoms;
  const int64_t ka = c - rl * a.kb_atoms;
  const int64_t r = a.row_offset + rl;
  uint32_t sfword = 0;
  if (rl < a.rows) {
    const float gs = __ldg(a.gs);
    const int64_t col0 = ka * 64;
    const int nblk = (int)(((a.cols - col0) >> 4) < 4 ? ((a.cols - col0) >> 4) : 4);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x + rl * a.ld + col0);
    uint4 in[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (i < 2 * nblk) {
        in[i] = __ldcs(src + i);  // streamed once: evict-first
      } else {
        in[i] = make_uint4(0, 0, 0, 0);
      }
    }
    uint32_t code[8];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const uint32_t w[8] = {in[2 * b].x, in[2 * b].y, in[2 * b].z, in[2 * b].w,
                             in[2 * b + 1].x, in[2 * b + 1].y, in[2 * b + 1].z, in[2 * b + 1].w};
      float xf[16];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        xf[2 * j] = bf16_lo(w[j]);
        xf[2 * j + 1] = bf16_hi(w[j]);
      }
      const uint32_t sf = quantize16(xf, gs, code[2 * b], code[2 * b + 1]);
      if (b < nblk) sfword |= sf << (8 * b);
    }
    uint8_t *dst = a.codes + r * (a.cols >> 1) + col0 / 2;
    if (nblk == 4 && (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
      uint4 *d4 = reinterpret_cast<uint4 *>(dst);
      __stcs(d4, make_uint4(code[0], code[1], code[2], code[3]));
      __stcs(d4 + 1, make_uint4(code[4], code[5], code[6], code[7]));
    } else {
      uint2 *d2 = reinterpret_cast<uint2 *>(dst);
#pragma unroll
      for (int b = 0; b < 4; ++b)
        if (b < nblk) d2[b] = make_uint2(code[2 * b], code[2 * b + 1]);
    }
  }
  *reinterpret_cast<uint32_t *>(a.scales + scale_word_offset(r, ka, a.kb_atoms)) = sfword;
}

}  // namespace nvfp4
