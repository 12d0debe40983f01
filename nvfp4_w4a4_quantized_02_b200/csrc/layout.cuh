// Layout utilities of packed NVFP4 tensors: reading the swizzled block scales back in
// logical order, and packing separately quantised modules into one fused weight.
//
// Blog "27BハイブリッドLLMを4ビットで動かす", section 罠①: modules that run as one GEMM
// (GDN q|k|v|z and b|a, MLP gate|up) keep the global scales they were calibrated
// with.  pack_weight_kernel builds such a fused operand from modules quantised one by
// one (each with its own scale buffer): codes are copied row by row, every scale word
// is moved from the module's 128 x 4 atoms to the fused tensor's, and rows past the
// modules (padding of the output dimension) get zero codes and zero scales.  Both
// kernels are HBM-bound byte movers.
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kLayoutThreads = 256;

struct UnswizzleArgs {
  const uint8_t *scales;  // swizzled [rows x cols] scale buffer
  uint8_t *out;           // logical [rows x kb] E4M3 bytes, row stride ld
  int64_t rows, kb, kb_atoms, ld;
};

// One thread per (row, 4-block word): the word's 4 bytes (fewer in a ragged last word).
__global__ void __launch_bounds__(kLayoutThreads) unswizzle_scales_kernel(const __grid_constant__ UnswizzleArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t total = a.rows * a.kb_atoms;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = t / a.kb_atoms;
    const int64_t ka = t - r * a.kb_atoms;
    const uint32_t w = *reinterpret_cast<const uint32_t *>(a.scales + scale_word_offset(r, ka, a.kb_atoms));
    uint8_t *dst = a.out + r * a.ld + 4 * ka;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (4 * ka + i < a.kb) dst[i] = static_cast<uint8_t>(w >> (8 * i));
  }
}

struct PackArgs {
  int nparts;
  const uint8_t *codes[16];   // module codes [rows_i x cols/2]
  const uint8_t *scales[16];  // module scale buffers (swizzled, own padding)
  int64_t row0[17];           // module i covers fused rows [row0[i], row0[i+1])
  uint8_t *out_codes;         // [rows_out x cols/2]
  uint8_t *out_scales;        // swizzled buffer of [rows_out x cols]
  int64_t rows_out;           // >= row0[nparts]; rows past the modules are zero
  int64_t code_vecs;          // 16-byte code vectors per row (cols / 32)
  int64_t kb_atoms;           // cols / 64
};

__device__ __forceinline__ int pack_part(const PackArgs &a, int64_t r) {
  int i = 0;
  while (i < a.nparts && r >= a.row0[i + 1]) ++i;
  return i;  // == nparts past the modules
}

// Grid-stride over two task lists: 16-byte code vectors of rows [0, rows_out), then
// scale words of rows [0, rows_out padded to 128) (padding rows and rows past the
// modules get zero).
__global__ void __launch_bounds__(kLayoutThreads) pack_weight_kernel(const __grid_constant__ PackArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int64_t n_code = a.rows_out * a.code_vecs;
  const int64_t rows_pad = (a.rows_out + 127) / 128 * 128;
  const int64_t n_sf = rows_pad * a.kb_atoms;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_code + n_sf; t += stride) {
    if (t < n_code) {
      const int64_t r = t / a.code_vecs;
      const int64_t v = t - r * a.code_vecs;
      const int i = pack_part(a, r);
      uint4 w = make_uint4(0, 0, 0, 0);
      if (i < a.nparts) w = reinterpret_cast<const uint4 *>(a.codes[i] + (r - a.row0[i]) * a.code_vecs * 16)[v];
      reinterpret_cast<uint4 *>(a.out_codes + r * a.code_vecs * 16)[v] = w;
    } else {
      const int64_t u = t - n_code;
      const int64_t r = u / a.kb_atoms;
      const int64_t ka = u - r * a.kb_atoms;
      uint32_t w = 0;
      if (r < a.rows_out) {
        const int i = pack_part(a, r);
        if (i < a.nparts)
          w = *reinterpret_cast<const uint32_t *>(a.scales[i] + scale_word_offset(r - a.row0[i], ka, a.kb_atoms));
      }
      *reinterpret_cast<uint32_t *>(a.out_scales + scale_word_offset(r, ka, a.kb_atoms)) = w;
    }
  }
}

}  // namespace nvfp4
