// Fused-group repair of a packed NVFP4 weight (blog "27BハイブリッドLLMを4ビットで動かす",
// section 罠①: the modules fused into one GEMM are rewritten to a common global scale
// and the ratio is folded into their block scales).  The common scale is the smallest
// module scale, so every ratio is <= 1 and no block scale saturates; every block scale
// of module i becomes E4M3(dec(sf) * fl32(gs_c / gs_i)) (nearest even, FP32 product);
// codes are untouched.  HBM-bound over the scale buffer (1/16 byte per element).
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kFoldThreads = 256;

struct FoldArgs {
  uint8_t *scales;   // swizzled scale buffer of the fused weight, rewritten in place
  int64_t rows;      // weight rows (= GEMM output columns)
  int64_t kb;        // blocks per row (cols / 16)
  int64_t kb_atoms;  // ceil(kb / 4)
  int64_t bytes;     // scale buffer bytes (multiple of 512)
  int nseg;
  int seg_begin[16], seg_end[16];
  const float *gs[16];
  float *gs_common;  // out: min of the module scales (written by thread 0 of CTA 0)
};

__global__ void __launch_bounds__(kFoldThreads) fold_scales_kernel(const __grid_constant__ FoldArgs a) {
  __shared__ float ratio[16];
  __shared__ float gs_c;
  grid_dep_wait();
  grid_dep_launch();
  if (threadIdx.x == 0) {
    float m = __ldg(a.gs[0]);
    for (int i = 1; i < a.nseg; ++i) m = fminf(m, __ldg(a.gs[i]));
    gs_c = m;
    if (blockIdx.x == 0) *a.gs_common = m;
  }
  __syncthreads();
  if (threadIdx.x < a.nseg) ratio[threadIdx.x] = __fdiv_rn(gs_c, __ldg(a.gs[threadIdx.x]));
  __syncthreads();
  const int64_t n16 = a.bytes / 16;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < n16; v += (int64_t)gridDim.x * blockDim.x) {
    uint4 w = reinterpret_cast<const uint4 *>(a.scales)[v];
    uint8_t *b = reinterpret_cast<uint8_t *>(&w);
    const int64_t o0 = v * 16;
    const int64_t atom = o0 >> 9;
    const int64_t arow = atom / a.kb_atoms;
    const int64_t acol = atom - arow * a.kb_atoms;
    const int within = static_cast<int>(o0 & 511);  // 16 bytes: one TMEM-lane row of the atom
    const int64_t r0 = arow * 128 + (within >> 4);  // rows r0 + 32 * (byte / 4)
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int64_t r = r0 + 32 * (i >> 2);
      const int64_t j = acol * 4 + (i & 3);
      if (r >= a.rows || j >= a.kb) continue;  // padding stays as it is
      float rt = 1.0f;
      for (int s = 0; s < a.nseg; ++s)
        if (r >= a.seg_begin[s] && r < a.seg_end[s]) rt = ratio[s];
      const float sv = __fmul_rn(e4m3_to_f32(b[i]), rt);
      b[i] = static_cast<uint8_t>(cvt_e4m3x2(0.0f, sv) & 0xFFu);
    }
    reinterpret_cast<uint4 *>(a.scales)[v] = w;
  }
}

}  // namespace nvfp4
