// FP8 KV cache with static per-tensor scales (blog "27BハイブリッドLLMを4ビットで動かす",
// section "KVキャッシュはFP8で十分？": the attention layers' K and V tensors are cached in
// FP8 with calibrated scales shipped in the checkpoint).  Each token row of K and V is
// written to its cache slot as E4M3(fl32(x / scale)) (nearest even, saturating at +-448,
// sign kept); a negative slot skips the token.  HBM-bound: 2 bytes read and 1 written
// per element.
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kKvThreads = 256;
constexpr int kStatusBadIndex = 7;  // == NVFP4_ERR_DEVICE_INDEX

struct KvArgs {
  const uint16_t *k, *v;  // BF16 [tokens x width], row stride ld elements
  int64_t tokens, width, ld;
  const float *k_scale, *v_scale;
  const int64_t *slots;   // [tokens]
  uint8_t *k_cache, *v_cache;  // [num_slots x width]
  int64_t num_slots;
};

__global__ void __launch_bounds__(kKvThreads) kv_cache_fp8_kernel(const __grid_constant__ KvArgs a) {
  const float ks = __ldg(a.k_scale), vs = __ldg(a.v_scale);
  const int64_t per_row = a.width / 16;
  const int64_t n = a.tokens * per_row;  // 16-element chunks per tensor
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < 2 * n;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const bool is_v = idx >= n;
    const int64_t i = is_v ? idx - n : idx;
    const int64_t t = i / per_row;
    const int64_t c = (i - t * per_row) * 16;
    const int64_t slot = __ldg(a.slots + t);
    if (slot < 0) continue;
    if (slot >= a.num_slots) {  // never write outside the cache; report it
      atomicCAS(&g_device_status, 0, kStatusBadIndex);
      continue;
    }
    const uint4 *src = reinterpret_cast<const uint4 *>((is_v ? a.v : a.k) + t * a.ld + c);
    const uint4 w0 = __ldcs(src), w1 = __ldcs(src + 1);
    const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
    const float s = is_v ? vs : ks;
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float x0 = __fdiv_rn(__uint_as_float(w[2 * j] << 16), s);
      const float x1 = __fdiv_rn(__uint_as_float(w[2 * j] & 0xFFFF0000u), s);
      const float x2 = __fdiv_rn(__uint_as_float(w[2 * j + 1] << 16), s);
      const float x3 = __fdiv_rn(__uint_as_float(w[2 * j + 1] & 0xFFFF0000u), s);
      out[j] = static_cast<uint32_t>(cvt_e4m3x2(x1, x0)) | (static_cast<uint32_t>(cvt_e4m3x2(x3, x2)) << 16);
    }
    uint8_t *dst = (is_v ? a.v_cache : a.k_cache) + slot * a.width + c;
    *reinterpret_cast<uint4 *>(dst) = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

// scale = fl32(amax / 448); amax == 0 -> 1.  In place: amax bits in, scale out.
__global__ void fp8_scale_finalize_kernel(float *scale) {
  const float amax = *scale;
  *scale = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

}  // namespace nvfp4
