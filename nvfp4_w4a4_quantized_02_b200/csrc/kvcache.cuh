// FP8 KV cache with static per-tensor scales (blog "27BハイブリッドLLMを4ビットで動かす",
// section "KVキャッシュはFP8で十分？": the attention layers' K and V tensors are cached in
// FP8 with calibrated scales shipped in the checkpoint).  Each token row of K and V is
// written to its cache slot as E4M3(fl32(x * fl32(1 / scale))) (nearest even,
// saturating at +-448, sign kept); a negative slot skips the token.  HBM-bound: 2 bytes
// read and 1 written per element.  A thread handles one 16-element chunk of a token
// row in K and the same chunk in V (one slot read for both); two such chunks are
// loaded before either is converted, so eight 16-byte loads per thread are in flight
// (+3 % over one chunk at 32768 and 131072 tokens of width 1024; four chunks were slower).
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

constexpr int kKvThreads = 256;

struct KvArgs {
  const uint16_t *k, *v;  // BF16 [tokens x width], row stride ld elements
  int64_t tokens, width, ld;
  const float *k_scale, *v_scale;
  const int64_t *slots;   // [tokens]
  uint8_t *k_cache, *v_cache;  // [num_slots x width]
  int64_t num_slots;
};

// 16 BF16 values (two 16-byte words) -> 16 E4M3 bytes of x * inv.
__device__ __forceinline__ uint4 fp8_chunk(const uint4 &w0, const uint4 &w1, float inv) {
  const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  uint32_t out[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float x0 = __fmul_rn(__uint_as_float(w[2 * j] << 16), inv);
    const float x1 = __fmul_rn(__uint_as_float(w[2 * j] & 0xFFFF0000u), inv);
    const float x2 = __fmul_rn(__uint_as_float(w[2 * j + 1] << 16), inv);
    const float x3 = __fmul_rn(__uint_as_float(w[2 * j + 1] & 0xFFFF0000u), inv);
    out[j] = static_cast<uint32_t>(cvt_e4m3x2(x1, x0)) | (static_cast<uint32_t>(cvt_e4m3x2(x3, x2)) << 16);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(kKvThreads) kv_cache_fp8_kernel(const __grid_constant__ KvArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const float k_inv = __frcp_rn(__ldg(a.k_scale)), v_inv = __frcp_rn(__ldg(a.v_scale));
  const int64_t per_row = a.width / 16;
  const bool pow2 = (per_row & (per_row - 1)) == 0;
  const int shift = __ffsll(per_row) - 1;
  const int64_t total = (int64_t)gridDim.x * kKvThreads;
  const int64_t n = a.tokens * per_row;
  // chunk idx = token * per_row + column chunk: shifts when per_row is a power of two
  for (int64_t base = (int64_t)blockIdx.x * kKvThreads + threadIdx.x; base < n; base += 2 * total) {
    uint4 k0[2], k1[2], v0[2], v1[2];  // chunks base and base + total
    int64_t slot[2], dst[2];           // slot -1: nothing to write
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t idx = base + u * total;
      slot[u] = -1;
      if (idx < n) {
        const int64_t t = pow2 ? idx >> shift : idx / per_row;
        const int64_t cc = idx - t * per_row;
        const int64_t sl = __ldg(a.slots + t);
        if (sl >= a.num_slots) {  // never write outside the cache; report it
          atomicCAS(&g_device_status, 0, kStatusBadIndex);
        } else if (sl >= 0) {
          slot[u] = sl;
          const int64_t off = t * a.ld + cc * 16;
          const uint4 *ks = reinterpret_cast<const uint4 *>(a.k + off);
          const uint4 *vs = reinterpret_cast<const uint4 *>(a.v + off);
          k0[u] = __ldcs(ks);
          k1[u] = __ldcs(ks + 1);
          v0[u] = __ldcs(vs);
          v1[u] = __ldcs(vs + 1);
          dst[u] = sl * a.width + cc * 16;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (slot[u] < 0) continue;
      *reinterpret_cast<uint4 *>(a.k_cache + dst[u]) = fp8_chunk(k0[u], k1[u], k_inv);
      *reinterpret_cast<uint4 *>(a.v_cache + dst[u]) = fp8_chunk(v0[u], v1[u], v_inv);
    }
  }
}

// scale = fl32(amax / 448); amax == 0 -> 1.  In place: amax bits in, scale out.
__global__ void fp8_scale_finalize_kernel(float *scale) {
  grid_dep_wait();
  grid_dep_launch();
  const float amax = *scale;
  *scale = amax == 0.0f ? 1.0f : __fdiv_rn(amax, 448.0f);
}

}  // namespace nvfp4
