// Global scale and NVFP4 block quantisation of BF16 matrices (HBM-bound kernels).
//
// Format: blog "27BハイブリッドLLMを4ビットで動かす" (section 機構①: E2M1 values, one
// E4M3 scale per 16 consecutive elements of a row, the block maximum sets the
// scale; section 罠①: one FP32 global scale per module).  The formulas and their
// FP32 operation order are this library's reading (each step is IEEE FP32, round
// to nearest even, no contraction):
//   gs = 2688 / amax_t ;  s = (amax_b / 6) * gs ;  sf = E4M3(s) ;
//   inv = gs / e4m3(sf) (0 when sf == 0) ;  code = E2M1(x * inv).
//
// quantize_kernel stages the input through shared memory with TMA: a persistent
// CTA walks 128-row x 64-column tiles (16 KB of BF16, one 512-byte scale atom of
// the output), kQStages tiles in flight.  Each thread quantises two blocks of one
// row (64 bytes of the tile, read conflict-free thanks to the 128-byte swizzle),
// stores their 32 codes with one 16-byte store and its half of the row's scale
// word into a shared atom, which 32 threads then write out as 512 contiguous
// bytes.  gs / e4m3(sf) takes one of 127 values per call: it is tabulated once
// per CTA (the same FP32 division, so bit-identical).
//
// Two stages per CTA with four CTAs per SM (the register limit at 256 threads)
// streamed fastest: 0.84 of the measured copy bandwidth at 32768 x 5120 against 0.79
// with four stages and 0.70 with six (more tiles in flight per CTA presumably spread
// the concurrent reads over more DRAM rows).  The codes and scales are stored with the
// default L2 policy (not evict-first): the GEMM that consumes them usually runs next.
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {

// ------------------------------------------------------------------ amax pass
constexpr int kAmaxThreads = 256;

struct AmaxArgs {
  const uint16_t *x;
  int64_t rows, cols, ld;   // cols % 16 == 0, ld % 8 == 0
  unsigned int *amax_bits;  // float bits of max|x|, pre-zeroed
};

__device__ __forceinline__ uint32_t absmax_bits(uint32_t m, const uint4 &v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    m = max(m, w[j] & 0x7FFFu);
    m = max(m, (w[j] >> 16) & 0x7FFFu);
  }
  return m;
}

// max over |x| of the BF16 bit patterns (order-preserving for non-negative values).
// Contiguous rows (ld == cols) are one flat vector stream with eight 16-byte loads in
// flight per thread; otherwise each warp takes whole rows, four loads at a time.
__global__ void __launch_bounds__(kAmaxThreads) amax_kernel(AmaxArgs a) {
  grid_dep_wait();
  grid_dep_launch();
  const int lane = threadIdx.x & 31;
  uint32_t m = 0;
  if (a.ld == a.cols) {
    const uint4 *x = reinterpret_cast<const uint4 *>(a.x);
    const int64_t n = a.rows * a.cols / 8;
    const int64_t T = (int64_t)gridDim.x * blockDim.x;
    int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; v + 7 * T < n; v += 8 * T) {
      uint4 q[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) q[i] = __ldcs(x + v + i * T);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = absmax_bits(m, q[i]);
    }
    for (; v < n; v += T) m = absmax_bits(m, __ldcs(x + v));
  } else {
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t nvec = a.cols / 8;
    for (int64_t r = warp; r < a.rows; r += nwarps) {
      const uint4 *row = reinterpret_cast<const uint4 *>(a.x + r * a.ld);
      int64_t v = lane;
      for (; v + 96 < nvec; v += 128) {
        uint4 q[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) q[i] = __ldcs(row + v + 32 * i);
#pragma unroll
        for (int i = 0; i < 4; ++i) m = absmax_bits(m, q[i]);
      }
      for (; v < nvec; v += 32) m = absmax_bits(m, __ldcs(row + v));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t red[kAmaxThreads / 32];
  if (lane == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kAmaxThreads / 32 ? red[threadIdx.x] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0 && m) atomicMax(a.amax_bits, m << 16);
  }
}

// gs = fl32(2688 / amax); amax == 0 -> 1.  In place: amax bits in, gs out.
__global__ void global_scale_finalize_kernel(float *gs) {
  grid_dep_wait();
  grid_dep_launch();
  const float amax = *gs;
  *gs = amax == 0.0f ? 1.0f : __fdiv_rn(2688.0f, amax);
}

// ------------------------------------------------------------- block quantiser
constexpr int kQThreads = 256;
constexpr int kQTileRows = 128;
constexpr int kQTileCols = 64;
constexpr int kQStages = 2;
constexpr int kQTileBytes = kQTileRows * kQTileCols * 2;  // 16 KB of BF16
constexpr int kQAtomOff = kQStages * kQTileBytes;         // 512-byte scale atom
constexpr int kQInvOff = kQAtomOff + 512;                 // 128 floats: gs / e4m3(sf)
constexpr int kQBarOff = kQInvOff + 512;
constexpr int kQSmemBytes = kQBarOff + 8 * kQStages + 1024;  // + slack to align the base to 1024

struct QuantArgs {
  const float *gs;
  uint8_t *codes;      // codes of the whole destination tensor (row 0)
  uint8_t *scales;     // scale buffer of the whole destination tensor
  int64_t rows, cols;  // source matrix (described by the tensor map)
  int64_t row_offset;  // destination row of source row 0
  int64_t own_end;     // destination rows [row_offset, own_end) are this call's (padding rows included)
  int64_t code_ld;     // bytes per code row (cols / 2)
  int64_t kb_atoms;    // ceil(cols / 64): scale words per row
  int64_t tile_r0;     // first 128-row destination tile (row_offset / 128)
  int64_t n_tiles;     // row tiles x kb_atoms
};

__global__ void __launch_bounds__(kQThreads) quantize_kernel(const __grid_constant__ CUtensorMap tmX,
                                                            const __grid_constant__ QuantArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint32_t *atom = reinterpret_cast<uint32_t *>(smem + kQAtomOff);
  float *inv_tab = reinterpret_cast<float *>(smem + kQInvOff);
  uint64_t *full = reinterpret_cast<uint64_t *>(smem + kQBarOff);
  const int tid = threadIdx.x;
  if (tid == 0) {
    for (int s = 0; s < kQStages; ++s) mbar_init(&full[s], 1);
    fence_barrier_init();
    prefetch_tensormap(&tmX);
  }
  grid_dep_wait();  // gs and the input may come from the previous kernel
  grid_dep_launch();
  const float gs = __ldg(a.gs);
  if (tid < 128) inv_tab[tid] = (tid == 0 || tid == 127) ? 0.0f : __fdiv_rn(gs, e4m3_to_f32(tid));
  __syncthreads();

  const int64_t my_n = a.n_tiles > blockIdx.x ? (a.n_tiles - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  int64_t issued = 0;
  auto issue = [&](int64_t i) {  // thread 0 only
    const int64_t t = blockIdx.x + i * gridDim.x;
    const int64_t rq = t / a.kb_atoms;
    const int s = static_cast<int>(i % kQStages);
    mbar_arrive_expect_tx(&full[s], kQTileBytes);
    tma_load_2d(smem + s * kQTileBytes, &tmX, &full[s], static_cast<int32_t>((t - rq * a.kb_atoms) * kQTileCols),
                static_cast<int32_t>((a.tile_r0 + rq) * kQTileRows - a.row_offset));
  };
  if (tid == 0) {
    for (; issued < my_n && issued < kQStages; ++issued) issue(issued);
  }

  const int rho = tid >> 1;  // tile row of this thread
  const int h = tid & 1;     // which pair of blocks (columns 32h .. 32h+31 of the tile)
  const bool vec16 = (a.code_ld & 15) == 0;
  int64_t done = 0;
  for (int64_t i = 0; i < my_n; ++i) {
    const int s = static_cast<int>(i % kQStages);
    const int64_t t = blockIdx.x + i * gridDim.x;
    const int64_t rq = t / a.kb_atoms;
    const int64_t ka = t - rq * a.kb_atoms;
    const int64_t rt = a.tile_r0 + rq;
    const bool ok = mbar_wait(&full[s], static_cast<uint32_t>((i / kQStages) & 1));
    // 64 bytes of row rho: 16-byte chunks 4h..4h+3, stored at chunk ^ (rho % 8) (128-byte swizzle)
    const uint8_t *rowp = smem + s * kQTileBytes + rho * 128;
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = *reinterpret_cast<const uint4 *>(rowp + (((4 * h + q) ^ (rho & 7)) << 4));
    uint32_t code[4];
    uint32_t sf2 = 0;
#pragma unroll
    for (int b = 0; b < 2; ++b) {
      const uint32_t w[8] = {v[2 * b].x, v[2 * b].y, v[2 * b].z, v[2 * b].w,
                             v[2 * b + 1].x, v[2 * b + 1].y, v[2 * b + 1].z, v[2 * b + 1].w};
      float x[16];
      float amax = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        x[2 * j] = __uint_as_float(w[j] << 16);
        x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
        amax = fmaxf(amax, fmaxf(fabsf(x[2 * j]), fabsf(x[2 * j + 1])));
      }
      const uint32_t sf = block_scale_byte(amax, gs);
      const float inv = inv_tab[sf & 127];  // sf <= 0x7E for finite input
      code[2 * b] = encode8(x, inv);
      code[2 * b + 1] = encode8(x + 8, inv);
      sf2 |= sf << (8 * b);
    }
    // Stage s is refilled by the TMA (async proxy) once every thread is past this
    // point: the proxy fence orders this thread's shared loads of the stage before
    // that write, so the copy cannot overtake a load still in flight.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (__syncthreads_or(!ok)) break;  // (or a copy never landed)
    done = i + 1;
    if (tid == 0 && issued < my_n) issue(issued++);

    const int64_t dest = rt * kQTileRows + rho;
    const bool own = dest >= a.row_offset && dest < a.own_end;
    const int64_t col = ka * kQTileCols + 32 * h;
    if (own && dest - a.row_offset < a.rows && col < a.cols &&
        NVFP4_DCHECK(dest >= 0 && col % 32 == 0 && col / 2 + 8 <= a.code_ld)) {
      uint8_t *dst = a.codes + dest * a.code_ld + col / 2;
      if (col + 32 <= a.cols) {
        if (vec16) {
          __stcg(reinterpret_cast<uint4 *>(dst), make_uint4(code[0], code[1], code[2], code[3]));
        } else {
          __stcg(reinterpret_cast<uint2 *>(dst), make_uint2(code[0], code[1]));
          __stcg(reinterpret_cast<uint2 *>(dst + 8), make_uint2(code[2], code[3]));
        }
      } else {
        __stcg(reinterpret_cast<uint2 *>(dst), make_uint2(code[0], code[1]));  // cols % 16 == 0: one block left
      }
    }
    // scale word of row rho: blocks 0,1 from thread 2*rho, blocks 2,3 from thread 2*rho+1
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, sf2, 1);
    const uint32_t word = sf2 | (other << 16);
    const bool full_atom = rt * kQTileRows >= a.row_offset && rt * kQTileRows + kQTileRows <= a.own_end;
    if (full_atom) {
      if (h == 0) atom[(rho & 31) * 4 + (rho >> 5)] = word;
      __syncthreads();
      if (tid < 32) {
        uint4 *dst = reinterpret_cast<uint4 *>(a.scales + (rt * a.kb_atoms + ka) * 512);
        __stcg(dst + tid, reinterpret_cast<const uint4 *>(atom)[tid]);
      }
    } else if (h == 0 && own && NVFP4_DCHECK(ka >= 0 && ka < a.kb_atoms)) {
      *reinterpret_cast<uint32_t *>(a.scales + scale_word_offset(dest, ka, a.kb_atoms)) = word;
    }
  }
  // error path only: let copies that were issued but not consumed land before exit
  if (tid == 0) {
    for (int64_t i = done; i < issued; ++i)
      mbar_wait(&full[i % kQStages], static_cast<uint32_t>((i / kQStages) & 1));
  }
}

// ---------------------------------------------------- a few rows (decode sizes)
// Up to 64 rows the tile quantiser would stage 128-row tiles that are mostly padding
// and pay its TMA and barrier set-up for a single tile per CTA.  Here one thread
// quantises one 16-element block straight from global memory (two 16-byte loads) with
// quantize16, the same FP32 operations as quantize_kernel, so the output is the same
// bit for bit.  Scale slots of this call's padding rows and of blocks past `cols` (the
// 4-block scale words of the last atom column) are written as zero.
constexpr int kQSmallThreads = 256;

__global__ void __launch_bounds__(kQSmallThreads) quantize_small_kernel(const uint16_t *x, int64_t ld,
                                                                      const __grid_constant__ QuantArgs a) {
  grid_dep_wait();  // gs and the input may come from the previous kernel
  grid_dep_launch();
  const int64_t slots = 4 * a.kb_atoms;  // scale slots per row
  const int64_t idx = (int64_t)blockIdx.x * kQSmallThreads + threadIdx.x;
  if (idx >= (a.own_end - a.row_offset) * slots) return;
  const int64_t r = idx / slots, kb = idx - r * slots;
  const int64_t dest = a.row_offset + r;
  if (!NVFP4_DCHECK(dest < a.own_end && kb < 4 * a.kb_atoms)) return;
  uint8_t *sc = a.scales + scale_word_offset(dest, kb / 4, a.kb_atoms) + (kb & 3);
  if (r >= a.rows || 16 * kb >= a.cols) {
    *sc = 0;
    return;
  }
  const uint4 *src = reinterpret_cast<const uint4 *>(x + r * ld + 16 * kb);
  const uint4 w0 = __ldg(src), w1 = __ldg(src + 1);
  const uint32_t w[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
  float v[16];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    v[2 * j] = __uint_as_float(w[j] << 16);
    v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
  uint32_t c0, c1;
  const uint32_t sf = quantize16(v, __ldg(a.gs), c0, c1);
  *reinterpret_cast<uint2 *>(a.codes + dest * a.code_ld + 8 * kb) = make_uint2(c0, c1);
  *sc = static_cast<uint8_t>(sf);
}

}  // namespace nvfp4
