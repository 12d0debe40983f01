// Chunked form of the gated delta-rule recurrence on the tensor cores (blog
// "27BハイブリッドLLMを4ビットで動かす", section "Gated DeltaNetの仕組み"; the per-token form
// and its notation are in gdn.cuh):
//     S_t = alpha_t S_{t-1} + k_t u_t^T,   u_t = beta_t (v_t - S_{t-1}^T k_t),   o_t = S_t^T q_t.
// Over a chunk of C tokens that starts from the state S_0, with the chunk-local
// cumulative log-decays G_t = g_1 + ... + g_t (G_0 = 0), unrolling the recurrence gives
//     (I + L) U = R,   R = diag(beta) (V - diag(e^{G_{t-1}}) K S_0),
//         L[t][s] = beta_t e^{G_{t-1} - G_s} (k_t . k_s) for s < t, else 0;
//     O   = diag(e^{G_t}) Q S_0 + P U,   P[t][s] = e^{G_t - G_s} (q_t . k_s) for s <= t, else 0;
//     S_C = e^{G_C} S_0 + K^T W,         W = diag(e^{G_C - G_s}) U,
// with K, Q, V, U, O the chunk's token rows.  Every exponent is a difference G_a - G_b
// with a >= b, so every factor lies in (0, 1]; g is clamped at -80 (e^-80 is below
// FP32 resolution next to any other term) so that alpha = 0 (g = -inf) gives finite
// differences.  Tokens past a sequence's end are zero rows with g = beta = 0: they
// leave U, O and the state unchanged.
//
// The dense products run as BF16 mma.sync (m16n8k16, FP32 accumulate).  q and k are
// BF16, so K K^T, Q K^T and every product with K or Q as the BF16 operand are exact
// up to FP32 accumulation.  The FP32 operands (the state, U, W and P) are split into
// x = hi + lo with hi = bf16(x), lo = bf16(x - hi) (16 significant bits), and each
// product takes the hi and lo parts (P U also drops the lo x lo term, below 2^-16 of
// the result).  The triangular solve stays in FP32 on the CUDA cores.  These are
// latency-bound products of 64 x 64 .. 128 x 64 tiles in a sequential chunk loop, where
// the register-level mma.sync suits better than a TMEM round trip per product.
//
// A CTA owns one (sequence, value head, block of kCDV value columns): the state block
// (128 x kCDV, FP32) lives in the accumulator registers of the K^T W product (warp w:
// state rows 16 w .. 16 w + 15), and its hi / lo split in shared memory for the K S_0
// and Q S_0 products of the next chunk.
#pragma once

#include "gdn.cuh"

namespace nvfp4 {
namespace gdn {

constexpr int kChunk = 64;              // tokens per chunk
constexpr int kCDV = 64;                // value columns per CTA
constexpr int kChunkColBlocks = kDim / kCDV;
constexpr int kChunkThreads = 256;      // 8 warps
constexpr float kMinLogAlpha = -80.0f;
constexpr int kLdKQ = kDim + 8;         // BF16 row strides: 8-row ldmatrix groups hit distinct banks
constexpr int kLdC = kCDV + 8;
constexpr int kLdT = kChunk + 8;
constexpr int kLdU = kCDV + 4;          // FP32 rows of R / U
constexpr int kLdL = kChunk + 8;        // FP32 rows of L^T, see lt_idx

// L[t][s] is stored at row s (the solve step that reads it), column perm(t) =
// 16 (t % 4) + t / 4 (the solve's lane group t % 4 holds rows t % 4, t % 4 + 4, ...), with
// columns 32 .. 63 shifted by 4 so that the four lane groups read distinct banks.
__host__ __device__ constexpr int lt_col(int t) { return 16 * (t & 3) + (t >> 2); }
__host__ __device__ constexpr int lt_idx(int s, int c) { return s * kLdL + c + 4 * (c >> 5); }

struct ChunkSmem {
  alignas(16) uint16_t K[kChunk][kLdKQ];    // k_t (BF16), token-major
  alignas(16) uint16_t Q[kChunk][kLdKQ];    // q_t
  alignas(16) uint16_t Shi[kDim][kLdC];     // state split, S[i][j]
  alignas(16) uint16_t Slo[kDim][kLdC];
  alignas(16) uint16_t Vb[kChunk][kLdC];    // v_t (this CTA's columns)
  alignas(16) uint16_t Phi[kChunk][kLdT];   // P[t][s] split
  alignas(16) uint16_t Plo[kChunk][kLdT];
  alignas(16) uint16_t Uhi[kChunk][kLdC];   // U split
  alignas(16) uint16_t Ulo[kChunk][kLdC];
  alignas(16) uint16_t Whi[kChunk][kLdC];   // W split
  alignas(16) uint16_t Wlo[kChunk][kLdC];
  alignas(16) float U[kChunk][kLdU];        // R, then U after the solve
  alignas(16) float Lt[kChunk * kLdL];      // L[t][s] at lt_idx(s, t)
  float G[kChunk];                          // G_t for t = 1 .. C at index t - 1
  float eG[kChunk];                         // e^{G_t}
  float eGm[kChunk];                        // e^{G_{t-1}}
  float beta[kChunk];
  float wC[kChunk];                         // e^{G_C - G_s}
};

// One chunk of inputs in flight in registers.  Rows are read as 16-byte pieces with
// consecutive lanes on consecutive pieces of a row: piece p = tid + 256 n of k (and q)
// is token p / 16, d_k columns 8 (p % 16) ..; piece p of v is token p / 8, columns
// 8 (p % 8) .. of this CTA's block.  Thread t < 64 also holds token t's g and beta.
struct ChunkStage {
  uint4 k[4], q[4], v[2];
  float g, b;
};

__device__ __forceinline__ void chunk_load(const Args &a, ChunkStage &st, int64_t t0, int64_t end, int hk, int h,
                                           int cb) {
  const int tid = threadIdx.x;
  const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int p = tid + kChunkThreads * n;
    const int64_t tok = t0 + (p >> 4);
    const int64_t off = tok * a.ld_qk + hk * kDim + (p & 15) * 8;
    st.k[n] = tok < end ? __ldg(reinterpret_cast<const uint4 *>(a.k + off)) : zero;
    st.q[n] = tok < end ? __ldg(reinterpret_cast<const uint4 *>(a.q + off)) : zero;
  }
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int p = tid + kChunkThreads * n;
    const int64_t tok = t0 + (p >> 3);
    const int64_t off = tok * a.ld_v + h * kDim + cb * kCDV + (p & 7) * 8;
    st.v[n] = tok < end ? __ldg(reinterpret_cast<const uint4 *>(a.v + off)) : zero;
  }
  st.g = 0.0f;
  st.b = 0.0f;
  if (tid < kChunk) {
    const int64_t tok = t0 + tid;
    if (tok < end) {
      st.g = fmaxf(__ldg(a.g + tok * a.ld_gate + h), kMinLogAlpha);
      st.b = __ldg(a.beta + tok * a.ld_gate + h);
    }
  }
}

__device__ __forceinline__ void chunk_store(ChunkSmem &sm, const ChunkStage &st) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    const int p = tid + kChunkThreads * n;
    *reinterpret_cast<uint4 *>(&sm.K[p >> 4][(p & 15) * 8]) = st.k[n];
    *reinterpret_cast<uint4 *>(&sm.Q[p >> 4][(p & 15) * 8]) = st.q[n];
  }
#pragma unroll
  for (int n = 0; n < 2; ++n) {
    const int p = tid + kChunkThreads * n;
    *reinterpret_cast<uint4 *>(&sm.Vb[p >> 3][(p & 7) * 8]) = st.v[n];
  }
  if (tid < kChunk) {
    sm.beta[tid] = st.b;
    sm.G[tid] = st.g;  // replaced by the cumulative sums
  }
}

// Writes the chunk's outputs, staged as FP32 rows in sm.U, for its first n tokens from
// token row0: full 16-byte pieces of each row, consecutive lanes on consecutive pieces.
__device__ __forceinline__ void store_outputs(const Args &a, const ChunkSmem &sm, int64_t row0, int n, int h,
                                              int cb) {
  const int tid = threadIdx.x;
  const int64_t col0 = (int64_t)h * kDim + cb * kCDV;
  if (a.out_fp32) {  // 16 pieces of 4 floats per row
#pragma unroll
    for (int i = 0; i < kChunk * kCDV / 4 / kChunkThreads; ++i) {
      const int p = tid + kChunkThreads * i;
      const int t = p >> 4, j = (p & 15) * 4;
      if (t < n)
        *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + (row0 + t) * a.ld_out + col0 + j) =
            *reinterpret_cast<const float4 *>(&sm.U[t][j]);
    }
  } else {  // 8 pieces of 8 BF16 per row
#pragma unroll
    for (int i = 0; i < kChunk * kCDV / 8 / kChunkThreads; ++i) {
      const int p = tid + kChunkThreads * i;
      const int t = p >> 3, j = (p & 7) * 8;
      if (t < n) {
        const float4 x = *reinterpret_cast<const float4 *>(&sm.U[t][j]);
        const float4 y = *reinterpret_cast<const float4 *>(&sm.U[t][j + 4]);
        const __nv_bfloat162 b0 = __floats2bfloat162_rn(x.x, x.y), b1 = __floats2bfloat162_rn(x.z, x.w);
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(y.x, y.y), b3 = __floats2bfloat162_rn(y.z, y.w);
        *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + (row0 + t) * a.ld_out + col0 + j) =
            make_uint4(*reinterpret_cast<const uint32_t *>(&b0), *reinterpret_cast<const uint32_t *>(&b1),
                       *reinterpret_cast<const uint32_t *>(&b2), *reinterpret_cast<const uint32_t *>(&b3));
      }
    }
  }
}

// Inclusive prefix sum over a warp.
__device__ __forceinline__ float warp_scan(float x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// ------------------------------------------------------------ mma.sync helpers
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += a (16 x 16, row-major fragment) * b (16 x 8, K-major fragment b0, b1)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Lane addresses (shared-window byte addresses) of the four 8 x 8 matrices of:
// an A fragment at (r0, k0) of a row-major [rows][ld] BF16 array;
__device__ __forceinline__ uint32_t a_addr(const uint16_t *base, int ld, int r0, int k0, int lane) {
  return smem_u32(base + (r0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + k0 + (lane >> 4) * 8);
}
// two B fragments (n-tiles n0 and n0 + 8) at k0 of an [n][k] (K contiguous) array;
__device__ __forceinline__ uint32_t b_addr_nk(const uint16_t *base, int ld, int n0, int k0, int lane) {
  return smem_u32(base + (n0 + (lane & 7) + (lane >> 4) * 8) * ld + k0 + ((lane >> 3) & 1) * 8);
}
// two B fragments (n-tiles n0 and n0 + 8) at k0 of a [k][n] (N contiguous) array, for
// ldsm_x4_t; also an A fragment at (m0 = n0, k0) of A stored transposed as [k][m]
// (a_t_addr) — the matrix order differs, see below.
__device__ __forceinline__ uint32_t b_addr_kn(const uint16_t *base, int ld, int n0, int k0, int lane) {
  return smem_u32(base + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * ld + n0 + (lane >> 4) * 8);
}
__device__ __forceinline__ uint32_t a_t_addr(const uint16_t *base, int ld, int m0, int k0, int lane) {
  return smem_u32(base + (k0 + (lane & 7) + (lane >> 4) * 8) * ld + m0 + ((lane >> 3) & 1) * 8);
}

__device__ __forceinline__ uint16_t bf16_bits(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t *>(&b);
}
__device__ __forceinline__ float bf16_value(uint16_t b) { return __uint_as_float(static_cast<uint32_t>(b) << 16); }
// x = hi + lo (hi = bf16(x), lo = bf16(x - hi)), stored at hi[0..1], lo[0..1] for x0, x1
__device__ __forceinline__ void split2(float x0, float x1, uint16_t *hi, uint16_t *lo) {
  const uint16_t h0 = bf16_bits(x0), h1 = bf16_bits(x1);
  *reinterpret_cast<uint32_t *>(hi) = static_cast<uint32_t>(h0) | (static_cast<uint32_t>(h1) << 16);
  *reinterpret_cast<uint32_t *>(lo) = static_cast<uint32_t>(bf16_bits(x0 - bf16_value(h0))) |
                                      (static_cast<uint32_t>(bf16_bits(x1 - bf16_value(h1))) << 16);
}

// Grid (kChunkColBlocks, H_v, n_seqs), kChunkThreads threads, sizeof(ChunkSmem) bytes
// of dynamic shared memory.
__global__ void __launch_bounds__(kChunkThreads, 1) chunk_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  ChunkSmem &sm = *reinterpret_cast<ChunkSmem *>(smem_raw);
  const int cb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / a.heads_per_key;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g8 = lane >> 2, c4 = lane & 3;  // fragment row group and column pair of this lane
  // P and Lt above the diagonal blocks stay zero (only the lower blocks are written)
  for (int i = tid; i < kChunk * kLdT; i += kChunkThreads) {
    (&sm.Phi[0][0])[i] = 0;
    (&sm.Plo[0][0])[i] = 0;
  }
  for (int i = tid; i < kChunk * kLdL; i += kChunkThreads) sm.Lt[i] = 0.0f;
  grid_dep_wait();
  grid_dep_launch();
  const int64_t start = __ldg(a.cu_seqlens + b), end = __ldg(a.cu_seqlens + b + 1);
  if (start < 0 || end < start || end > a.tokens) {
    if (tid == 0) atomicCAS(&g_device_status, 0, kStatusBadIndex);
    return;
  }
  // state block in the K^T W accumulators: st[nt][r] = S[16 warp + g8 + 8 (r / 2)][8 nt + 2 c4 + r % 2];
  // global [b][h][j][i] holds S[i][j]
  float *gstate = a.state + (((int64_t)b * gridDim.y + h) * kDim + cb * kCDV) * kDim;
  float st[kCDV / 8][4];
  const int srow = 16 * warp + g8;
#pragma unroll
  for (int nt = 0; nt < kCDV / 8; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = srow + 8 * (r >> 1), j = 8 * nt + 2 * c4 + (r & 1);
      st[nt][r] = a.initial ? gstate[(int64_t)j * kDim + i] : 0.0f;
    }
  auto write_state_split = [&]() {
#pragma unroll
    for (int nt = 0; nt < kCDV / 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = srow + 8 * hh, j = 8 * nt + 2 * c4;
        split2(st[nt][2 * hh], st[nt][2 * hh + 1], &sm.Shi[i][j], &sm.Slo[i][j]);
      }
  };
  write_state_split();

  const int64_t nchunks = (end - start + kChunk - 1) / kChunk;
  ChunkStage stg;
  if (nchunks > 0) chunk_load(a, stg, start, end, hk, h, cb);
  const int mt = warp & 3;   // token rows 16 mt .. of the [C x kCDV] products
  const int nh = warp >> 2;  // value columns 32 nh ..
  for (int64_t c = 0; c < nchunks; ++c) {
    const int64_t c0 = start + c * kChunk;
    __syncthreads();  // the previous chunk is done with every buffer
    if (c > 0) store_outputs(a, sm, c0 - kChunk, kChunk, h, cb);  // the previous chunk's (full) outputs
    chunk_store(sm, stg);
    __syncthreads();
    if (warp == 0) {  // G (inclusive prefix), e^G, e^{G_{t-1}}, e^{G_C - G}: tokens lane, lane + 32
      const float lo = warp_scan(sm.G[lane], lane);
      const float lo31 = __shfl_sync(0xffffffffu, lo, 31);
      const float hi = warp_scan(sm.G[lane + 32], lane) + lo31;
      const float up_lo = __shfl_up_sync(0xffffffffu, lo, 1);
      const float up_hi = __shfl_up_sync(0xffffffffu, hi, 1);
      const float plo = lane == 0 ? 0.0f : up_lo;  // G_{t-1}
      const float phi = lane == 0 ? lo31 : up_hi;
      const float gc = __shfl_sync(0xffffffffu, hi, 31);  // G at the chunk's end
      __syncwarp();
      sm.G[lane] = lo;
      sm.G[lane + 32] = hi;
      sm.eG[lane] = expf(lo);
      sm.eG[lane + 32] = expf(hi);
      sm.eGm[lane] = expf(plo);
      sm.eGm[lane + 32] = expf(phi);
      sm.wC[lane] = expf(gc - lo);
      sm.wC[lane + 32] = expf(gc - hi);
    }
    if (c + 1 < nchunks) chunk_load(a, stg, c0 + kChunk, end, hk, h, cb);
    __syncthreads();

    // ---- K S_0 -> R, Q S_0 (kept in registers): warp tile rows 16 mt, columns 32 nh
    float qs[4][4];
    {
      float ks[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int r = 0; r < 4; ++r) ks[j][r] = qs[j][r] = 0.0f;
#pragma unroll 2
      for (int kk = 0; kk < kDim / 16; ++kk) {
        uint32_t ak[4], aq[4];
        ldsm_x4(a_addr(&sm.K[0][0], kLdKQ, 16 * mt, 16 * kk, lane), ak);
        ldsm_x4(a_addr(&sm.Q[0][0], kLdKQ, 16 * mt, 16 * kk, lane), aq);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bh[4], bl[4];
          const int n0 = 32 * nh + 16 * np;
          ldsm_x4_t(b_addr_kn(&sm.Shi[0][0], kLdC, n0, 16 * kk, lane), bh);
          ldsm_x4_t(b_addr_kn(&sm.Slo[0][0], kLdC, n0, 16 * kk, lane), bl);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            mma16816(ks[2 * np + i], ak, bh[2 * i], bh[2 * i + 1]);
            mma16816(ks[2 * np + i], ak, bl[2 * i], bl[2 * i + 1]);
            mma16816(qs[2 * np + i], aq, bh[2 * i], bh[2 * i + 1]);
            mma16816(qs[2 * np + i], aq, bl[2 * i], bl[2 * i + 1]);
          }
        }
      }
      // R[t][j] = beta_t (v_t[j] - e^{G_{t-1}} (K S_0)[t][j])
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * mt + g8 + 8 * hh;
        const float be = sm.beta[t], em = sm.eGm[t];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = 32 * nh + 8 * j + 2 * c4;
          const uint32_t vv = *reinterpret_cast<const uint32_t *>(&sm.Vb[t][col]);
          const float v0 = __uint_as_float(vv << 16), v1 = __uint_as_float(vv & 0xFFFF0000u);
          *reinterpret_cast<float2 *>(&sm.U[t][col]) =
              make_float2(be * (v0 - em * ks[j][2 * hh]), be * (v1 - em * ks[j][2 * hh + 1]));
        }
      }
    }
    // ---- lower 16 x 16 blocks of K K^T (-> Lt) and Q K^T (-> P split): 20 tasks, warp w
    // runs tasks w, w + 8, w + 16 side by side (independent accumulators)
    {
      constexpr int kTasks = 20, kPer = 3;
      int bt[kPer], bs[kPer];
      bool valid[kPer], is_q[kPer];
#pragma unroll
      for (int x = 0; x < kPer; ++x) {
        const int task = warp + 8 * x;
        valid[x] = task < kTasks;
        is_q[x] = task >= 10;
        int blk = valid[x] ? (is_q[x] ? task - 10 : task) : 0;  // row-major over the lower triangle
        int b = 0;
        while (blk > b) {
          blk -= b + 1;
          ++b;
        }
        bt[x] = b;
        bs[x] = blk;
      }
      float acc[kPer][2][4];
#pragma unroll
      for (int x = 0; x < kPer; ++x)
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[x][i][r] = 0.0f;
#pragma unroll 2
      for (int kk = 0; kk < kDim / 16; ++kk) {
#pragma unroll
        for (int x = 0; x < kPer; ++x) {
          if (!valid[x]) continue;  // warp-uniform
          uint32_t af[4], bf[4];
          ldsm_x4(a_addr(is_q[x] ? &sm.Q[0][0] : &sm.K[0][0], kLdKQ, 16 * bt[x], 16 * kk, lane), af);
          ldsm_x4(b_addr_nk(&sm.K[0][0], kLdKQ, 16 * bs[x], 16 * kk, lane), bf);
          mma16816(acc[x][0], af, bf[0], bf[1]);
          mma16816(acc[x][1], af, bf[2], bf[3]);
        }
      }
#pragma unroll
      for (int x = 0; x < kPer; ++x) {
        if (!valid[x]) continue;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = 16 * bt[x] + g8 + 8 * hh;
          const float gt = sm.G[t], gm = t > 0 ? sm.G[t - 1] : 0.0f, be = sm.beta[t];
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int s = 16 * bs[x] + 8 * i + 2 * c4;
            const float x0 = acc[x][i][2 * hh], x1 = acc[x][i][2 * hh + 1];
            if (is_q[x]) {
              const float p0 = s <= t ? expf(gt - sm.G[s]) * x0 : 0.0f;
              const float p1 = s + 1 <= t ? expf(gt - sm.G[s + 1]) * x1 : 0.0f;
              split2(p0, p1, &sm.Phi[t][s], &sm.Plo[t][s]);
            } else {
              sm.Lt[lt_idx(s, lt_col(t))] = s < t ? be * expf(gm - sm.G[s]) * x0 : 0.0f;
              sm.Lt[lt_idx(s + 1, lt_col(t))] = s + 1 < t ? be * expf(gm - sm.G[s + 1]) * x1 : 0.0f;
            }
          }
        }
      }
    }
    __syncthreads();

    // ---- (I + L) U = R, right-looking, on warps 0 .. 3.  Warp w: columns 16 w .. 16 w + 15;
    // lane (rg, cj): columns 16 w + 2 cj and + 1, rows 4 i + rg (i = 0 .. 15) in registers.
    // At step t the lanes of group t % 4 hold row t (final by then) and broadcast it with
    // two shuffles; every lane subtracts L[t'][t] u_t from its rows t' = 4 i + rg with
    // i >= t / 4 (L[t'][t] = 0 for t' <= t, and every row below 4 (t / 4) is final).  The
    // loop is fully unrolled so that the row range is static: 1088 FMAs per lane instead
    // of 2048 for updating every row at every step.  U and W = diag(e^{G_C - G_s}) U are
    // then split for the tensor cores straight from the registers.
    if (warp < 4) {
      const int rg = lane >> 3, cj = lane & 7;
      const int col = 16 * warp + 2 * cj;
      float r[16][2];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float2 x = *reinterpret_cast<const float2 *>(&sm.U[4 * i + rg][col]);
        r[i][0] = x.x;
        r[i][1] = x.y;
      }
      const float *lrow = &sm.Lt[lt_idx(0, 16 * rg)];  // + lt_idx(t, .) - lt_idx(0, .): row t
#pragma unroll
      for (int t = 0; t < kChunk; ++t) {
        const int i0 = t >> 2;  // first row index still to update
        float l[16];
#pragma unroll
        for (int q = i0 >> 2; q < 4; ++q)
          *reinterpret_cast<float4 *>(&l[4 * q]) = *reinterpret_cast<const float4 *>(lrow + t * kLdL + 4 * q);
        const float u0 = __shfl_sync(0xffffffffu, r[i0][0], (t & 3) * 8 + cj);  // row t
        const float u1 = __shfl_sync(0xffffffffu, r[i0][1], (t & 3) * 8 + cj);
#pragma unroll
        for (int i = i0; i < 16; ++i) {
          r[i][0] = fmaf(-l[i], u0, r[i][0]);
          r[i][1] = fmaf(-l[i], u1, r[i][1]);
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int t = 4 * i + rg;
        const float w = sm.wC[t];
        split2(r[i][0], r[i][1], &sm.Uhi[t][col], &sm.Ulo[t][col]);
        split2(w * r[i][0], w * r[i][1], &sm.Whi[t][col], &sm.Wlo[t][col]);
      }
    }
    __syncthreads();

    // ---- O = diag(e^G) Q S_0 + P U (warp tile as Q S_0), stored for the real tokens
    {
      float o[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int r = 0; r < 4; ++r) o[j][r] = 0.0f;
      for (int kk = 0; kk <= mt; ++kk) {  // P[t][s] = 0 for s > t
        uint32_t ph[4], pl[4];
        ldsm_x4(a_addr(&sm.Phi[0][0], kLdT, 16 * mt, 16 * kk, lane), ph);
        ldsm_x4(a_addr(&sm.Plo[0][0], kLdT, 16 * mt, 16 * kk, lane), pl);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t uh[4], ul[4];
          const int n0 = 32 * nh + 16 * np;
          ldsm_x4_t(b_addr_kn(&sm.Uhi[0][0], kLdC, n0, 16 * kk, lane), uh);
          ldsm_x4_t(b_addr_kn(&sm.Ulo[0][0], kLdC, n0, 16 * kk, lane), ul);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            mma16816(o[2 * np + i], ph, uh[2 * i], uh[2 * i + 1]);
            mma16816(o[2 * np + i], ph, ul[2 * i], ul[2 * i + 1]);
            mma16816(o[2 * np + i], pl, uh[2 * i], uh[2 * i + 1]);
          }
        }
      }
      // staged as FP32 rows in sm.U (no longer needed: U is split) and written out at
      // the next chunk's first barrier
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * mt + g8 + 8 * hh;
        const float e = sm.eG[t];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = 32 * nh + 8 * j + 2 * c4;
          *reinterpret_cast<float2 *>(&sm.U[t][col]) =
              make_float2(fmaf(e, qs[j][2 * hh], o[j][2 * hh]), fmaf(e, qs[j][2 * hh + 1], o[j][2 * hh + 1]));
        }
      }
    }
    // ---- S = e^{G_C} S + K^T W: warp w owns state rows 16 w .. 16 w + 15
    {
      const float ec = sm.eG[kChunk - 1];
#pragma unroll
      for (int nt = 0; nt < kCDV / 8; ++nt)
#pragma unroll
        for (int r = 0; r < 4; ++r) st[nt][r] *= ec;
#pragma unroll
      for (int kk = 0; kk < kChunk / 16; ++kk) {
        uint32_t af[4];
        ldsm_x4_t(a_t_addr(&sm.K[0][0], kLdKQ, 16 * warp, 16 * kk, lane), af);
#pragma unroll
        for (int np = 0; np < kCDV / 16; ++np) {
          uint32_t wh[4], wl[4];
          ldsm_x4_t(b_addr_kn(&sm.Whi[0][0], kLdC, 16 * np, 16 * kk, lane), wh);
          ldsm_x4_t(b_addr_kn(&sm.Wlo[0][0], kLdC, 16 * np, 16 * kk, lane), wl);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            mma16816(st[2 * np + i], af, wh[2 * i], wh[2 * i + 1]);
            mma16816(st[2 * np + i], af, wl[2 * i], wl[2 * i + 1]);
          }
        }
      }
      write_state_split();  // read by the next chunk after its first two barriers
    }
  }
  if (nchunks > 0) {
    __syncthreads();
    const int64_t c0 = start + (nchunks - 1) * kChunk;
    store_outputs(a, sm, c0, static_cast<int>(end - c0), h, cb);
  }
  // final state
#pragma unroll
  for (int nt = 0; nt < kCDV / 8; ++nt)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = srow + 8 * (r >> 1), j = 8 * nt + 2 * c4 + (r & 1);
      gstate[(int64_t)j * kDim + i] = st[nt][r];
    }
}

}  // namespace gdn
}  // namespace nvfp4
