// Block-scaled NVFP4 x NVFP4 GEMM for sm_100a (tcgen05, TMEM accumulators, TMA),
// with the fused-module per-segment global-scale correction and the epilogues of
// the W4A4 linear.
//
// Method: blog "27BハイブリッドLLMを4ビットで動かす", FAQ (W4A4 runs on 4-bit tensor
// cores), section 罠① (modules fused into one GEMM keep their own global scales:
// here every output column n is scaled by alpha = 1 / (gs_A * gs_W[seg(n)])),
// section 機構② (GDN gates beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias)).
//
// Kernel structure (one persistent CTA per SM, 320 threads):
//   warp 0      TMA producer: A / W code tiles (cp.async.bulk.tensor, 128-byte
//               swizzle) and their scale tiles (cp.async.bulk, already in the
//               MMA's atom layout) into a 4-stage shared-memory ring.
//   warp 1      MMA issuer: copies the stage's scales to TMEM (tcgen05.cp), issues
//               4 tcgen05.mma kind::mxf4nvf4 (128 x 256 x 64 each) into the TMEM
//               accumulator, and frees the stage with tcgen05.commit.
//   warps 2..9  epilogue: tcgen05.ld the 128 x 256 FP32 accumulator (each warp a
//               32-lane quadrant x 128 columns) into registers, hand TMEM back to the
//               MMA warp at once, then scale / activate / store from registers.
// Tile 128 x 256 x 256 (K in FP4 elements); output tiles are visited in groups of
// 16 M-tiles so that concurrently running CTAs share A and W tiles in L2.
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 256;                  // FP4 elements per stage = 128 bytes per row
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK / 2;     // 16 KB
constexpr int B_HALF_BYTES = 128 * BK / 2;
constexpr int B_BYTES = BN * BK / 2;     // 32 KB
constexpr int SF_ATOM = 512;             // 128 rows x 4 scale bytes
constexpr int SFA_BYTES = 4 * SF_ATOM;   // 4 MMA k-steps
constexpr int SFB_HALF_BYTES = 4 * SF_ATOM;
constexpr int SFB_BYTES = 2 * SFB_HALF_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int GROUP_M = 16;

// TMEM columns (allocation of 512 = the whole TMEM of the SM)
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;     // 256 FP32 columns
constexpr uint32_t SFA_COL = 256;   // 4 k-steps x 4 columns
constexpr uint32_t SFB_COL = 272;   // 4 k-steps x 8 columns

constexpr int CTRL_BYTES = 1024;
constexpr int SMEM_A_OFF = CTRL_BYTES;
constexpr int SMEM_B_OFF = SMEM_A_OFF + STAGES * A_BYTES;
constexpr int SMEM_SFA_OFF = SMEM_B_OFF + STAGES * B_BYTES;
constexpr int SMEM_SFB_OFF = SMEM_SFA_OFF + STAGES * SFA_BYTES;
constexpr int SMEM_END = SMEM_SFB_OFF + STAGES * SFB_BYTES;
constexpr int SMEM_BYTES = SMEM_END + 1024;  // slack to align the base to 1024

enum Mode : int { MODE_NONE = 0, MODE_SILU_MUL = 1, MODE_GDN = 2 };
enum OutKind : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_NVFP4 = 2 };

struct Segment {
  int n_begin, n_end;
  const float *gs_w;
};

struct Params {
  int M, N, K, Nout;
  int mode, out_kind;
  int m_tiles, n_tiles, k_tiles;
  int up_row0;              // SILU_MUL: first weight row of the `up` half
  int64_t kb_atoms;         // K / 64
  const uint8_t *sfa;       // swizzled scales of A
  const uint8_t *sfb;       // swizzled scales of W
  int w_rows_pad;           // W rows padded to 128 (rows present in sfb)
  const float *gs_a;
  int nseg;
  Segment seg[16];
  void *out;
  int64_t ldo;
  // GDN gates
  int beta_begin, alpha_begin, n_heads;
  const float *A_log, *dt_bias;
  float *beta_out, *g_out;
  // NVFP4 output
  const float *gs_out;
  uint8_t *out_scales;
  int64_t out_kb_atoms;
};

struct Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint32_t tmem_base;
  int seg_begin[16];
  int seg_end[16];
  float seg_alpha[16];
};
static_assert(sizeof(Ctrl) <= CTRL_BYTES, "control block too large");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: E2M1 A and B (format 1),
// UE4M3 scales, K-major operands, M = 128, N = 256, dense K = 64, scale ids 0.
__host__ __device__ constexpr uint32_t make_idesc(int m, int n) {
  return (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void tile_coords(const Params &p, int tile, int &mt, int &nt) {
  const int per_group = GROUP_M * p.n_tiles;
  const int g = tile / per_group;
  const int idx = tile - g * per_group;
  const int gm = min(GROUP_M, p.m_tiles - g * GROUP_M);
  mt = g * GROUP_M + idx % gm;
  nt = idx / gm;
}

// First weight rows of the two 128-row halves of the B tile of N-tile nt.
__device__ __forceinline__ void b_rows(const Params &p, int nt, int &rb0, int &rb1) {
  if (p.mode == MODE_SILU_MUL) {
    rb0 = nt * 128;
    rb1 = p.up_row0 + nt * 128;
  } else {
    rb0 = nt * BN;
    rb1 = nt * BN + 128;
  }
}

__device__ __forceinline__ float seg_alpha(const Ctrl &c, int nseg, int n) {
  float a = 0.0f;
  for (int s = 0; s < nseg; ++s)
    if (n >= c.seg_begin[s] && n < c.seg_end[s]) a = c.seg_alpha[s];
  return a;
}

__device__ __forceinline__ float sigmoid_f(float x) { return 1.0f / (1.0f + expf(-x)); }
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.0f) + log1pf(expf(-fabsf(x))); }

// Store 16 consecutive output values of one row.
__device__ __forceinline__ void store16(const Params &p, int row, int col, const float (&y)[16]) {
  if (p.out_kind == OUT_BF16) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.ldo + col);
    dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
    dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
  } else if (p.out_kind == OUT_F32) {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (int64_t)row * p.ldo + col);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
  }
}

// Re-quantise 64 consecutive outputs (one scale word) of one row: round to BF16,
// then the NVFP4 block quantiser with the output's global scale.
__device__ __forceinline__ void store64_nvfp4(const Params &p, int row, int col, const float (&y)[64],
                                              float gs_out) {
  uint32_t codes[8];
  uint32_t sfword = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = __bfloat162float(__float2bfloat16_rn(y[16 * b + i]));
    const uint32_t sf = quantize16(x, gs_out, codes[2 * b], codes[2 * b + 1]);
    sfword |= sf << (8 * b);
  }
  uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint8_t *>(p.out) + (int64_t)row * (p.Nout / 2) + col / 2);
  dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
  dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
  *reinterpret_cast<uint32_t *>(p.out_scales + scale_word_offset(row, col / 64, p.out_kb_atoms)) = sfword;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl &c = *reinterpret_cast<Ctrl *>(smem);
  uint8_t *sA = smem + SMEM_A_OFF;
  uint8_t *sB = smem + SMEM_B_OFF;
  uint8_t *sSFA = smem + SMEM_SFA_OFF;
  uint8_t *sSFB = smem + SMEM_SFB_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
    }
    mbar_init(&c.acc_full, 1);
    mbar_init(&c.acc_empty, NUM_EPI_WARPS);
    mbar_init(&c.drain, 1);
    fence_barrier_init();
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + p.nseg) {
    const int s = threadIdx.x - 64;
    c.seg_begin[s] = p.seg[s].n_begin;
    c.seg_end[s] = p.seg[s].n_end;
    c.seg_alpha[s] = __frcp_rn(__fmul_rn(__ldg(p.gs_a), __ldg(p.seg[s].gs_w)));
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int num_tiles = p.m_tiles * p.n_tiles;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;  // per-stage bit masks
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int mt, nt, rb0, rb1;
        tile_coords(p, tile, mt, nt);
        b_rows(p, nt, rb0, rb1);
        const bool second = rb1 < p.N;  // any valid row in the second half
        const uint32_t bytes = A_BYTES + B_HALF_BYTES + SFA_BYTES + SFB_HALF_BYTES +
                               (second ? (B_HALF_BYTES + SFB_HALF_BYTES) : 0);
        const uint8_t *sfa_src = p.sfa + ((int64_t)mt * p.kb_atoms) * SF_ATOM;
        const uint8_t *sfb0_src = p.sfb + ((int64_t)(rb0 >> 7) * p.kb_atoms) * SF_ATOM;
        const uint8_t *sfb1_src = p.sfb + ((int64_t)(rb1 >> 7) * p.kb_atoms) * SF_ATOM;
        for (int kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait(&c.empty[stage], phase ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.full[stage], bytes);
          const int kx = kt * (BK / 2);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &c.full[stage], kx, mt * BM);
          tma_load_2d(sB + stage * B_BYTES, &tmB, &c.full[stage], kx, rb0);
          bulk_load(sSFA + stage * SFA_BYTES, sfa_src + (int64_t)kt * SFA_BYTES, SFA_BYTES, &c.full[stage]);
          bulk_load(sSFB + stage * SFB_BYTES, sfb0_src + (int64_t)kt * SFB_HALF_BYTES, SFB_HALF_BYTES,
                    &c.full[stage]);
          if (second) {
            tma_load_2d(sB + stage * B_BYTES + B_HALF_BYTES, &tmB, &c.full[stage], kx, rb1);
            bulk_load(sSFB + stage * SFB_BYTES + SFB_HALF_BYTES, sfb1_src + (int64_t)kt * SFB_HALF_BYTES,
                      SFB_HALF_BYTES, &c.full[stage]);
          }
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // let every copy this thread issued land before the CTA can exit
      for (int s = 0; s < STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&c.full[s], (armed_phase >> s) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = make_idesc(BM, BN);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(&c.acc_empty, acc_phase ^ 1)) break;
        acc_phase ^= 1;
        tc_fence_after();
        for (int kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait(&c.full[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_BYTES);
          const uint32_t b_addr = smem_u32(sB + stage * B_BYTES);
          const uint32_t sfa_addr = smem_u32(sSFA + stage * SFA_BYTES);
          const uint32_t sfb_addr = smem_u32(sSFB + stage * SFB_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            tc_cp_32x128b_x4(tmem + SFA_COL + 4 * j, sdesc_plain_32x16B(sfa_addr + j * SF_ATOM));
            tc_cp_32x128b_x4(tmem + SFB_COL + 8 * j, sdesc_plain_32x16B(sfb_addr + j * SF_ATOM));
            tc_cp_32x128b_x4(tmem + SFB_COL + 8 * j + 4,
                             sdesc_plain_32x16B(sfb_addr + SFB_HALF_BYTES + j * SF_ATOM));
          }
          const uint64_t a_desc = sdesc_sw128_kmajor(a_addr);
          const uint64_t b_desc = sdesc_sw128_kmajor(b_addr);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // advance 64 FP4 = 32 bytes along K inside the swizzle atom (+2 in 16-byte units)
            mma_nvfp4(tmem + ACC_COL, a_desc + 2 * j, b_desc + 2 * j, idesc, tmem + SFA_COL + 4 * j,
                      tmem + SFB_COL + 8 * j, (kt | j) != 0);
          }
          tc_commit(&c.empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(&c.acc_full);
      }
      // wait for every tcgen05 operation this thread issued
      tc_commit(&c.drain);
      mbar_wait(&c.drain, 0);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;           // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2; // which 128 of the 256 accumulator columns
    uint32_t acc_phase = 0;
    const float gs_out = p.out_kind == OUT_NVFP4 ? __ldg(p.gs_out) : 1.0f;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      int mt, nt;
      tile_coords(p, tile, mt, nt);
      if (!mbar_wait(&c.acc_full, acc_phase)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[4][32];
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
      if (p.mode == MODE_SILU_MUL) {
        tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 64, v[0]);
        tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 64 + 32, v[1]);
        tmem_ld_32x32b_x32(lane_addr + ACC_COL + 128 + half * 64, v[2]);
        tmem_ld_32x32b_x32(lane_addr + ACC_COL + 128 + half * 64 + 32, v[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 128 + 32 * i, v[i]);
      }
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.acc_empty);

      const int row = mt * BM + 32 * q + lane;
      if (row >= p.M) {
        // padding rows of an NVFP4 output: their scale words are written as zero
        if (p.out_kind == OUT_NVFP4) {
          const int span = p.mode == MODE_SILU_MUL ? 64 : 128;
          const int cbeg = p.mode == MODE_SILU_MUL ? nt * 128 + half * 64 : nt * BN + half * 128;
          for (int cg = cbeg; cg < cbeg + span && cg < p.Nout; cg += 64)
            *reinterpret_cast<uint32_t *>(p.out_scales + scale_word_offset(row, cg / 64, p.out_kb_atoms)) = 0u;
        }
        continue;
      }
      if (p.mode == MODE_SILU_MUL) {
        // output columns [nt*128 + half*64, +64): gate = weight row n, up = row up_row0 + n
        const int col0 = nt * 128 + half * 64;
        const float ag = seg_alpha(c, p.nseg, col0);
        const float au = seg_alpha(c, p.nseg, p.up_row0 + col0);
        float h[64];
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float g = ag * __uint_as_float(v[i >> 5][i & 31]);
          const float u = au * __uint_as_float(v[2 + (i >> 5)][i & 31]);
          h[i] = (g / (1.0f + expf(-g))) * u;
        }
        if (p.out_kind == OUT_NVFP4) {
          store64_nvfp4(p, row, col0, h, gs_out);
        } else {
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = h[16 * b + i];
            store16(p, row, col0 + 16 * b, y);
          }
        }
      } else {
        const int col0 = nt * BN + half * 128;
#pragma unroll
        for (int hb = 0; hb < 2; ++hb) {  // two 64-column groups
          const int cg = col0 + 64 * hb;
          if (cg >= p.Nout) break;
          float y[64];
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            const float a = seg_alpha(c, p.nseg, cg + 16 * b);
#pragma unroll
            for (int i = 0; i < 16; ++i) y[16 * b + i] = a * __uint_as_float(v[2 * hb + (b >> 1)][(b & 1) * 16 + i]);
          }
          if (p.mode == MODE_GDN) {
#pragma unroll
            for (int i = 0; i < 64; ++i) {
              const int n = cg + i;
              if (n >= p.beta_begin && n < p.beta_begin + p.n_heads) {
                const float bt = sigmoid_f(y[i]);
                y[i] = bt;
                if (p.beta_out) p.beta_out[(int64_t)row * p.n_heads + (n - p.beta_begin)] = bt;
              } else if (n >= p.alpha_begin && n < p.alpha_begin + p.n_heads) {
                const int hh = n - p.alpha_begin;
                const float g = -expf(__ldg(p.A_log + hh)) * softplus_f(y[i] + __ldg(p.dt_bias + hh));
                y[i] = g;
                if (p.g_out) p.g_out[(int64_t)row * p.n_heads + hh] = g;
              }
            }
          }
          if (p.out_kind == OUT_NVFP4) {
            store64_nvfp4(p, row, cg, y, gs_out);
          } else {
#pragma unroll
            for (int b = 0; b < 4; ++b) {
              if (cg + 16 * b < p.Nout) {
                float yy[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) yy[i] = y[16 * b + i];
                store16(p, row, cg + 16 * b, yy);
              }
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

}  // namespace gemm
}  // namespace nvfp4
