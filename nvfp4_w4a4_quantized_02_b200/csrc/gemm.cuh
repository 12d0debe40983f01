// Block-scaled NVFP4 x NVFP4 GEMM for sm_100a (tcgen05, TMEM accumulators, TMA),
// with the fused-module per-segment global-scale correction and the epilogues of
// the W4A4 linear.
//
// Method: blog "27BハイブリッドLLMを4ビットで動かす", FAQ (W4A4 runs on 4-bit tensor
// cores), section 罠① (modules fused into one GEMM keep their own global scales:
// here every output column n is scaled by alpha = 1 / (gs_A * gs_W[seg(n)])),
// section 機構② (GDN gates beta = sigmoid(b), g = -exp(A_log) * softplus(a + dt_bias)).
//
// Two kernels share the tile shape per CTA (128 output rows x 256 output columns,
// K staged 256 FP4 elements = 128 bytes per row at a time) and the epilogue; a last
// N-tile narrower than 256 runs an MMA of its width rounded up to 32.  A third,
// decode_kernel (further down), serves up to 64 token rows with the weight as the
// MMA's 128-row side; splitk_epilogue_kernel reduces split-K partial sums.
//
// gemm_kernel (1 CTA per tile, used when M <= 128): tcgen05.mma.cta_group::1,
//   M = 128, N = 256; the CTA loads both 128-row halves of the B tile.
// gemm2_kernel (a cluster of 2 CTAs per 256 x 256 tile): tcgen05.mma.cta_group::2,
//   M = 256, N = 256, issued by the even CTA; each CTA loads its own 128 rows of A
//   and its own 128-row half of B, so per SM the shared-memory traffic per MMA is
//   halved against the 1-CTA kernel.  Every load signals the even CTA's stage
//   barrier; one tcgen05.commit signals the MMA's completion to the barriers of
//   both CTAs.  Each TMA load is a plain load of one CTA's own tile from this GPU's
//   memory.
//
// Roles (one persistent CTA per SM, 384 threads):
//   warp 0      TMA producer: code tiles (128-byte swizzle) and scale tiles (already
//               in the MMA's 128 x 4 atom layout) into a shared-memory ring.
//   warp 1      MMA issuer: 4 block-scaled MMAs (K = 64 each) per stage into the
//               TMEM accumulator, then frees the stage with tcgen05.commit.  It waits on
//               one barrier per stage, sf_ready: the copiers copy a stage's scales only
//               after its bytes landed, so their commit covers the operands too.  (A
//               second wait on the stage's load barrier cost ~190 cycles of the issuer's
//               per-stage loop: 2.47 -> 2.27 ms on the MLP block's gate|up GEMM.)
//   warps 2..9  epilogue: tcgen05.ld the 128 x 256 FP32 accumulator (each warp a
//               32-lane quadrant x 128 columns) into registers, hand TMEM back to the
//               MMA warp at once, then scale / activate / store from registers.  Its
//               warps share the sub-partitions (and their issue slots) with the
//               producer, copier and MMA threads, so its instruction count shows in
//               the mainloop: FP32 products and sums run two per packed instruction,
//               and a lane stores 32 bytes at once where the output rows allow it.
//   warps 10,11 scale copiers: per stage, 12 tcgen05.cp of the A and B scale atoms
//               (6 per warp) into that stage's TMEM scale columns, then
//               tcgen05.commit to the MMA issuer.  Issued from their own threads, the
//               copies of stage s+1 overlap the MMAs of stage s; issued in line with
//               the MMAs they ran in series with them and cost ~60 cycles each
//               (measured on the MLP block's gate|up GEMM, 1-CTA kernel: 3.26 ms in
//               line, 2.76 ms with one copier; CTA-pair kernel: 2.55 ms with one
//               copier, 2.50 ms with two).
// Output tiles are visited in groups of M-tiles (16, or 32 for a wide weight whose
// group of A rows fits a quarter of L2; chosen by the host) so that concurrently running
// CTAs share A and W tiles in L2.
#pragma once

#include "quant_math.cuh"

namespace nvfp4 {
namespace gemm {

constexpr int BM = 128;                  // output rows per CTA
constexpr int BN = 256;
constexpr int BK = 256;                  // FP4 elements per stage = 128 bytes per row
constexpr int A_BYTES = BM * BK / 2;     // 16 KB
constexpr int B_HALF_BYTES = 128 * BK / 2;
constexpr int SF_ATOM = 512;             // 128 rows x 4 scale bytes
constexpr int SFA_BYTES = 4 * SF_ATOM;   // 4 MMA k-steps
constexpr int SFB_HALF_BYTES = 4 * SF_ATOM;
constexpr int SFB_BYTES = 2 * SFB_HALF_BYTES;
constexpr int NUM_EPI_WARPS = 8;
constexpr int COPY_WARP = 2 + NUM_EPI_WARPS;  // first of the scale-copy warps
constexpr int NUM_COPY_WARPS = 2;  // copy_scales splits a stage's 12 atoms in two halves
constexpr int NUM_THREADS = 32 * (COPY_WARP + NUM_COPY_WARPS);
constexpr int GROUP_M = 16;        // M-tiles per raster group (Params::group_m), the default

// TMEM columns (allocation of 512 = the whole TMEM of the SM): the 256-column FP32
// accumulator, then one set of scale columns per shared-memory stage, so that the
// scales of stage s are rewritten only after the producer refilled stage s, which
// needs the MMAs that read them to have completed.
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t ACC_COL = 0;        // 256 FP32 columns
constexpr uint32_t SF_COL = 256;       // first scale set
constexpr uint32_t SF_SET_COLS = 48;   // SFA: 4 k-steps x 4 columns, then SFB: 4 k-steps x 8 columns
constexpr uint32_t SFB_OFF_COLS = 16;
__host__ __device__ constexpr uint32_t sfa_col(int stage) { return SF_COL + SF_SET_COLS * stage; }
__host__ __device__ constexpr uint32_t sfb_col(int stage) { return SF_COL + SF_SET_COLS * stage + SFB_OFF_COLS; }

// Shared-memory plan of a kernel whose CTA loads `b_halves` 128-row halves of B.
template <int kStages, int kBHalves>
struct SmemPlan {
  static constexpr int STAGES = kStages;
  static constexpr int B_BYTES = kBHalves * B_HALF_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int CTRL_BYTES = 1024;
  static constexpr int A_OFF = CTRL_BYTES;
  static constexpr int B_OFF = A_OFF + STAGES * A_BYTES;
  static constexpr int SFA_OFF = B_OFF + STAGES * B_BYTES;
  static constexpr int SFB_OFF = SFA_OFF + STAGES * SFA_BYTES;
  static constexpr int END = SFB_OFF + STAGES * SFB_BYTES;
  static constexpr int BYTES = END + 1024;  // slack to align the base to 1024
};
using Plan1 = SmemPlan<4, 2>;  // 1-CTA kernel: 54 KB per stage
using Plan2 = SmemPlan<5, 1>;  // 2-CTA kernel: 38 KB per stage
static_assert(Plan1::BYTES <= 227 * 1024 && Plan2::BYTES <= 227 * 1024, "shared memory");
static_assert(sfb_col(Plan1::STAGES - 1) + 32 <= TMEM_COLS && sfb_col(Plan2::STAGES - 1) + 32 <= TMEM_COLS,
              "TMEM columns");

enum Mode : int { MODE_NONE = 0, MODE_SILU_MUL = 1, MODE_GDN = 2 };
enum OutKind : int { OUT_BF16 = 0, OUT_F32 = 1, OUT_NVFP4 = 2 };

struct Segment {
  int n_begin, n_end;
  const float *gs_w;
};

struct Params {
  int M, N, K, Nout;
  int mode, out_kind;
  int tile_mode;                  // how B tiles are formed and read back: mode, or MODE_NONE for split-K
  int m_tiles, n_tiles, k_tiles;  // m_tiles counts tiles of BM * (CTAs per tile) rows
  int splits, kt_per_split;       // split-K: K tiles [s * kt_per_split, ...) form split s (1 split: whole K)
  float *partial;                 // split-K: FP32 partial sums [splits][M][N]; null otherwise
  int up_row0;              // SILU_MUL: first weight row of the `up` half
  int64_t kb_atoms;         // K / 64
  const uint8_t *sfa;       // swizzled scales of A
  const uint8_t *sfb;       // swizzled scales of W
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
  // decode kernel: token rows per MMA (32 or 64)
  int dn;
  // stalled-pipeline self-test only: the producer never loads this stage (counted over
  // the CTA's run); unused by every product instantiation
  int stall_stage;
  // the output's base and row stride are 32-byte aligned: stores of 32 bytes per lane
  int st32;
  // output tiles are visited in groups of group_m M-tiles (every N-tile of the group's
  // rows before the next group), so that concurrently running CTAs share A and W tiles
  // in L2; chosen by the host
  int group_m;
};

template <int STAGES>
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
  float inv_out[128];  // NVFP4 output: gs_out / e4m3(sf) for sf = 0..127 (0 for 0 and NaN)
  uint64_t sf_ready[STAGES];  // the stage's scales are in TMEM (tcgen05.commit of both copiers)
  uint64_t sf_drain[NUM_COPY_WARPS];
};
static_assert(sizeof(Ctrl<6>) <= 1024, "control block too large");

// Instruction descriptor of tcgen05.mma kind::mxf4nvf4: E2M1 A and B (format 1),
// UE4M3 scales, K-major operands, dense K = 64, scale ids 0; M and N of the MMA.
__host__ __device__ constexpr uint32_t make_idesc(int m, int n) {
  return (1u << 7) | (1u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void tile_coords(const Params &p, int tile, int &mt, int &nt) {
  const int per_group = p.group_m * p.n_tiles;
  const int g = tile / per_group;
  const int idx = tile - g * per_group;
  const int gm = min(p.group_m, p.m_tiles - g * p.group_m);
  mt = g * p.group_m + idx % gm;
  nt = idx / gm;
}

// MMA N of N-tile nt: BN, or for a narrower last tile its valid width rounded up to 32
// (the CTA pair then holds half of it per CTA, a multiple of 16 rows), so that the tail
// tile of, e.g., a 12352-row fused weight runs a quarter-width MMA instead of a full one.
// SILU_MUL tiles are always full (N % 256 == 0).
__device__ __forceinline__ int tile_mma_n(const Params &p, int nt) {
  const int w = p.N - nt * BN;
  return (p.tile_mode == MODE_SILU_MUL || w >= BN) ? BN : (w + 31) / 32 * 32;
}

// First weight rows of the two 128-row halves of the B tile of N-tile nt.
__device__ __forceinline__ void b_rows(const Params &p, int nt, int &rb0, int &rb1) {
  if (p.tile_mode == MODE_SILU_MUL) {
    rb0 = nt * 128;
    rb1 = p.up_row0 + nt * 128;
  } else {
    rb0 = nt * BN;
    rb1 = nt * BN + 128;
  }
}

// Work unit u of a launch: output tile u / splits, K tiles [k0, k1) of split u % splits.
__device__ __forceinline__ void unit_coords(const Params &p, int u, int &tile, int &split, int &k0, int &k1) {
  tile = u / p.splits;
  split = u - tile * p.splits;
  k0 = split * p.kt_per_split;
  k1 = min(p.k_tiles, k0 + p.kt_per_split);
}

template <int STAGES>
__device__ __forceinline__ float seg_alpha(const Ctrl<STAGES> &c, int nseg, int n) {
  float a = 0.0f;
  for (int s = 0; s < nseg; ++s)
    if (n >= c.seg_begin[s] && n < c.seg_end[s]) a = c.seg_alpha[s];
  return a;
}

// Alphas of the four 16-column blocks [n0, n0 + 64): one lookup when the group lies in
// one segment (segments are sorted, contiguous from column 0 and 16-aligned), else one
// per block.  The epilogue's instruction count matters: its warps share the issue slots
// of the producer, copier and MMA threads.
template <int STAGES>
__device__ __forceinline__ void seg_alpha4(const Ctrl<STAGES> &c, int nseg, int n0, float (&a)[4]) {
  int s = 0;
  while (s + 1 < nseg && n0 >= c.seg_end[s]) ++s;
  if (n0 >= c.seg_begin[s] && n0 + 64 <= c.seg_end[s]) {
#pragma unroll
    for (int b = 0; b < 4; ++b) a[b] = c.seg_alpha[s];
  } else {
#pragma unroll
    for (int b = 0; b < 4; ++b) a[b] = seg_alpha(c, nseg, n0 + 16 * b);
  }
}

// Gate and activation functions with the hardware approximations (relative error of
// order 1e-6: far below the BF16 store and the 1e-3 bar of the gates).  softplus uses
// the stable form max(x, 0) + log(1 + e^-|x|); 1 + e^-|x| lies in (1, 2], where the
// logarithm's absolute error stays below 1e-6.
__device__ __forceinline__ float sigmoid_f(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ float silu_mul_f(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }
// silu_mul_f of two elements: the same operations, the sum and the products packed.
__device__ __forceinline__ float2 silu_mul_f2(float2 g, float2 u) {
  const float2 d = add_f32x2(make_float2(1.0f, 1.0f), make_float2(__expf(-g.x), __expf(-g.y)));
  return mul_f32x2(make_float2(__fdividef(g.x, d.x), __fdividef(g.y, d.y)), u);
}
__device__ __forceinline__ float softplus_f(float x) { return fmaxf(x, 0.0f) + __logf(1.0f + __expf(-fabsf(x))); }

// Store 16 consecutive output values of one row.
__device__ __forceinline__ void store16(const Params &p, int row, int col, const float (&y)[16]) {
  if (!NVFP4_DCHECK(row >= 0 && row < p.M && col >= 0 && col % 16 == 0 && col + 16 <= p.Nout)) return;
  if (p.out_kind == OUT_BF16) {
    uint32_t w[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(y[2 * i], y[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t *>(&h);
    }
    __nv_bfloat16 *d = static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.ldo + col;
    if (p.st32) {
      st_global_v8(d, w);
    } else {
      uint4 *dst = reinterpret_cast<uint4 *>(d);
      dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
      dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
    }
  } else if (p.out_kind == OUT_F32) {
    float *d = static_cast<float *>(p.out) + (int64_t)row * p.ldo + col;
    if (p.st32) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        uint32_t w[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) w[i] = __float_as_uint(y[8 * h + i]);
        st_global_v8(d + 8 * h, w);
      }
    } else {
      float4 *dst = reinterpret_cast<float4 *>(d);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_float4(y[4 * i], y[4 * i + 1], y[4 * i + 2], y[4 * i + 3]);
    }
  }
}

// Re-quantise 64 consecutive outputs (one scale word) of one row: round to BF16,
// then the NVFP4 block quantiser with the output's global scale (gs_out / e4m3(sf)
// read from the CTA's table, the same FP32 division).
__device__ __forceinline__ void store64_nvfp4(const Params &p, const float *inv_out, int row, int col,
                                              const float (&y)[64], float gs_out) {
  if (!NVFP4_DCHECK(row >= 0 && row < p.M && col >= 0 && col % 64 == 0 && col + 64 <= p.Nout)) return;
  uint32_t codes[8];
  uint32_t sfword = 0;
#pragma unroll
  for (int b = 0; b < 4; ++b) {
    float x[16];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i += 2) {  // round to BF16 two at a time (RNE, as one by one)
      const __nv_bfloat162 hb = __floats2bfloat162_rn(y[16 * b + i], y[16 * b + i + 1]);
      x[i] = __low2float(hb);
      x[i + 1] = __high2float(hb);
      amax = fmaxf(amax, fmaxf(fabsf(x[i]), fabsf(x[i + 1])));
    }
    const uint32_t sf = block_scale_byte(amax, gs_out);
    const float inv = inv_out[sf & 127];
    codes[2 * b] = encode8(x, inv);
    codes[2 * b + 1] = encode8(x + 8, inv);
    sfword |= sf << (8 * b);
  }
  uint8_t *d = static_cast<uint8_t *>(p.out) + (int64_t)row * (p.Nout / 2) + col / 2;
  if (p.st32) {
    st_global_v8(d, codes);
  } else {
    uint4 *dst = reinterpret_cast<uint4 *>(d);
    dst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
    dst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
  }
  *reinterpret_cast<uint32_t *>(p.out_scales + scale_word_offset(row, col / 64, p.out_kb_atoms)) = sfword;
}

// GDN gates of the W outputs starting at column cg of one row, in place in the
// caller's registers, for the columns that fall in the beta or alpha head blocks
// (blocks are disjoint; only the N-tile holding them gets here).  Unrolled over the
// columns so that the exp / log / division chains of neighbouring columns overlap.
template <int W>
__device__ __forceinline__ void gdn_gates(const Params &p, int row, int cg, float (&y)[W]) {
#pragma unroll
  for (int i = 0; i < W; ++i) {
    const int n = cg + i;
    if (n >= p.beta_begin && n < p.beta_begin + p.n_heads) {
      y[i] = sigmoid_f(y[i]);
      if (p.beta_out && NVFP4_DCHECK(row >= 0 && row < p.M))
        p.beta_out[(int64_t)row * p.n_heads + (n - p.beta_begin)] = y[i];
    } else if (n >= p.alpha_begin && n < p.alpha_begin + p.n_heads) {
      const int hh = n - p.alpha_begin;
      y[i] = -__expf(__ldg(p.A_log + hh)) * softplus_f(y[i] + __ldg(p.dt_bias + hh));
      if (p.g_out && NVFP4_DCHECK(row >= 0 && row < p.M)) p.g_out[(int64_t)row * p.n_heads + hh] = y[i];
    }
  }
}

// Whether columns [cg, cg + w) touch a GDN head block.
__device__ __forceinline__ bool touches_gates(const Params &p, int cg, int w) {
  return p.mode == MODE_GDN && ((cg < p.beta_begin + p.n_heads && cg + w > p.beta_begin) ||
                                (cg < p.alpha_begin + p.n_heads && cg + w > p.alpha_begin));
}

// TMEM -> registers for one epilogue warp: 32 lanes of quadrant q, 128 columns
// (SILU_MUL: 64 gate columns and the matching 64 up columns).
__device__ __forceinline__ void epilogue_load(const Params &p, uint32_t tmem, int q, int half,
                                              uint32_t (&v)[4][32]) {
  const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
  if (p.tile_mode == MODE_SILU_MUL) {
    tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 64, v[0]);
    tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 64 + 32, v[1]);
    tmem_ld_32x32b_x32(lane_addr + ACC_COL + 128 + half * 64, v[2]);
    tmem_ld_32x32b_x32(lane_addr + ACC_COL + 128 + half * 64 + 32, v[3]);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) tmem_ld_32x32b_x32(lane_addr + ACC_COL + half * 128 + 32 * i, v[i]);
  }
  tmem_ld_wait();
}

// Scale / activate / store the accumulator values of one output row held by this
// thread (columns as loaded by epilogue_load) for N-tile nt.
template <int STAGES>
__device__ __forceinline__ void epilogue_row(const Params &p, const Ctrl<STAGES> &c, const uint32_t (&v)[4][32],
                                             int row, int nt, int half, float gs_out) {
  if (row >= p.M) {
    // padding rows of an NVFP4 output: their scale words are written as zero
    if (p.out_kind == OUT_NVFP4) {
      const int span = p.mode == MODE_SILU_MUL ? 64 : 128;
      const int cbeg = p.mode == MODE_SILU_MUL ? nt * 128 + half * 64 : nt * BN + half * 128;
      const int rows_pad = (p.M + 127) / 128 * 128;
      if (row < rows_pad)
        for (int cg = cbeg; cg < cbeg + span && cg < p.Nout; cg += 64)
          if (NVFP4_DCHECK(cg % 64 == 0 && cg / 64 < p.out_kb_atoms))
            *reinterpret_cast<uint32_t *>(p.out_scales + scale_word_offset(row, cg / 64, p.out_kb_atoms)) = 0u;
    }
    return;
  }
  if (p.mode == MODE_SILU_MUL) {
    // output columns [nt*128 + half*64, +64): gate = weight row n, up = row up_row0 + n
    const int col0 = nt * 128 + half * 64;
    float h[64];
    float ag[4], au[4];
    seg_alpha4(c, p.nseg, col0, ag);
    seg_alpha4(c, p.nseg, p.up_row0 + col0, au);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
#pragma unroll
      for (int i = 16 * b; i < 16 * b + 16; i += 2) {
        const float2 g = mul_f32x2(make_float2(ag[b], ag[b]), make_float2(__uint_as_float(v[i >> 5][i & 31]),
                                                                          __uint_as_float(v[i >> 5][(i & 31) + 1])));
        const float2 u = mul_f32x2(make_float2(au[b], au[b]),
                                   make_float2(__uint_as_float(v[2 + (i >> 5)][i & 31]),
                                               __uint_as_float(v[2 + (i >> 5)][(i & 31) + 1])));
        const float2 hh = silu_mul_f2(g, u);
        h[i] = hh.x;
        h[i + 1] = hh.y;
      }
    }
    if (p.out_kind == OUT_NVFP4) {
      store64_nvfp4(p, c.inv_out, row, col0, h, gs_out);
    } else {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        float y[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) y[i] = h[16 * b + i];
        store16(p, row, col0 + 16 * b, y);
      }
    }
    return;
  }
  const int col0 = nt * BN + half * 128;
#pragma unroll
  for (int hb = 0; hb < 2; ++hb) {  // two 64-column groups
    const int cg = col0 + 64 * hb;
    if (cg >= p.Nout) break;
    float y[64];
    float a[4];
    seg_alpha4(c, p.nseg, cg, a);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const uint32_t *src = &v[2 * hb + (b >> 1)][(b & 1) * 16 + i];
        const float2 r = mul_f32x2(make_float2(a[b], a[b]), make_float2(__uint_as_float(src[0]), __uint_as_float(src[1])));
        y[16 * b + i] = r.x;
        y[16 * b + i + 1] = r.y;
      }
    }
    if (touches_gates(p, cg, 64)) gdn_gates<64>(p, row, cg, y);
    if (p.out_kind == OUT_NVFP4) {
      store64_nvfp4(p, c.inv_out, row, cg, y, gs_out);
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

// Split-K: the raw FP32 sums of 128 consecutive columns of one row, for split `split`.
__device__ __forceinline__ void store_partial(const Params &p, const uint32_t (&v)[4][32], int split, int row,
                                              int col0) {
  if (row >= p.M) return;
  if (!NVFP4_DCHECK(split >= 0 && split < p.splits && col0 >= 0 && col0 % 16 == 0)) return;
  float *dst = p.partial + ((int64_t)split * p.M + row) * p.N + col0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int c4 = 0; c4 < 8; ++c4) {
      if (col0 + 32 * i + 4 * c4 < p.N)  // N % 16 == 0: a vector is all in or all out
        *reinterpret_cast<float4 *>(dst + 32 * i + 4 * c4) =
            make_float4(__uint_as_float(v[i][4 * c4]), __uint_as_float(v[i][4 * c4 + 1]),
                        __uint_as_float(v[i][4 * c4 + 2]), __uint_as_float(v[i][4 * c4 + 3]));
    }
  }
}

// Barrier over the epilogue warps only (warps 2 .. 2 + NUM_EPI_WARPS - 1).
__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * NUM_EPI_WARPS) : "memory");
}

// Per-CTA epilogue tables: the segments' alphas and, for an NVFP4 output, the
// 128 possible values of gs_out / e4m3(sf).  Written by threads 64 .. 255, all of
// them epilogue threads of the GEMM kernels.
template <int STAGES>
__device__ __forceinline__ void load_segments(const Params &p, Ctrl<STAGES> &c) {
  if (threadIdx.x >= 64 && threadIdx.x < 64 + p.nseg) {
    const int s = threadIdx.x - 64;
    c.seg_begin[s] = p.seg[s].n_begin;
    c.seg_end[s] = p.seg[s].n_end;
    c.seg_alpha[s] = __frcp_rn(__fmul_rn(__ldg(p.gs_a), __ldg(p.seg[s].gs_w)));
  }
  if (p.out_kind == OUT_NVFP4 && threadIdx.x >= 128 && threadIdx.x < 256) {
    const int sf = threadIdx.x - 128;
    c.inv_out[sf] = (sf == 0 || sf == 127) ? 0.0f : __fdiv_rn(__ldg(p.gs_out), e4m3_to_f32(sf));
  }
}

// Scale copier `part` (one thread of warp COPY_WARP + part): for each stage of the
// CTA's run, once the stage's bytes landed, copy half of its 12 scale atoms into the
// stage's TMEM scale set and commit to sf_ready[stage] (which waits for both
// copiers).  Part 0: A's 4 k-steps and B's first half for k-steps 0, 1; part 1: B's
// first half for k-steps 2, 3 and B's second half.  Set s is rewritten only after
// full[s] completed again, i.e. after the producer refilled stage s, which waited
// for the MMAs that read set s.
template <bool kPair>
__device__ __forceinline__ void cp_scale_atom(uint32_t taddr, uint32_t saddr) {
  if constexpr (kPair) {  // each CTA's atom goes to its own TMEM (same addresses in both)
    tc_cp_32x128b_x4_cg2(taddr, sdesc_plain_32x16B(saddr));
  } else {
    tc_cp_32x128b_x4(taddr, sdesc_plain_32x16B(saddr));
  }
}

template <int STAGES, bool kPair, uint64_t kWait = kMaxWaitNs>
__device__ __forceinline__ void copy_scales(Ctrl<STAGES> &c, uint32_t tmem, const uint8_t *sSFA,
                                            const uint8_t *sSFB, int total, int part) {
  int stage = 0;
  uint32_t phase = 0;
  for (int g = 0; g < total; ++g) {
    if (!mbar_wait<kWait>(&c.full[stage], phase)) break;
    tc_fence_after();
    const uint32_t sfa = smem_u32(sSFA + stage * SFA_BYTES);
    const uint32_t sfb = smem_u32(sSFB + stage * SFB_BYTES);
    if (part == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j) cp_scale_atom<kPair>(tmem + sfa_col(stage) + 4 * j, sfa + j * SF_ATOM);
#pragma unroll
      for (int j = 0; j < 2; ++j) cp_scale_atom<kPair>(tmem + sfb_col(stage) + 8 * j, sfb + j * SF_ATOM);
    } else {
#pragma unroll
      for (int j = 2; j < 4; ++j) cp_scale_atom<kPair>(tmem + sfb_col(stage) + 8 * j, sfb + j * SF_ATOM);
#pragma unroll
      for (int j = 0; j < 4; ++j)
        cp_scale_atom<kPair>(tmem + sfb_col(stage) + 8 * j + 4, sfb + SFB_HALF_BYTES + j * SF_ATOM);
    }
    if constexpr (kPair) {
      tc_commit_cg2(&c.sf_ready[stage]);
    } else {
      tc_commit(&c.sf_ready[stage]);
    }
    if (++stage == STAGES) { stage = 0; phase ^= 1; }
  }
  // wait for every copy this thread issued
  uint64_t *drain = &c.sf_drain[part];
  if constexpr (kPair) {
    tc_commit_cg2(drain);
  } else {
    tc_commit(drain);
  }
  mbar_wait<kWait>(drain, 0);
}

template <int STAGES>
__device__ __forceinline__ void init_barriers(Ctrl<STAGES> &c, uint32_t acc_empty_count) {
  for (int s = 0; s < STAGES; ++s) {
    mbar_init(&c.full[s], 1);
    mbar_init(&c.empty[s], 1);
    mbar_init(&c.sf_ready[s], NUM_COPY_WARPS);
  }
  mbar_init(&c.acc_full, 1);
  mbar_init(&c.acc_empty, acc_empty_count);
  mbar_init(&c.drain, 1);
  for (int i = 0; i < NUM_COPY_WARPS; ++i) mbar_init(&c.sf_drain[i], 1);
  fence_barrier_init();
}

// ============================================================ 1-CTA kernel
// kPartial: the split-K form, whose epilogue only stores the raw FP32 sums (the
// epilogue of the linear runs in splitk_epilogue_kernel).  A separate instantiation
// keeps its code small: a decode-size launch spends much of its few microseconds
// fetching instructions.
// kStallTest: the failure-detection self-test.  The producer skips stage
// p.stall_stage (no expected bytes, no loads), so the consumers of that stage wait for
// a phase that never completes; every wait gives up after kTestWaitNs (1 ms).  Each
// role then records NVFP4_ERR_DEVICE_TIMEOUT, waits for the work it already issued
// and leaves; TMEM is freed and the kernel returns.
template <bool kPartial, bool kStallTest = false>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ Params p) {
  using P = Plan1;
  constexpr int STAGES = P::STAGES;
  constexpr uint64_t kWait = kStallTest ? kTestWaitNs : kMaxWaitNs;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl<STAGES> &c = *reinterpret_cast<Ctrl<STAGES> *>(smem);
  uint8_t *sA = smem + P::A_OFF;
  uint8_t *sB = smem + P::B_OFF;
  uint8_t *sSFA = smem + P::SFA_OFF;
  uint8_t *sSFB = smem + P::SFB_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    init_barriers(c, NUM_EPI_WARPS);
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  grid_dep_wait();  // operands, scales and global scales may come from the previous kernel
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int num_units = p.m_tiles * p.n_tiles * p.splits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;  // per-stage bit masks
      bool ok = true;
      int g = 0;  // stages issued so far (the self-test's stall counter)
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        int tile, split, k0, k1, mt, nt, rb0, rb1;
        unit_coords(p, u, tile, split, k0, k1);
        tile_coords(p, tile, mt, nt);
        b_rows(p, nt, rb0, rb1);
        const bool second = rb1 < p.N;  // any valid row in the second half
        const uint32_t bytes = A_BYTES + B_HALF_BYTES + SFA_BYTES + SFB_HALF_BYTES +
                               (second ? (B_HALF_BYTES + SFB_HALF_BYTES) : 0);
        const uint8_t *sfa_src = p.sfa + ((int64_t)mt * p.kb_atoms) * SF_ATOM;
        const uint8_t *sfb0_src = p.sfb + ((int64_t)(rb0 >> 7) * p.kb_atoms) * SF_ATOM;
        const uint8_t *sfb1_src = p.sfb + ((int64_t)(rb1 >> 7) * p.kb_atoms) * SF_ATOM;
        for (int kt = k0; kt < k1; ++kt, ++g) {
          if (!mbar_wait<kWait>(&c.empty[stage], phase ^ 1)) { ok = false; break; }
          if constexpr (kStallTest) {
            if (g == p.stall_stage) {  // never filled: its full barrier stays in this phase
              if (++stage == STAGES) { stage = 0; phase ^= 1; }
              continue;
            }
          }
          mbar_arrive_expect_tx(&c.full[stage], bytes);
          const int kx = kt * (BK / 2);
          tma_load_2d(sA + stage * A_BYTES, &tmA, &c.full[stage], kx, mt * BM);
          tma_load_2d(sB + stage * P::B_BYTES, &tmB, &c.full[stage], kx, rb0);
          bulk_load(sSFA + stage * SFA_BYTES, sfa_src + (int64_t)kt * SFA_BYTES, SFA_BYTES, &c.full[stage]);
          bulk_load(sSFB + stage * SFB_BYTES, sfb0_src + (int64_t)kt * SFB_HALF_BYTES, SFB_HALF_BYTES,
                    &c.full[stage]);
          if (second) {
            tma_load_2d(sB + stage * P::B_BYTES + B_HALF_BYTES, &tmB, &c.full[stage], kx, rb1);
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
        if (armed & (1u << s)) mbar_wait<kWait>(&c.full[s], (armed_phase >> s) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        int tile, split, k0, k1, mt, nt;
        unit_coords(p, u, tile, split, k0, k1);
        tile_coords(p, tile, mt, nt);
        const uint32_t idesc = make_idesc(BM, tile_mma_n(p, nt));  // B rows 0.. of the tile
        if (!mbar_wait<kWait>(&c.acc_empty, acc_phase ^ 1)) break;
        acc_phase ^= 1;
        tc_fence_after();
        for (int kt = k0; kt < k1; ++kt) {
          // sf_ready completes only after a copier saw full[stage] (the stage's bytes
          // landed) and its copies of the stage's scales completed: one wait covers both.
          if (!mbar_wait<kWait>(&c.sf_ready[stage], phase)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a_desc = sdesc_sw128_kmajor(smem_u32(sA + stage * A_BYTES));
          const uint64_t b_desc = sdesc_sw128_kmajor(smem_u32(sB + stage * P::B_BYTES));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // advance 64 FP4 = 32 bytes along K inside the swizzle atom (+2 in 16-byte units)
            mma_nvfp4(tmem + ACC_COL, a_desc + 2 * j, b_desc + 2 * j, idesc, tmem + sfa_col(stage) + 4 * j,
                      tmem + sfb_col(stage) + 8 * j, (kt != k0) | (j != 0));
          }
          tc_commit(&c.empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(&c.acc_full);
      }
      // wait for every tcgen05 operation this thread issued
      tc_commit(&c.drain);
      mbar_wait<kWait>(&c.drain, 0);
    }
  } else if (warp >= COPY_WARP) {
    if (lane == 0) {
      int total = 0;  // stages this CTA runs through
      for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
        int tile, split, k0, k1;
        unit_coords(p, u, tile, split, k0, k1);
        total += k1 - k0;
      }
      copy_scales<STAGES, false, kWait>(c, tmem, sSFA, sSFB, total, warp - COPY_WARP);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // The epilogue tables (global scales of the segments and of the output) are read
    // here, off the prologue: the first loads need not wait for them.  (The split-K
    // form stores raw sums and needs none.)
    if constexpr (!kPartial) {
      load_segments(p, c);
      epilogue_bar();
    }
    const int q = warp & 3;           // TMEM lane quadrant this warp may access
    const int half = (warp - 2) >> 2; // which 128 of the 256 accumulator columns
    uint32_t acc_phase = 0;
    const float gs_out = !kPartial && p.out_kind == OUT_NVFP4 ? __ldg(p.gs_out) : 1.0f;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
      int tile, split, k0, k1, mt, nt;
      unit_coords(p, u, tile, split, k0, k1);
      tile_coords(p, tile, mt, nt);
      if (!mbar_wait<kWait>(&c.acc_full, acc_phase)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[4][32];
      epilogue_load(p, tmem, q, half, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.acc_empty);
      const int row = mt * BM + 32 * q + lane;
      if constexpr (kPartial) {
        store_partial(p, v, split, row, nt * BN + half * 128);
      } else {
        epilogue_row(p, c, v, row, nt, half, gs_out);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ============================================================ 2-CTA kernel
// Bytes one stage brings into ONE CTA (A rows, its B half, SFA, both SFB halves).
constexpr uint32_t STAGE2_TX = A_BYTES + B_HALF_BYTES + SFA_BYTES + SFB_BYTES;

__global__ void __launch_bounds__(NUM_THREADS, 1)
    gemm2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                 const __grid_constant__ Params p) {
  using P = Plan2;
  constexpr int STAGES = P::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Ctrl<STAGES> &c = *reinterpret_cast<Ctrl<STAGES> *>(smem);
  uint8_t *sA = smem + P::A_OFF;
  uint8_t *sB = smem + P::B_OFF;
  uint8_t *sSFA = smem + P::SFA_OFF;
  uint8_t *sSFB = smem + P::SFB_OFF;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();  // 0: issues the MMAs and scale copies; 1: its peer
  const int cid = blockIdx.x >> 1;
  const int nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    init_barriers(c, 2 * NUM_EPI_WARPS);
    prefetch_tensormap(&tmA);
    prefetch_tensormap(&tmB);
    prefetch_tensormap(&tmSFA);
    prefetch_tensormap(&tmSFB);
  }
  if (warp == 1) {
    tmem_alloc_cg2(&c.tmem_base, TMEM_COLS);
    tmem_relinquish_cg2();
  }
  grid_dep_wait();  // operands, scales and global scales may come from the previous kernel
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int num_tiles = p.m_tiles * p.n_tiles;
  const int my_tiles = num_tiles > cid ? (num_tiles - 1 - cid) / nclusters + 1 : 0;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;  // per-stage bit masks (rank 0 only)
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters) {
        int mt, nt, rb0, rb1;
        tile_coords(p, tile, mt, nt);
        b_rows(p, nt, rb0, rb1);
        const int a_row = mt * (2 * BM) + (int)rank * BM;
        const int n_mma = tile_mma_n(p, nt);  // the CTA pair splits the MMA's N rows of B in halves
        const int b_row = rank == 0 ? rb0 : (n_mma == BN ? rb1 : rb0 + n_mma / 2);
        for (int kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait(&c.empty[stage], phase ^ 1)) { ok = false; break; }
          if (rank == 0) mbar_arrive_expect_tx(&c.full[stage], 2 * STAGE2_TX);
          const uint32_t bar = mapa_shared(smem_u32(&c.full[stage]), 0);
          const int kx = kt * (BK / 2);
          const int ksf = kt * (SFA_BYTES / 8);  // scale tensor maps count 8-byte elements
          tma_load_2d_cg2(sA + stage * A_BYTES, &tmA, bar, kx, a_row);
          tma_load_2d_cg2(sB + stage * P::B_BYTES, &tmB, bar, kx, b_row);
          tma_load_2d_cg2(sSFA + stage * SFA_BYTES, &tmSFA, bar, ksf, a_row >> 7);
          tma_load_2d_cg2(sSFB + stage * SFB_BYTES, &tmSFB, bar, ksf, rb0 >> 7);
          tma_load_2d_cg2(sSFB + stage * SFB_BYTES + SFB_HALF_BYTES, &tmSFB, bar, ksf, rb1 >> 7);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // the even CTA's barriers count both CTAs' bytes: let them all land before exit
      if (rank == 0)
        for (int s = 0; s < STAGES; ++s)
          if (armed & (1u << s)) mbar_wait(&c.full[s], (armed_phase >> s) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && rank == 0) {
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = cid; tile < num_tiles && ok; tile += nclusters) {
        int mt, nt;
        tile_coords(p, tile, mt, nt);
        const uint32_t idesc = make_idesc(2 * BM, tile_mma_n(p, nt));
        if (!mbar_wait_cluster(&c.acc_empty, acc_phase ^ 1)) break;
        acc_phase ^= 1;
        tc_fence_after();
        for (int kt = 0; kt < p.k_tiles; ++kt) {
          if (!mbar_wait(&c.sf_ready[stage], phase)) { ok = false; break; }  // implies full[stage]
          tc_fence_after();
          const uint64_t a_desc = sdesc_sw128_kmajor(smem_u32(sA + stage * A_BYTES));
          const uint64_t b_desc = sdesc_sw128_kmajor(smem_u32(sB + stage * P::B_BYTES));
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            mma_nvfp4_cg2(tmem + ACC_COL, a_desc + 2 * j, b_desc + 2 * j, idesc, tmem + sfa_col(stage) + 4 * j,
                          tmem + sfb_col(stage) + 8 * j, (kt | j) != 0);
          }
          tc_commit_mc_cg2(&c.empty[stage], 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit_mc_cg2(&c.acc_full, 0x3);
      }
      // wait for every tcgen05 operation this thread issued
      tc_commit_cg2(&c.drain);
      mbar_wait(&c.drain, 0);
    }
  } else if (warp >= COPY_WARP) {
    if (lane == 0 && rank == 0)
      copy_scales<STAGES, true>(c, tmem, sSFA, sSFB, my_tiles * p.k_tiles, warp - COPY_WARP);
  } else {
    // ----------------------------------------------------------- epilogue
    load_segments(p, c);  // off the prologue, as in gemm_kernel
    epilogue_bar();
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    uint32_t acc_phase = 0;
    const float gs_out = p.out_kind == OUT_NVFP4 ? __ldg(p.gs_out) : 1.0f;
    const uint32_t acc_empty0 = mapa_shared(smem_u32(&c.acc_empty), 0);
    for (int tile = cid; tile < num_tiles; tile += nclusters) {
      int mt, nt;
      tile_coords(p, tile, mt, nt);
      if (!mbar_wait(&c.acc_full, acc_phase)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[4][32];
      epilogue_load(p, tmem, q, half, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0);
      epilogue_row(p, c, v, mt * (2 * BM) + (int)rank * BM + 32 * q + lane, nt, half, gs_out);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the other may still signal it
  tc_fence_after();
  if (warp == 1) tmem_dealloc_cg2(tmem, TMEM_COLS);
}

// ======================================================== decode kernel
// The decode regime (a few token rows against a large weight) with the operands'
// roles swapped: 128 weight rows are the MMA's M and the DN (32 or 64) token rows its
// N, so no MMA row is padding and a stage carries a 16 KB weight tile, a small token
// tile and two scale sets of 4 atoms each (8 copies, against 12 for a 128 x 256 tile).
// Seven stages stay in flight to keep HBM busy while the weights stream through.
// Work units are (128-row weight tile, K range); each writes its raw FP32 sums to
// partial[split][m][n] (n = weight row = output column), and splitk_epilogue_kernel
// applies the epilogue of the linear, as for the split-K form of gemm_kernel.
// Accumulator: TMEM lane = weight row, column = token.  B's scales (the tokens'): row
// 32c + i at lane 32q + i, column base + c, c < DN / 32, all inside one atom copy.
constexpr int DEC_BM = 128;              // weight rows per tile (MMA M)
constexpr int DEC_DN_MAX = 64;           // token rows per MMA (N)
constexpr int DEC_STAGES = 7;
constexpr int DEC_W_BYTES = DEC_BM * BK / 2;       // 16 KB
constexpr int DEC_X_BYTES = DEC_DN_MAX * BK / 2;   // 8 KB
constexpr int DEC_SF_BYTES = 4 * SF_ATOM;          // 2 KB: 4 k-steps of one 128-row group
constexpr int DEC_THREADS = 256;                   // producer, MMA, 4 epilogue, 2 copier warps
constexpr int DEC_COPY_WARP = 6;
constexpr uint32_t DEC_ACC_COL = 0;                // DEC_DN_MAX FP32 columns
constexpr uint32_t DEC_SF_COL = DEC_DN_MAX;        // then one 32-column scale set per stage
__host__ __device__ constexpr uint32_t dec_sfw_col(int stage) { return DEC_SF_COL + 32 * stage; }
__host__ __device__ constexpr uint32_t dec_sfx_col(int stage) { return DEC_SF_COL + 32 * stage + 16; }
static_assert(dec_sfx_col(DEC_STAGES - 1) + 16 <= TMEM_COLS, "TMEM columns");

struct PlanD {
  static constexpr int CTRL_BYTES = 1024;
  static constexpr int W_OFF = CTRL_BYTES;
  static constexpr int X_OFF = W_OFF + DEC_STAGES * DEC_W_BYTES;
  static constexpr int SFW_OFF = X_OFF + DEC_STAGES * DEC_X_BYTES;
  static constexpr int SFX_OFF = SFW_OFF + DEC_STAGES * DEC_SF_BYTES;
  static constexpr int END = SFX_OFF + DEC_STAGES * DEC_SF_BYTES;
  static constexpr int BYTES = END + 1024;  // slack to align the base to 1024
};
static_assert(PlanD::BYTES <= 227 * 1024, "shared memory");

struct CtrlD {
  uint64_t full[DEC_STAGES];
  uint64_t empty[DEC_STAGES];
  uint64_t sf_ready[DEC_STAGES];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain;
  uint64_t sf_drain[2];
  uint32_t tmem_base;
};
static_assert(sizeof(CtrlD) <= PlanD::CTRL_BYTES, "control block too large");

// Unsplit decode linear, epilogue applied in place of the FP32 partials (no reduction
// kernel): output column n of every token row, y = alpha_seg(n) * acc, the GDN gate of
// column n where it is one, stored as BF16 or FP32 (the launch takes this path only
// for one split, epilogue none or GDN gates, and a BF16 / FP32 output).  The same
// arithmetic as splitk_epilogue_kernel on a single split, element by element.
__device__ __forceinline__ void decode_direct_epilogue(const Params &p, int n, const uint32_t (&v)[2][32]) {
  float alpha = 0.0f;
  for (int s = 0; s < p.nseg; ++s)
    if (n >= p.seg[s].n_begin && n < p.seg[s].n_end)
      alpha = __frcp_rn(__fmul_rn(__ldg(p.gs_a), __ldg(p.seg[s].gs_w)));
  int gate = 0, hh = 0;  // 1: beta column (sigmoid), 2: alpha column (decay)
  float la = 0.0f, db = 0.0f;
  if (p.mode == MODE_GDN) {
    if (n >= p.beta_begin && n < p.beta_begin + p.n_heads) {
      gate = 1;
      hh = n - p.beta_begin;
    } else if (n >= p.alpha_begin && n < p.alpha_begin + p.n_heads) {
      gate = 2;
      hh = n - p.alpha_begin;
      la = -__expf(__ldg(p.A_log + hh));
      db = __ldg(p.dt_bias + hh);
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (h == 1 && p.dn <= 32) break;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int m = 32 * h + i;
      if (m >= p.M) break;
      float y = alpha * __uint_as_float(v[h][i]);
      if (gate == 1) {
        y = sigmoid_f(y);
        if (p.beta_out) p.beta_out[(int64_t)m * p.n_heads + hh] = y;
      } else if (gate == 2) {
        y = la * softplus_f(y + db);
        if (p.g_out) p.g_out[(int64_t)m * p.n_heads + hh] = y;
      }
      if (!NVFP4_DCHECK(n >= 0 && n < p.Nout && m < p.M)) continue;
      if (p.out_kind == OUT_BF16)
        static_cast<__nv_bfloat16 *>(p.out)[(int64_t)m * p.ldo + n] = __float2bfloat16_rn(y);
      else
        static_cast<float *>(p.out)[(int64_t)m * p.ldo + n] = y;
    }
  }
}

// tmW: weight codes, boxes of 128 rows; tmX: token codes, boxes of p.dn rows.
// p.sfb: the weight's scales, p.sfa: the tokens' (one 128-row group: p.M <= 64).
__global__ void __launch_bounds__(DEC_THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                  const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  CtrlD &c = *reinterpret_cast<CtrlD *>(smem);
  uint8_t *sW = smem + PlanD::W_OFF;
  uint8_t *sX = smem + PlanD::X_OFF;
  uint8_t *sSFW = smem + PlanD::SFW_OFF;
  uint8_t *sSFX = smem + PlanD::SFX_OFF;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < DEC_STAGES; ++s) {
      mbar_init(&c.full[s], 1);
      mbar_init(&c.empty[s], 1);
      mbar_init(&c.sf_ready[s], 2);
    }
    mbar_init(&c.acc_full, 1);
    mbar_init(&c.acc_empty, 4);
    mbar_init(&c.drain, 1);
    mbar_init(&c.sf_drain[0], 1);
    mbar_init(&c.sf_drain[1], 1);
    fence_barrier_init();
    prefetch_tensormap(&tmW);
    prefetch_tensormap(&tmX);
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  grid_dep_wait();  // the tokens' codes and scales may come from the previous kernel
  grid_dep_launch();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  const int num_units = p.n_tiles * p.splits;
  const uint32_t x_bytes = static_cast<uint32_t>(p.dn) * (BK / 2);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t armed = 0, armed_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        int nt, split, k0, k1;
        unit_coords(p, u, nt, split, k0, k1);
        const uint8_t *sfw_src = p.sfb + ((int64_t)nt * p.kb_atoms) * SF_ATOM;
        for (int kt = k0; kt < k1; ++kt) {
          if (!mbar_wait(&c.empty[stage], phase ^ 1)) { ok = false; break; }
          mbar_arrive_expect_tx(&c.full[stage], DEC_W_BYTES + x_bytes + 2 * DEC_SF_BYTES);
          const int kx = kt * (BK / 2);
          tma_load_2d(sW + stage * DEC_W_BYTES, &tmW, &c.full[stage], kx, nt * DEC_BM);
          tma_load_2d(sX + stage * DEC_X_BYTES, &tmX, &c.full[stage], kx, 0);
          bulk_load(sSFW + stage * DEC_SF_BYTES, sfw_src + (int64_t)kt * DEC_SF_BYTES, DEC_SF_BYTES, &c.full[stage]);
          bulk_load(sSFX + stage * DEC_SF_BYTES, p.sfa + (int64_t)kt * DEC_SF_BYTES, DEC_SF_BYTES, &c.full[stage]);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == DEC_STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // let every copy this thread issued land before the CTA can exit
      for (int s = 0; s < DEC_STAGES; ++s)
        if (armed & (1u << s)) mbar_wait(&c.full[s], (armed_phase >> s) & 1);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t idesc = make_idesc(DEC_BM, p.dn);
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < num_units && ok; u += gridDim.x) {
        int nt, split, k0, k1;
        unit_coords(p, u, nt, split, k0, k1);
        if (!mbar_wait(&c.acc_empty, acc_phase ^ 1)) break;
        acc_phase ^= 1;
        tc_fence_after();
        for (int kt = k0; kt < k1; ++kt) {
          if (!mbar_wait(&c.sf_ready[stage], phase)) { ok = false; break; }  // implies full[stage]
          tc_fence_after();
          const uint64_t w_desc = sdesc_sw128_kmajor(smem_u32(sW + stage * DEC_W_BYTES));
          const uint64_t x_desc = sdesc_sw128_kmajor(smem_u32(sX + stage * DEC_X_BYTES));
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_nvfp4(tmem + DEC_ACC_COL, w_desc + 2 * j, x_desc + 2 * j, idesc, tmem + dec_sfw_col(stage) + 4 * j,
                      tmem + dec_sfx_col(stage) + 4 * j, (kt != k0) | (j != 0));
          tc_commit(&c.empty[stage]);
          if (++stage == DEC_STAGES) { stage = 0; phase ^= 1; }
        }
        if (ok) tc_commit(&c.acc_full);
      }
      tc_commit(&c.drain);
      mbar_wait(&c.drain, 0);
    }
  } else if (warp >= DEC_COPY_WARP) {
    // ---------------------------------------------------------- scale copiers
    // Part 0: the weight's 4 atoms of the stage; part 1: the tokens' 4 atoms.
    if (lane == 0) {
      const int part = warp - DEC_COPY_WARP;
      int total = 0;
      for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
        int nt, split, k0, k1;
        unit_coords(p, u, nt, split, k0, k1);
        total += k1 - k0;
      }
      int stage = 0;
      uint32_t phase = 0;
      for (int g = 0; g < total; ++g) {
        if (!mbar_wait(&c.full[stage], phase)) break;
        tc_fence_after();
        const uint32_t src = smem_u32((part == 0 ? sSFW : sSFX) + stage * DEC_SF_BYTES);
        const uint32_t col = part == 0 ? dec_sfw_col(stage) : dec_sfx_col(stage);
#pragma unroll
        for (int j = 0; j < 4; ++j) cp_scale_atom<false>(tmem + col + 4 * j, src + j * SF_ATOM);
        tc_commit(&c.sf_ready[stage]);
        if (++stage == DEC_STAGES) { stage = 0; phase ^= 1; }
      }
      tc_commit(&c.sf_drain[part]);
      mbar_wait(&c.sf_drain[part], 0);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    // Warps 2..5: TMEM lane quadrant q = warp % 4, lane = weight row 32 q + lane of the
    // tile, one column per token.
    const int q = warp & 3;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < num_units; u += gridDim.x) {
      int nt, split, k0, k1;
      unit_coords(p, u, nt, split, k0, k1);
      if (!mbar_wait(&c.acc_full, acc_phase)) break;
      acc_phase ^= 1;
      tc_fence_after();
      uint32_t v[2][32];
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16) + DEC_ACC_COL;
      tmem_ld_32x32b_x32(lane_addr, v[0]);
      if (p.dn > 32) tmem_ld_32x32b_x32(lane_addr + 32, v[1]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.acc_empty);
      const int n = nt * DEC_BM + 32 * q + lane;
      if (n < p.N && p.partial == nullptr) {
        decode_direct_epilogue(p, n, v);
      } else if (n < p.N && NVFP4_DCHECK(split >= 0 && split < p.splits)) {
        float *dst = p.partial + (int64_t)split * p.M * p.N + n;
#pragma unroll
        for (int m = 0; m < 32; ++m)
          if (m < p.M) dst[(int64_t)m * p.N] = __uint_as_float(v[0][m]);
        if (p.dn > 32) {
#pragma unroll
          for (int m = 0; m < 32; ++m)
            if (32 + m < p.M) dst[(int64_t)(32 + m) * p.N] = __uint_as_float(v[1][m]);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
}

// ======================================================= split-K epilogue
// Sums the splits' partials and applies the epilogue of the linear, W consecutive
// output columns of one row per thread: W = 16 (one E4M3 block) for an NVFP4 output,
// so the thread writes its scale byte itself; W = 4 otherwise, so that a decode-size
// output (tens of rows) spreads over four times as many threads and loads in flight.
// Rows past M up to the next multiple of 128 only write zero scale bytes (NVFP4
// output).  Per output element the splits are added in split order.
constexpr int REDUCE_THREADS = 256;

// W consecutive column sums (col % W == 0, col + W <= N), added split by split in
// order, with several splits' loads in flight.
template <int W>
__device__ __forceinline__ void partial_sum(const Params &p, int row, int col, float (&y)[W]) {
  constexpr int V = W / 4;                 // float4 per split
  constexpr int F = W == 16 ? 2 : 4;       // splits loaded together
#pragma unroll
  for (int i = 0; i < W; ++i) y[i] = 0.0f;
  const int64_t stride4 = (int64_t)p.M * p.N / 4;
  const float4 *src = reinterpret_cast<const float4 *>(p.partial + (int64_t)row * p.N + col);
  int sp = 0;
  for (; sp + F <= p.splits; sp += F) {
    float4 a[F][V];
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
      for (int i = 0; i < V; ++i) a[f][i] = src[(sp + f) * stride4 + i];
#pragma unroll
    for (int f = 0; f < F; ++f)
#pragma unroll
      for (int i = 0; i < V; ++i) {
        y[4 * i] += a[f][i].x, y[4 * i + 1] += a[f][i].y, y[4 * i + 2] += a[f][i].z, y[4 * i + 3] += a[f][i].w;
      }
  }
  for (; sp < p.splits; ++sp) {
#pragma unroll
    for (int i = 0; i < V; ++i) {
      const float4 a = src[sp * stride4 + i];
      y[4 * i] += a.x, y[4 * i + 1] += a.y, y[4 * i + 2] += a.z, y[4 * i + 3] += a.w;
    }
  }
}

// Store W consecutive BF16 or FP32 outputs of one row.
template <int W>
__device__ __forceinline__ void store_w(const Params &p, int row, int col, const float (&y)[W]) {
  if constexpr (W == 16) {
    store16(p, row, col, y);
  } else {
    if (!NVFP4_DCHECK(row >= 0 && row < p.M && col >= 0 && col % W == 0 && col + W <= p.Nout)) return;
    if (p.out_kind == OUT_BF16) {
      const __nv_bfloat162 h0 = __floats2bfloat162_rn(y[0], y[1]), h1 = __floats2bfloat162_rn(y[2], y[3]);
      *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.out) + (int64_t)row * p.ldo + col) =
          make_uint2(*reinterpret_cast<const uint32_t *>(&h0), *reinterpret_cast<const uint32_t *>(&h1));
    } else if (p.out_kind == OUT_F32) {
      *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + (int64_t)row * p.ldo + col) =
          make_float4(y[0], y[1], y[2], y[3]);
    }
  }
}

// Re-quantise 16 consecutive outputs (one block) of one row: the per-block arithmetic
// of store64_nvfp4.
__device__ __forceinline__ void store16_nvfp4(const Params &p, const float *inv_out, int row, int col,
                                              const float (&y)[16], float gs_out) {
  if (!NVFP4_DCHECK(row >= 0 && row < p.M && col >= 0 && col % 16 == 0 && col + 16 <= p.Nout)) return;
  float x[16];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    x[i] = __bfloat162float(__float2bfloat16_rn(y[i]));
    amax = fmaxf(amax, fabsf(x[i]));
  }
  const uint32_t sf = block_scale_byte(amax, gs_out);
  const float inv = inv_out[sf & 127];
  *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(p.out) + (int64_t)row * (p.Nout / 2) + col / 2) =
      make_uint2(encode8(x, inv), encode8(x + 8, inv));
  p.out_scales[scale_word_offset(row, col / 64, p.out_kb_atoms) + (col / 16) % 4] = static_cast<uint8_t>(sf);
}

template <int W>
__global__ void __launch_bounds__(REDUCE_THREADS, 1) splitk_epilogue_kernel(const __grid_constant__ Params p) {
  __shared__ Ctrl<1> c;  // segment alphas and the NVFP4 output table
  grid_dep_wait();  // the partial sums come from the previous kernel
  grid_dep_launch();
  load_segments(p, c);
  __syncthreads();
  const int groups = p.Nout / W;  // Nout % 16 == 0
  const int64_t rows_cover = p.out_kind == OUT_NVFP4 ? (int64_t)(p.M + 127) / 128 * 128 : p.M;
  const int64_t idx = (int64_t)blockIdx.x * REDUCE_THREADS + threadIdx.x;
  if (idx >= rows_cover * groups) return;
  const int row = static_cast<int>(idx / groups);
  const int col = static_cast<int>(idx - (int64_t)row * groups) * W;
  if constexpr (W == 16) {
    if (row >= p.M) {
      p.out_scales[scale_word_offset(row, col / 64, p.out_kb_atoms) + (col / 16) % 4] = 0;
      return;
    }
  }
  float y[W];
  if (p.mode == MODE_SILU_MUL) {
    float u[W];
    partial_sum<W>(p, row, col, y);
    partial_sum<W>(p, row, p.up_row0 + col, u);
    const float ag = seg_alpha(c, p.nseg, col);
    const float au = seg_alpha(c, p.nseg, p.up_row0 + col);
#pragma unroll
    for (int i = 0; i < W; ++i) y[i] = silu_mul_f(ag * y[i], au * u[i]);
  } else {
    partial_sum<W>(p, row, col, y);
    const float a = seg_alpha(c, p.nseg, col);
#pragma unroll
    for (int i = 0; i < W; ++i) y[i] *= a;
  }
  if (touches_gates(p, col, W)) gdn_gates<W>(p, row, col, y);
  if constexpr (W == 16) {
    if (p.out_kind == OUT_NVFP4) {
      store16_nvfp4(p, c.inv_out, row, col, y, __ldg(p.gs_out));
      return;
    }
  }
  store_w<W>(p, row, col, y);
}

}  // namespace gemm
}  // namespace nvfp4
