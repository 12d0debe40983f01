// Gated delta-rule recurrence of the GDN layers (blog "27BハイブリッドLLMを4ビットで動かす",
// section "Gated DeltaNetの仕組み"): per value head the FP32 state S (d_k x d_v) takes,
// token by token,
//     S_t = alpha_t S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T,   alpha_t = exp(g_t),
// with g and beta the gate outputs of the in-projection's epilogue, and the layer reads
// o_t = S_t^T q_t.
//
// Every column j of S evolves on its own: (S^T k)_j, the write and (S^T q)_j only touch
// column j.  So the state is split by columns across CTAs and held in registers: a CTA
// owns 32 columns of one (sequence, value head); a thread owns two columns and an eighth
// (16 rows) of them, and dot products over d_k are finished with three shuffles inside
// an 8-lane group.  Two restatements keep the per-token work at three FMAs per state
// element:
//  * both dot products are taken on the state before the update, since
//        S_t^T q_t = alpha_t (S_{t-1}^T q_t) + (k_t . q_t) u_t,  u_t = beta_t (v_t - S_{t-1}^T k_t);
//  * the state is held as S = A S' with A the running product of the alphas, so the
//    decay is a scalar update and the write is one FMA per element:
//        A <- A alpha_t,   S' <- S' + k_t (u_t / A)^T.
//    Before A would drop below 2^-60, the scale is folded back into S' and that token
//    is applied in plain form (S' <- (A alpha_t) S' + k_t u_t^T, A <- 1); the branch is
//    uniform over the CTA.
// The inputs of TC tokens (k and q as BF16, k . q, v, alpha = exp(g), beta) are staged
// in double-buffered shared memory, loaded into registers one chunk ahead; outputs are
// gathered in shared memory and written once per chunk as full rows.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {
namespace gdn {

constexpr int kDim = 128;                 // d_k = d_v
constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kLanes = 8;                 // lanes per column pair
constexpr int kRows = kDim / kLanes;      // state rows per thread (16)
constexpr int kCols = 2 * (32 / kLanes) * kWarps;  // value columns per CTA (32)
constexpr int kColBlocks = kDim / kCols;  // CTAs per (sequence, value head)
constexpr int kGroupBytes = 48;           // 16 BF16 rows + 16 bytes: the eight row groups hit distinct banks
constexpr int kRowBytes = kLanes * kGroupBytes;  // one staged k or q row
constexpr float kMinScale = 0x1p-60f;     // fold A into S' before it drops below this

struct Args {
  const uint16_t *q, *k, *v;  // BF16 token rows: key head hk at column hk * 128, value head h at h * 128
  int64_t ld_qk, ld_v;        // row strides (elements) of q and k, and of v
  const float *g, *beta;  // FP32 [tokens x ld_gate], head h at column h
  int64_t ld_gate;
  const int32_t *cu_seqlens;  // [n_seqs + 1]
  int64_t tokens;
  int heads_per_key;  // value heads per key head
  float *state;       // [n_seqs][H_v][d_v][d_k]: element (i, j) of S at j * d_k + i
  int initial;        // 0: start from S = 0
  void *out;          // [tokens x ld_out], head h at column h * 128; BF16 or FP32
  int64_t ld_out;
  int out_fp32;
};

template <int TC>
struct Smem {
  alignas(16) unsigned char k[2][TC][kRowBytes];
  alignas(16) unsigned char q[2][TC][kRowBytes];
  alignas(16) float v[2][TC][kCols];
  alignas(16) float o[2][TC][kCols];
  float alpha[2][TC];
  float beta[2][TC];
  float kq[2][TC];
};

// One chunk of inputs in flight in registers.
template <int TC>
struct Stage {
  static constexpr int KQ = TC * 16 / kThreads;  // 16-byte words of k (and of q) per thread
  static_assert(TC * 16 % kThreads == 0 && TC * 4 <= kThreads, "chunk must be 8, 16 or 32 tokens");
  uint4 k[KQ], q[KQ], v;
  float g, b;
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)),
        "l"(*reinterpret_cast<uint64_t *>(&c)));
  return *reinterpret_cast<float2 *>(&d);
}

__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}

// 8 BF16 values -> 8 floats in shared memory (two 16-byte stores).
__device__ __forceinline__ void store_bf16x8(float *dst, const uint4 &w) {
  reinterpret_cast<float4 *>(dst)[0] = make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xFFFF0000u),
                                                   __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xFFFF0000u));
  reinterpret_cast<float4 *>(dst)[1] = make_float4(__uint_as_float(w.z << 16), __uint_as_float(w.z & 0xFFFF0000u),
                                                   __uint_as_float(w.w << 16), __uint_as_float(w.w & 0xFFFF0000u));
}

// Dot product of 8 BF16 pairs, in FP32.
__device__ __forceinline__ float dot_bf16x8(const uint4 &a, const uint4 &b) {
  const uint32_t x[4] = {a.x, a.y, a.z, a.w}, y[4] = {b.x, b.y, b.z, b.w};
  float d = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    d = fmaf(__uint_as_float(x[i] << 16), __uint_as_float(y[i] << 16), d);
    d = fmaf(__uint_as_float(x[i] & 0xFFFF0000u), __uint_as_float(y[i] & 0xFFFF0000u), d);
  }
  return d;
}

template <int TC>
__device__ __forceinline__ void load_stage(const Args &a, Stage<TC> &st, int64_t t0, int64_t end, int hk, int h,
                                           int cb) {
  const int tid = threadIdx.x;
  const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int n = 0; n < Stage<TC>::KQ; ++n) {
    const int idx = tid + n * kThreads;
    const int64_t tok = t0 + (idx >> 4);
    const int64_t off = tok * a.ld_qk + hk * kDim + (idx & 15) * 8;
    st.k[n] = tok < end ? __ldg(reinterpret_cast<const uint4 *>(a.k + off)) : zero;
    st.q[n] = tok < end ? __ldg(reinterpret_cast<const uint4 *>(a.q + off)) : zero;
  }
  st.v = zero;
  if (tid < TC * 4) {
    const int64_t tok = t0 + (tid >> 2);
    if (tok < end) st.v = __ldg(reinterpret_cast<const uint4 *>(a.v + tok * a.ld_v + h * kDim + cb * kCols + (tid & 3) * 8));
  }
  st.g = 0.0f;
  st.b = 0.0f;
  if (tid < TC) {
    const int64_t tok = t0 + tid;
    if (tok < end) {
      st.g = __ldg(a.g + tok * a.ld_gate + h);
      st.b = __ldg(a.beta + tok * a.ld_gate + h);
    }
  }
}

template <int TC>
__device__ __forceinline__ void store_stage(Smem<TC> &sm, const Stage<TC> &st, int buf) {
  const int tid = threadIdx.x;
#pragma unroll
  for (int n = 0; n < Stage<TC>::KQ; ++n) {
    const int idx = tid + n * kThreads;
    const int tt = idx >> 4, cc = idx & 15;  // 16 consecutive lanes hold one token's 128 rows
    const int off = (cc >> 1) * kGroupBytes + (cc & 1) * 16;  // row group, then 8 rows within it
    *reinterpret_cast<uint4 *>(&sm.k[buf][tt][off]) = st.k[n];
    *reinterpret_cast<uint4 *>(&sm.q[buf][tt][off]) = st.q[n];
    float d = dot_bf16x8(st.k[n], st.q[n]);
    d += __shfl_xor_sync(0xffffffffu, d, 1);
    d += __shfl_xor_sync(0xffffffffu, d, 2);
    d += __shfl_xor_sync(0xffffffffu, d, 4);
    d += __shfl_xor_sync(0xffffffffu, d, 8);
    if (cc == 0) sm.kq[buf][tt] = d;  // k_t . q_t
  }
  if (tid < TC * 4) store_bf16x8(&sm.v[buf][tid >> 2][(tid & 3) * 8], st.v);
  if (tid < TC) {
    sm.alpha[buf][tid] = expf(st.g);
    sm.beta[buf][tid] = st.b;
  }
}

// Write the chunk's outputs (n tokens from t0) as rows of 32 columns.
template <int TC>
__device__ __forceinline__ void write_out(const Args &a, const Smem<TC> &sm, int buf, int64_t t0, int n, int h,
                                          int cb) {
  const int tid = threadIdx.x;
  const int64_t col = (int64_t)h * kDim + cb * kCols;
  if (a.out_fp32) {
    for (int idx = tid; idx < n * 8; idx += kThreads) {  // 4 floats per item
      const int tt = idx >> 3, part = idx & 7;
      const float4 x = *reinterpret_cast<const float4 *>(&sm.o[buf][tt][part * 4]);
      *reinterpret_cast<float4 *>(static_cast<float *>(a.out) + (t0 + tt) * a.ld_out + col + part * 4) = x;
    }
  } else {
    for (int idx = tid; idx < n * 4; idx += kThreads) {  // 8 BF16 per item
      const int tt = idx >> 2, part = idx & 3;
      const float *x = &sm.o[buf][tt][part * 8];
      uint32_t w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        __nv_bfloat162 b = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
        w[i] = *reinterpret_cast<uint32_t *>(&b);
      }
      *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + (t0 + tt) * a.ld_out + col + part * 8) =
          make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

// 8 BF16 values -> 4 float2 pairs.
__device__ __forceinline__ void unpack_bf16x8(const uint4 &w, float2 *f) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) f[i] = make_float2(__uint_as_float(x[i] << 16), __uint_as_float(x[i] & 0xFFFF0000u));
}

// Grid (d_v / 32, H_v, n_seqs), kThreads threads, sizeof(Smem<TC>) bytes of dynamic shared memory.
template <int TC>
__global__ void __launch_bounds__(kThreads) recurrence_kernel(const __grid_constant__ Args a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  Smem<TC> &sm = *reinterpret_cast<Smem<TC> *>(smem_raw);
  const int cb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / a.heads_per_key;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jl = 2 * (warp * (32 / kLanes) + lane / kLanes);  // first of the thread's two columns
  const int r = lane % kLanes;                                // row group: rows 16 r .. 16 r + 15
  grid_dep_wait();
  grid_dep_launch();
  const int64_t start = __ldg(a.cu_seqlens + b), end = __ldg(a.cu_seqlens + b + 1);
  if (start < 0 || end < start || end > a.tokens) {
    if (threadIdx.x == 0) atomicCAS(&g_device_status, 0, kStatusBadIndex);
    return;
  }
  float *srow = a.state + (((int64_t)b * gridDim.y + h) * kDim + cb * kCols + jl) * kDim + r * kRows;

  constexpr int P = kRows / 2;  // float2 pairs per column
  float2 S[2][P];               // S' of columns jl, jl + 1, rows 16 r .. 16 r + 15
  if (a.initial) {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int p = 0; p < P / 2; ++p) {
        const float4 x = reinterpret_cast<const float4 *>(srow + c * kDim)[p];
        S[c][2 * p] = make_float2(x.x, x.y);
        S[c][2 * p + 1] = make_float2(x.z, x.w);
      }
  } else {
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int p = 0; p < P; ++p) S[c][p] = make_float2(0.0f, 0.0f);
  }
  float A = 1.0f;  // S = A S'

  const int64_t len = end - start;
  const int64_t nchunks = (len + TC - 1) / TC;
  Stage<TC> st;
  if (nchunks > 0) load_stage<TC>(a, st, start, end, hk, h, cb);
  for (int64_t c = 0; c < nchunks; ++c) {
    const int buf = c & 1;
    const int64_t t0 = start + c * TC;
    store_stage<TC>(sm, st, buf);
    __syncthreads();  // chunk c staged; every warp is done with chunk c - 1
    if (c > 0) write_out<TC>(a, sm, buf ^ 1, t0 - TC, TC, h, cb);
    if (c + 1 < nchunks) load_stage<TC>(a, st, t0 + TC, end, hk, h, cb);
    const int n = static_cast<int>(end - t0 < TC ? end - t0 : TC);
    for (int t = 0; t < n; ++t) {
      const uint4 *kp = reinterpret_cast<const uint4 *>(&sm.k[buf][t][r * kGroupBytes]);
      const uint4 *qp = reinterpret_cast<const uint4 *>(&sm.q[buf][t][r * kGroupBytes]);
      float2 kk[P], qq[P];
      unpack_bf16x8(kp[0], kk);
      unpack_bf16x8(kp[1], kk + 4);
      unpack_bf16x8(qp[0], qq);
      unpack_bf16x8(qp[1], qq + 4);
      float pk[2], pq[2];
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float2 ak0 = make_float2(0.0f, 0.0f), ak1 = ak0, aq0 = ak0, aq1 = ak0;
#pragma unroll
        for (int p = 0; p < P; p += 2) {
          ak0 = ffma2(S[cc][p], kk[p], ak0);
          ak1 = ffma2(S[cc][p + 1], kk[p + 1], ak1);
          aq0 = ffma2(S[cc][p], qq[p], aq0);
          aq1 = ffma2(S[cc][p + 1], qq[p + 1], aq1);
        }
        pk[cc] = (ak0.x + ak0.y) + (ak1.x + ak1.y);
        pq[cc] = (aq0.x + aq0.y) + (aq1.x + aq1.y);
      }
#pragma unroll
      for (int m = 1; m < kLanes; m <<= 1) {
        pk[0] += __shfl_xor_sync(0xffffffffu, pk[0], m);
        pk[1] += __shfl_xor_sync(0xffffffffu, pk[1], m);
        pq[0] += __shfl_xor_sync(0xffffffffu, pq[0], m);
        pq[1] += __shfl_xor_sync(0xffffffffu, pq[1], m);
      }
      // A pk = (S_{t-1}^T k_t)_j, A pq = (S_{t-1}^T q_t)_j
      const float al = sm.alpha[buf][t], be = sm.beta[buf][t], kq = sm.kq[buf][t];
      const float2 vv = *reinterpret_cast<const float2 *>(&sm.v[buf][t][jl]);
      const float u0 = be * (vv.x - A * pk[0]), u1 = be * (vv.y - A * pk[1]);
      const float An = A * al;
      if (r == 0)
        *reinterpret_cast<float2 *>(&sm.o[buf][t][jl]) = make_float2(fmaf(kq, u0, An * pq[0]), fmaf(kq, u1, An * pq[1]));
      if (An >= kMinScale) {
        const float inv = __frcp_rn(An);
        const float2 w0 = make_float2(u0 * inv, u0 * inv), w1 = make_float2(u1 * inv, u1 * inv);
#pragma unroll
        for (int p = 0; p < P; ++p) {
          S[0][p] = ffma2(kk[p], w0, S[0][p]);
          S[1][p] = ffma2(kk[p], w1, S[1][p]);
        }
        A = An;
      } else {  // fold the scale in and apply this token as written
        const float2 a2 = make_float2(An, An), w0 = make_float2(u0, u0), w1 = make_float2(u1, u1);
#pragma unroll
        for (int p = 0; p < P; ++p) {
          S[0][p] = ffma2(kk[p], w0, fmul2(a2, S[0][p]));
          S[1][p] = ffma2(kk[p], w1, fmul2(a2, S[1][p]));
        }
        A = 1.0f;
      }
    }
  }
  if (nchunks > 0) {
    __syncthreads();
    const int64_t c = nchunks - 1;
    write_out<TC>(a, sm, c & 1, start + c * TC, static_cast<int>(end - start - c * TC), h, cb);
  }
  const float2 a2 = make_float2(A, A);
#pragma unroll
  for (int c = 0; c < 2; ++c)
#pragma unroll
    for (int p = 0; p < P / 2; ++p) {
      const float2 x = fmul2(a2, S[c][2 * p]), y = fmul2(a2, S[c][2 * p + 1]);
      reinterpret_cast<float4 *>(srow + c * kDim)[p] = make_float4(x.x, x.y, y.x, y.y);
    }
}

// ------------------------------------------------------ one warp per state columns
// Sequences of a few tokens (decode): every state element is read and written once per
// call, so the pass is HBM-bound, and the column-major state gives each column j of a
// (sequence, value head) its own contiguous 512 bytes.  One warp owns kColPerWarp
// columns: lane l holds rows 4 l .. 4 l + 3 of each (one 16-byte load per column, all in
// flight together), and a token's dot products, S^T k and S^T q per column and k . q,
// finish with warp reductions:
//     u = beta (v_j - (S^T k)_j),   S_j <- alpha S_j + u k,   o_j = alpha (S^T q)_j + (k . q) u.
constexpr int kColWarps = 8;
constexpr int kColPerWarp = 4;
constexpr int kColThreads = 32 * kColWarps;
constexpr int kColBlocksPerHead = kDim / (kColWarps * kColPerWarp);

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Grid (kColBlocksPerHead, H_v, n_seqs), kColThreads threads, no dynamic shared memory.
__global__ void __launch_bounds__(kColThreads) column_kernel(const __grid_constant__ Args a) {
  grid_dep_wait();
  grid_dep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = (blockIdx.x * kColWarps + warp) * kColPerWarp, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / a.heads_per_key;
  const int64_t start = __ldg(a.cu_seqlens + b), end = __ldg(a.cu_seqlens + b + 1);
  if (start < 0 || end < start || end > a.tokens) {
    if (threadIdx.x == 0 && blockIdx.x == 0) atomicCAS(&g_device_status, 0, kStatusBadIndex);
    return;
  }
  // global [b][h][j][i] holds S[i][j]
  float4 *col = reinterpret_cast<float4 *>(a.state + (((int64_t)b * gridDim.y + h) * kDim + j0) * kDim) + lane;
  float4 s[kColPerWarp];
#pragma unroll
  for (int c = 0; c < kColPerWarp; ++c) s[c] = a.initial ? col[c * (kDim / 4)] : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int64_t t = start; t < end; ++t) {
    const uint2 kw = __ldg(reinterpret_cast<const uint2 *>(a.k + t * a.ld_qk + hk * kDim) + lane);
    const uint2 qw = __ldg(reinterpret_cast<const uint2 *>(a.q + t * a.ld_qk + hk * kDim) + lane);
    const float k0 = __uint_as_float(kw.x << 16), k1 = __uint_as_float(kw.x & 0xFFFF0000u);
    const float k2 = __uint_as_float(kw.y << 16), k3 = __uint_as_float(kw.y & 0xFFFF0000u);
    const float q0 = __uint_as_float(qw.x << 16), q1 = __uint_as_float(qw.x & 0xFFFF0000u);
    const float q2 = __uint_as_float(qw.y << 16), q3 = __uint_as_float(qw.y & 0xFFFF0000u);
    const float alpha = expf(__ldg(a.g + t * a.ld_gate + h));
    const float be = __ldg(a.beta + t * a.ld_gate + h);
    const float kq = warp_sum(fmaf(k3, q3, fmaf(k2, q2, fmaf(k1, q1, k0 * q0))));
#pragma unroll
    for (int c = 0; c < kColPerWarp; ++c) {
      const int j = j0 + c;
      const float vj = __uint_as_float(static_cast<uint32_t>(__ldg(a.v + t * a.ld_v + h * kDim + j)) << 16);
      float4 &x = s[c];
      const float sk = warp_sum(fmaf(x.w, k3, fmaf(x.z, k2, fmaf(x.y, k1, x.x * k0))));
      const float sq = warp_sum(fmaf(x.w, q3, fmaf(x.z, q2, fmaf(x.y, q1, x.x * q0))));
      const float u = be * (vj - sk);
      x.x = fmaf(alpha, x.x, k0 * u);
      x.y = fmaf(alpha, x.y, k1 * u);
      x.z = fmaf(alpha, x.z, k2 * u);
      x.w = fmaf(alpha, x.w, k3 * u);
      if (lane == c) {
        const float o = fmaf(alpha, sq, kq * u);
        const int64_t at = t * a.ld_out + (int64_t)h * kDim + j;
        if (a.out_fp32) {
          static_cast<float *>(a.out)[at] = o;
        } else {
          const __nv_bfloat16 ob = __float2bfloat16_rn(o);
          static_cast<uint16_t *>(a.out)[at] = *reinterpret_cast<const uint16_t *>(&ob);
        }
      }
    }
  }
#pragma unroll
  for (int c = 0; c < kColPerWarp; ++c) col[c * (kDim / 4)] = s[c];
}

}  // namespace gdn
}  // namespace nvfp4
