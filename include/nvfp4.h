/*
 * nvfp4.h - C ABI of the B200 (sm_100a) NVFP4 W4A4 linear library.
 *
 * The method: every linear layer of a hybrid Gated-DeltaNet / attention LLM runs
 * with both weights and activations in NVFP4 (W4A4): 4-bit E2M1 values, one E4M3
 * scale per 16 consecutive elements, and one FP32 global scale per tensor; the
 * GEMM runs on 4-bit tensor cores.  Sources: blog "27BハイブリッドLLMを4ビットで動かす
 * ——Gated DeltaNetはなぜ量子化に耐えるのか", sections 機構① (block format, block maximum
 * sets the scale), 機構② (GDN gate formulas), 罠① (per-module global scales in a
 * fused GEMM) and FAQ; abstract page "Why Gated DeltaNet Survives 4-Bit
 * Quantization" (arXiv 2609.04098).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - All tensor pointers are DEVICE pointers owned by the caller.  The library never
 *   allocates, frees or keeps them; it launches work on `stream` and returns
 *   without synchronising.  Results are valid once the stream reaches that point.
 * - `stream` is a cudaStream_t (NULL = the legacy default stream).  The current
 *   CUDA device must be the device that owns the pointers.
 * - Matrices are row-major.  BF16 inputs are IEEE bfloat16 bit patterns.
 * - Packed NVFP4 codes: two E2M1 codes per byte, the element with the even column
 *   index in the low nibble; row r of a [rows x cols] tensor starts at byte r*cols/2.
 * - Block scales: unsigned E4M3 bytes, one per 16-element row block, stored in
 *   512-byte atoms of 128 rows x 4 blocks: row r, block j of an atom sits at byte
 *   (r%32)*16 + (r/32)*4 + j; atoms are ordered block-index fastest; rows are
 *   padded to a multiple of 128 and blocks to a multiple of 4 (padding written as 0
 *   by nvfp4_quantize).  This is the layout the tcgen05 block-scaled MMA reads.
 * - Global scale: gs = 2688 / amax(|x|) (2688 = 448 * 6), FP32, in device memory;
 *   a quantised value means e2m1(code) * e4m3(scale) / gs.
 * - Errors are returned, never printed, and no kernel is launched when a check fails.
 *   NVFP4_ERR_CUDA means a CUDA runtime call failed (cudaGetLastError is left set).
 */
#ifndef NVFP4_W4A4_H
#define NVFP4_W4A4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define NVFP4_API __attribute__((visibility("default")))
#else
#define NVFP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nvfp4_stream_t; /* same type as cudaStream_t */

typedef enum {
  NVFP4_OK = 0,
  NVFP4_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, unknown enum value */
  NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* a size violates the documented divisibility rules */
  NVFP4_ERR_MISALIGNED = 3,        /* a pointer or leading dimension violates alignment */
  NVFP4_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
  NVFP4_ERR_DEVICE_TIMEOUT = 5,    /* a kernel gave up a bounded wait (see nvfp4_get_device_status) */
  NVFP4_ERR_UNSUPPORTED_DEVICE = 6, /* current device is not sm_100 */
  NVFP4_ERR_DEVICE_INDEX = 7        /* a kernel skipped an out-of-range index (see nvfp4_get_device_status) */
} nvfp4_status_t;

/* Human-readable name of a status code (static storage). */
NVFP4_API const char *nvfp4_status_string(int status);

/* Bytes of the swizzled scale buffer of a [rows x cols] NVFP4 tensor:
 * ceil(rows/128)*128 * ceil(cols/64)*4.  Returns 0 for invalid sizes. */
NVFP4_API size_t nvfp4_scale_bytes(int64_t rows, int64_t cols);

/*
 * nvfp4_amax - max|x| of a BF16 tensor, written as FP32 to *amax_out (device).  The
 *   calibration step behind static global scales (blog section 罠①: every module keeps
 *   the global scale it was calibrated with): run it over calibration inputs and
 *   derive gs = 2688 / amax (the formula of nvfp4_global_scale) on the caller's side.
 *   Exact (a maximum of BF16 magnitudes).  Same requirements and errors as
 *   nvfp4_global_scale.
 */
NVFP4_API nvfp4_status_t nvfp4_amax(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld, float *amax_out,
                                    nvfp4_stream_t stream);

/*
 * nvfp4_global_scale - per-tensor FP32 global scale from the tensor's amax.
 *   Computes gs = fl32(2688 / max|x|) over x [rows x cols] (row stride `ld`
 *   elements) and writes it to *gs_out (device).  max|x| == 0 gives gs = 1.
 *   Source: blog section 罠① (each linear module has its own global scale); the
 *   formula is this library's reading (the pages give none).
 *   Requirements: rows, cols >= 1; ld >= cols; x 16-byte aligned and ld % 8 == 0;
 *   gs_out 4-byte aligned.  Non-finite inputs are unsupported.
 */
NVFP4_API nvfp4_status_t nvfp4_global_scale(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                  float *gs_out, nvfp4_stream_t stream);

/*
 * nvfp4_quantize - NVFP4 block quantisation of a BF16 matrix.
 *   For each 16-element row block b of x [rows x cols]:
 *     s    = fl32(fl32(amax_b / 6) * gs)
 *     sf_b = E4M3(s)  (round to nearest even, saturate at 448)
 *     code = E2M1(fl32(x * fl32(gs / e4m3(sf_b))))  (nearest even, saturate at 6,
 *            sign copied; 0 when sf_b == 0)
 *   Source: blog section 機構① (16-element blocks, E4M3 block scale set by the block
 *   maximum, E2M1 values).  Operation order and rounding are this library's reading.
 *   x: device BF16, row stride ld elements (ld >= cols, ld % 8 == 0, 16-byte aligned).
 *   gs: device FP32 scalar (static calibrated scale, or nvfp4_global_scale's output).
 *   codes: device, rows*cols/2 bytes, 16-byte aligned.
 *   scales: device, nvfp4_scale_bytes(rows, cols) bytes, 16-byte aligned; padding
 *   bytes are written with 0.
 *   Requirements: rows >= 1, cols >= 16, cols % 16 == 0.
 */
NVFP4_API nvfp4_status_t nvfp4_quantize(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                              const float *gs, uint8_t *codes, uint8_t *scales,
                              nvfp4_stream_t stream);

/*
 * nvfp4_quantize_rows - nvfp4_quantize into rows [row_offset, row_offset + rows) of
 *   a larger destination tensor of total_rows rows (same cols): `codes` and
 *   `scales` are the buffers of the whole destination.  This packs a fused weight
 *   whose modules keep their own global scales (blog section 罠①): one call per
 *   module, each with its own gs, into one weight.  Scale bytes of other rows are
 *   untouched, except that the call that ends at total_rows also zero-fills the
 *   padding rows up to a multiple of 128.  Calls on disjoint row ranges may run
 *   concurrently.  nvfp4_quantize(...) == nvfp4_quantize_rows(..., 0, rows, ...).
 *   Requirements as nvfp4_quantize, plus 0 <= row_offset, row_offset + rows <= total_rows.
 */
NVFP4_API nvfp4_status_t nvfp4_quantize_rows(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                             const float *gs, uint8_t *codes, uint8_t *scales,
                                             int64_t row_offset, int64_t total_rows, nvfp4_stream_t stream);

/* A quantised operand of the GEMM: [rows x K] NVFP4, both K-major. */
typedef struct {
  const uint8_t *codes;  /* device, rows*K/2 bytes, 16-byte aligned */
  const uint8_t *scales; /* device, nvfp4_scale_bytes(rows, K) bytes, 16-byte aligned */
  int64_t rows;
  int64_t K;
} nvfp4_operand_t;

/* One separately calibrated module inside a fused weight: weight rows (= output
 * columns of the GEMM) [n_begin, n_end) carry global scale *gs_w (device). */
typedef struct {
  int64_t n_begin;
  int64_t n_end;
  const float *gs_w;
} nvfp4_segment_t;

#define NVFP4_MAX_SEGMENTS 16

typedef enum {
  NVFP4_EPI_NONE = 0,      /* y = alpha(n) * acc */
  NVFP4_EPI_SILU_MUL = 1,  /* W = [gate; up] (2*Nh rows): y[:, j] = SiLU(y_gate[:, j]) * y_up[:, j] */
  NVFP4_EPI_GDN_GATES = 2  /* columns of the beta head block -> sigmoid; of the alpha block -> g */
} nvfp4_epilogue_t;

typedef enum {
  NVFP4_OUT_BF16 = 0,  /* out: BF16 [M x Nout], row stride ldo elements */
  NVFP4_OUT_F32 = 1,   /* out: FP32 [M x Nout], row stride ldo elements */
  NVFP4_OUT_NVFP4 = 2  /* out: packed codes [M x Nout/2] (ldo ignored) + ep->out_scales,
                          quantised with ep->gs_out after rounding y to BF16 */
} nvfp4_out_kind_t;

typedef struct {
  /* NVFP4_EPI_GDN_GATES: g = -exp(A_log[h]) * softplus(y + dt_bias[h]) on columns
   * [alpha_begin, alpha_begin + n_heads), beta = sigmoid(y) on columns
   * [beta_begin, beta_begin + n_heads); h = column - block begin.  The gated values
   * replace y in `out`; when non-NULL, FP32 copies go to beta_out / g_out
   * ([M x n_heads], row stride n_heads). */
  int64_t beta_begin;
  int64_t alpha_begin;
  int64_t n_heads;
  const float *A_log;   /* device [n_heads] */
  const float *dt_bias; /* device [n_heads] */
  float *beta_out;      /* device or NULL */
  float *g_out;         /* device or NULL */
  /* NVFP4_OUT_NVFP4: global scale of the output (device scalar) and its scale buffer
   * (nvfp4_scale_bytes(M, Nout) bytes). */
  const float *gs_out;
  uint8_t *out_scales;
} nvfp4_epilogue_params_t;

/*
 * nvfp4_linear - fused W4A4 linear: block-scaled FP4 x FP4 GEMM on tcgen05 tensor
 * cores with per-segment global-scale correction and a selectable epilogue.
 *   acc[m, n] = sum_k e2m1(A)[m,k] e4m3(sfA)[m,k/16] e2m1(W)[n,k] e4m3(sfW)[n,k/16]  (FP32)
 *   y[m, n]   = acc[m, n] / (gs_a * gs_w(seg(n)))
 *   then the epilogue; out = epilogue(y) stored as `out_kind`.
 *   Sources: blog FAQ (W4A4 on 4-bit tensor cores), section 罠① (fused modules need
 *   their own global-scale correction; here a per-segment alpha), section 機構② (gates).
 *   A: [M x K] activations; gs_a: device FP32 scalar.  W: [N x K] weights.
 *   segs/nseg: 1..16 segments, sorted, disjoint, covering [0, N); bounds % 16 == 0.
 *   Requirements: M >= 1; K % 256 == 0; N % 16 == 0; for SILU_MUL, N % 256 == 0
 *   and Nout = N/2, else Nout = N; ldo >= Nout; out 16-byte aligned and ldo*elem % 16 == 0;
 *   NVFP4 output needs Nout % 64 == 0.  GDN_GATES needs n_heads >= 1 and both head
 *   blocks inside [0, N).
 *   ep may be NULL for NVFP4_EPI_NONE with BF16/F32 output.
 */
NVFP4_API nvfp4_status_t nvfp4_linear(const nvfp4_operand_t *A, const float *gs_a, const nvfp4_operand_t *W,
                            const nvfp4_segment_t *segs, int nseg, int epilogue,
                            const nvfp4_epilogue_params_t *ep, void *out, int out_kind,
                            int64_t ldo, nvfp4_stream_t stream);

/*
 * nvfp4_linear_splitk - nvfp4_linear with the K dimension split over `split_k` work
 * units per output tile: the decode regime (few token rows), where one unit per
 * output tile would leave most SMs idle while the weights stream from HBM.
 *   Each unit accumulates its K range on the tensor cores and writes its raw FP32
 *   sums to `workspace` ([split_k x M x N] floats); a second kernel adds the splits
 *   and applies exactly the epilogue and output kind of nvfp4_linear (per-segment
 *   alpha, SiLU*mul or GDN gates, BF16 / FP32 / NVFP4 store).  Results equal
 *   nvfp4_linear's up to the order of the FP32 additions.
 *   Up to 64 token rows (M <= 64) a unit is 128 weight rows x all tokens x its K
 *   range, computed with the weight as the MMA's 128-row operand and the tokens
 *   (padded to 32 or 64) as its N; above 64 rows it is an output tile of 128 x 256.
 *   Source: the blog's results section (結果: decode at concurrency 32, 1,154 tok/s
 *   against 621 tok/s in BF16) is the regime; the method is nvfp4_linear's.
 *   Arguments as nvfp4_linear, plus:
 *   split_k: 1 .. K/256 (nvfp4_splitk_default gives the library's choice); with 1
 *   and M > 64 the call runs nvfp4_linear itself and does not touch the workspace
 *   (with M <= 64 one split still goes through the workspace and the second kernel);
 *   workspace: device, >= nvfp4_splitk_workspace_bytes(M, N, split_k) bytes,
 *   16-byte aligned, owned by the caller; its contents on entry do not matter and
 *   are overwritten.  Two calls that share a workspace must not overlap on the GPU.
 *   Errors: NVFP4_ERR_INVALID_ARG for a bad split_k, a NULL or too small workspace;
 *   otherwise as nvfp4_linear.
 */
NVFP4_API nvfp4_status_t nvfp4_linear_splitk(const nvfp4_operand_t *A, const float *gs_a,
                                             const nvfp4_operand_t *W, const nvfp4_segment_t *segs, int nseg,
                                             int epilogue, const nvfp4_epilogue_params_t *ep, void *out,
                                             int out_kind, int64_t ldo, int split_k, void *workspace,
                                             size_t workspace_bytes, nvfp4_stream_t stream);

/* Bytes of the workspace nvfp4_linear_splitk needs: split_k * M * N * 4 (0 for
 * invalid sizes). */
NVFP4_API size_t nvfp4_splitk_workspace_bytes(int64_t M, int64_t N, int split_k);

/* The split count the library would choose for an M x N x K linear on the current
 * device (>= 1, <= K/256): as many splits as keep all (tile, K range) work units in
 * one wave on the SMs, i.e. SMs / tiles rounded down, with at least 4 K tiles of 256
 * per split.  A tile is 128 weight rows for M <= 64 and 128 x 256 outputs above.  0
 * for invalid sizes or when the device cannot be queried. */
NVFP4_API int nvfp4_splitk_default(int64_t M, int64_t N, int64_t K);

/*
 * nvfp4_linear_splitk_noalloc - nvfp4_linear_splitk for callers that cannot allocate
 * device memory: the split-K partial sums go to a fixed scratch array inside the
 * library instead of a caller workspace.  The pages have no counterpart of this entry
 * point; it serves integrations whose interface hands the library only inputs and
 * outputs (a plugin or custom-op hook with no workspace argument), or which must not
 * allocate on the serving path, where cudaMalloc can synchronise the device and add
 * latency.
 *   Arguments and results as nvfp4_linear_splitk, without the workspace.  The call
 *   allocates nothing (no cudaMalloc, no cudaFree, no allocating library routine).
 *   Scratch: NVFP4_NOALLOC_SCRATCH_BYTES of device memory held by every GPU that loads
 *   the library until the process exits.  The first call on a device looks up the
 *   array's device address (once per device, with that device current); make that
 *   first call before any stream capture.  Every call shares the array and leaves
 *   its contents behind; each call overwrites all of the scratch it reads, so no
 *   state carries over, but calls that overlap on the GPU (other streams, other host
 *   threads) race on it and must be serialised by the caller.
 *   One split above 64 rows needs no partials: that call runs nvfp4_linear and uses
 *   no scratch (whatever M * N).  The array's device address is kept per device index
 *   for the life of the process; a cudaDeviceReset invalidates it, so a process that
 *   resets a device must not call this entry point on that device again.
 *   Errors: NVFP4_ERR_UNSUPPORTED_SHAPE when split_k * M * N * 4 bytes exceed
 *   NVFP4_NOALLOC_SCRATCH_BYTES (use fewer splits or nvfp4_linear_splitk);
 *   NVFP4_ERR_CUDA if the scratch address cannot be looked up; otherwise as
 *   nvfp4_linear_splitk.
 */
#define NVFP4_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
NVFP4_API nvfp4_status_t nvfp4_linear_splitk_noalloc(const nvfp4_operand_t *A, const float *gs_a,
                                                     const nvfp4_operand_t *W, const nvfp4_segment_t *segs,
                                                     int nseg, int epilogue, const nvfp4_epilogue_params_t *ep,
                                                     void *out, int out_kind, int64_t ldo, int split_k,
                                                     nvfp4_stream_t stream);

/*
 * nvfp4_unswizzle_scales - the block scales of a packed NVFP4 tensor in logical order.
 *   out[r * ld + j] = the E4M3 scale byte of row r, 16-element block j, for
 *   r < rows, j < cols / 16, read from the swizzled buffer `scales` (the layout of the
 *   conventions above).  For callers that inspect or export scales (checkpoint
 *   writers, debugging); the GEMM reads the swizzled form directly.
 *   scales: device, nvfp4_scale_bytes(rows, cols) bytes, 16-byte aligned.
 *   out: device, rows x ld bytes (any alignment), ld >= cols / 16.  Caller-owned.
 *   Errors: INVALID_ARG (NULL, rows < 1, ld too small), UNSUPPORTED_SHAPE
 *   (cols % 16), MISALIGNED (scales).
 */
NVFP4_API nvfp4_status_t nvfp4_unswizzle_scales(const uint8_t *scales, int64_t rows, int64_t cols, uint8_t *out,
                                                int64_t ld, nvfp4_stream_t stream);

/*
 * nvfp4_pack_weight - pack separately quantised modules into one fused NVFP4 weight
 * (blog section 罠①: modules fused into one GEMM keep their own global scales; pair
 * the result with a segment table [(row0_i, row0_i + rows_i, gs_i)] in nvfp4_linear).
 *   parts[i]: module i, codes [rows_i x K/2] and its own scale buffer (as written by
 *   nvfp4_quantize), all with the same K.  Module i lands at fused rows
 *   [row0_i, row0_i + rows_i), row0_i = rows_0 + ... + rows_{i-1} (unaligned offsets
 *   allowed).  Rows [sum rows_i, rows_out) are padding of the output dimension (for
 *   example to a multiple of the GEMM's 256-column tile): zero codes, zero scales.
 *   Scale padding (rows up to a multiple of 128) is written as zero.  The result is
 *   byte-identical to quantising the modules straight into the fused buffer with
 *   nvfp4_quantize_rows.  The gate|up order of a SiLU*mul weight needs no interleave:
 *   the GEMM reads the two halves at their logical offsets.
 *   codes: device [rows_out x K/2]; scales: device, nvfp4_scale_bytes(rows_out, K)
 *   bytes; both 16-byte aligned, caller-owned, not overlapping the parts.
 *   Requirements: 1 <= nparts <= NVFP4_MAX_SEGMENTS, K % 64 == 0, rows_out >= the
 *   modules' total rows.  Errors: INVALID_ARG, UNSUPPORTED_SHAPE (K % 64),
 *   MISALIGNED.
 */
NVFP4_API nvfp4_status_t nvfp4_pack_weight(const nvfp4_operand_t *parts, int nparts, uint8_t *codes, uint8_t *scales,
                                           int64_t rows_out, nvfp4_stream_t stream);

/*
 * nvfp4_fold_segments - fused-group scale repair, in place: rewrites a packed fused
 * weight whose modules carry their own global scales so that one global scale serves
 * them all (the pages' own repair of the fused-module mismatch: blog section 罠①,
 * "common global scale, ratio folded into the block scales, re-rounding <= 6.2 %").
 *   gs_c = min over the modules of *segs[i].gs_w, written to *gs_common_out (device);
 *   every block scale of module i becomes E4M3(fl32(dec(sf) * fl32(gs_c / gs_i)))
 *   (nearest even); codes are unchanged.  Afterwards nvfp4_linear with the single
 *   segment [(0, rows, gs_common_out)] approximates the per-module linear: each
 *   decoded weight moves by at most 2^-4 of itself (normal scales).  The per-segment
 *   alpha of nvfp4_linear needs no such repair and is exact; this entry point serves
 *   checkpoints and kernels that can apply only one global scale per GEMM.
 *   scales: device, nvfp4_scale_bytes(rows, cols) bytes, 16-byte aligned (rewritten).
 *   segs/nseg: the modules as weight-row ranges covering [0, rows) in order (1..16).
 *   gs_common_out: device float, must not be one of the segments' gs_w.
 *   Padding bytes are left as they are.  Errors as nvfp4_linear's argument checks.
 */
NVFP4_API nvfp4_status_t nvfp4_fold_segments(uint8_t *scales, int64_t rows, int64_t cols,
                                             const nvfp4_segment_t *segs, int nseg, float *gs_common_out,
                                             nvfp4_stream_t stream);

/*
 * nvfp4_fp8_scale - calibrated per-tensor FP8 scale of a BF16 tensor:
 *   *scale_out = fl32(max|x| / 448) (device), 1 when x is all zero.  The calibration
 *   step of the pages' "ship KV scales" recipe (blog section "KVキャッシュはFP8で十分？":
 *   static FP8 scales for the K and V tensors of every attention layer, computed on
 *   calibration data and shipped with the checkpoint); the formula is this library's
 *   reading.  Arguments and requirements as nvfp4_global_scale.
 */
NVFP4_API nvfp4_status_t nvfp4_fp8_scale(const void *x_bf16, int64_t rows, int64_t cols, int64_t ld,
                                         float *scale_out, nvfp4_stream_t stream);

/*
 * nvfp4_kv_cache_fp8 - write the K and V rows of `tokens` tokens into an FP8 KV cache
 * with static per-tensor scales (same source as nvfp4_fp8_scale):
 *   k_cache[slots[t], c] = E4M3(fl32(k[t, c] * fl32(1 / *k_scale))), likewise V with
 *   *v_scale; nearest even, saturating at +-448, sign kept (a value decodes to
 *   e4m3 * scale).
 *   k, v: device BF16 [tokens x width], row stride ld elements (ld >= width, ld % 8 == 0,
 *   16-byte aligned); width % 16 == 0.  slots: device int64 [tokens]; a negative slot
 *   skips the token; a slot >= num_slots is skipped and reported as
 *   NVFP4_ERR_DEVICE_INDEX by nvfp4_get_device_status.  k_cache, v_cache: device
 *   [num_slots x width] bytes, 16-byte aligned, owned by the caller; rows of other
 *   slots are not touched.
 */
NVFP4_API nvfp4_status_t nvfp4_kv_cache_fp8(const void *k_bf16, const void *v_bf16, int64_t tokens, int64_t width,
                                            int64_t ld, const float *k_scale, const float *v_scale,
                                            const int64_t *slots, uint8_t *k_cache, uint8_t *v_cache,
                                            int64_t num_slots, nvfp4_stream_t stream);

/*
 * nvfp4_gdn_recurrence - the gated delta-rule recurrence of the Gated DeltaNet layers,
 * fed by the gate epilogue of the fused in-projection (NVFP4_EPI_GDN_GATES):
 *   for each sequence s, value head h and token t of the sequence, in order,
 *     S <- exp(g[t,h]) * S + beta[t,h] * k_t (v_t - S^T k_t)^T
 *     out[t, h*128 : h*128+128] = S^T q_t
 *   with k_t, q_t the 128-vectors of key head h / (n_value_heads / n_key_heads) and v_t
 *   that of value head h.  Source: blog section "Gated DeltaNetの仕組み" (the state
 *   update, alpha = forget gate, beta = write strength); alpha = exp(g) follows the log-
 *   space decay the gate epilogue produces (section 機構②).  The read-out S^T q with the
 *   updated state is this library's reading (the pages give none); q and k are used as
 *   given (no normalisation or scaling).  FP32 state.  With 64 or more tokens per
 *   sequence on average the recurrence runs in its chunked form (64-token chunks, the
 *   same algebra) with the products on the tensor cores: BF16 q and k, the FP32
 *   operands split into two BF16 parts, FP32 accumulation, an FP32 triangular solve;
 *   there g below -80 counts as -80 (a decay below 2e-35).  Otherwise token by token in
 *   FP32.  Both agree with the exact recurrence within 1e-4 of the output scale.
 *   q, k: device BF16 rows [tokens x ld_qk] (key head hk at column hk*128); v: device
 *   BF16 [tokens x ld_v] (value head h at column h*128); q, k, v 16-byte aligned, ld_qk
 *   and ld_v multiples of 8.  They may be column ranges of one projection output.
 *   g, beta: device FP32 [tokens x ld_gate], head h at column h (the layout the gate
 *   epilogue writes).  cu_seqlens: device int32 [n_seqs + 1], sequence s = tokens
 *   cu_seqlens[s] .. cu_seqlens[s+1]-1 (empty sequences allowed); a sequence whose
 *   bounds are not 0 <= start <= end <= tokens is skipped (state and out untouched) and
 *   reported as NVFP4_ERR_DEVICE_INDEX by nvfp4_get_device_status.
 *   state: device FP32 [n_seqs][n_value_heads][128][128], 16-byte aligned: entry
 *   [s][h][j][i] holds S[i][j] (i over d_k, j over d_v).  Read as the initial state when
 *   initial_state != 0 (else S starts at 0), overwritten with the final state.
 *   out: device [tokens x ld_out] of out_kind NVFP4_OUT_BF16 (ld_out % 8 == 0) or
 *   NVFP4_OUT_F32 (ld_out % 4 == 0), 16-byte aligned.  head_dim must be 128;
 *   n_value_heads a multiple of n_key_heads; n_seqs, n_value_heads <= 65535.
 *   Buffers must not overlap except q, k and v (read only).
 */
NVFP4_API nvfp4_status_t nvfp4_gdn_recurrence(const void *q_bf16, const void *k_bf16, int64_t ld_qk,
                                              const void *v_bf16, int64_t ld_v, const float *g, const float *beta,
                                              int64_t ld_gate, const int32_t *cu_seqlens, int64_t n_seqs,
                                              int64_t tokens, int n_key_heads, int n_value_heads, int head_dim,
                                              float *state, int initial_state, void *out, int64_t ld_out,
                                              int out_kind, nvfp4_stream_t stream);

/*
 * nvfp4_get_device_status - read and clear the device status word of the current
 * device.  Kernels never spin forever: every wait on an mbarrier has an iteration
 * limit, and a wait that runs out records NVFP4_ERR_DEVICE_TIMEOUT here and the
 * kernel returns.  *code receives NVFP4_OK (0) when nothing was recorded.
 * Synchronises the device.
 */
NVFP4_API nvfp4_status_t nvfp4_get_device_status(int *code);

/*
 * nvfp4_selftest_stalled_linear - failure-detection self-test of the bounded waits.
 * The pages have no counterpart; it checks the library's own guarantee that a kernel
 * whose pipeline stops never hangs the GPU.  It runs the 1-CTA GEMM of nvfp4_linear
 * (epilogue NVFP4_EPI_NONE, FP32 output) with one pipeline stage never loaded: the
 * producer skips stage `stall_stage` (counted from 0 over the K tiles), so the scale
 * copiers and the MMA issuer wait on a barrier phase that never completes, and the
 * epilogue waits on an accumulator that is never committed.  In this instantiation
 * every wait gives up after a short limit (1 ms instead of the product's 0.5 s):
 * each role records NVFP4_ERR_DEVICE_TIMEOUT in the device status word, waits
 * for the work it already issued, TMEM is freed and the kernel returns.  The output
 * is left partly written and is meaningless.  The context stays usable: read and
 * clear the status with nvfp4_get_device_status, after which the other entry points
 * run as before.
 *   Arguments as nvfp4_linear with one output tile: A->rows <= 128, W->rows <= 256,
 *   out FP32 [A->rows x ldo] (device, 16-byte aligned), 0 <= stall_stage < K / 256.
 *   Errors: NVFP4_ERR_UNSUPPORTED_SHAPE for more than one tile, NVFP4_ERR_INVALID_ARG
 *   for a stall_stage outside the K tiles, otherwise as nvfp4_linear's checks.
 *   The call itself returns NVFP4_OK when the launch succeeded; the timeout shows only
 *   in the status word.
 */
NVFP4_API nvfp4_status_t nvfp4_selftest_stalled_linear(const nvfp4_operand_t *A, const float *gs_a,
                                                       const nvfp4_operand_t *W, const nvfp4_segment_t *segs,
                                                       int nseg, float *out, int64_t ldo, int stall_stage,
                                                       nvfp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_W4A4_H */
