/*
 * fp8q.h - C ABI of the B200 (sm_100a) library for online fine-grained quantization and
 * block-scaled low-precision GEMM.
 *
 * Sources of the operations (pages cited by title and section):
 *   [DSV3]  "Can you explain the role of FP8 precision in DeepSeek-V3 training":
 *           "Fine-grained quantization" (1x128 activation tiles, 128x128 weight blocks,
 *           one scale each), "Online quantization" (scales from the live amax),
 *           "Increased accumulation precision" (partial sums promoted to FP32 at fixed
 *           intervals), "Unified E4M3 format" (E4M3 for all tensors), "Mixed-precision
 *           framework" (the compute-heavy GEMMs in FP8).
 *   [NeMo]  "Accelerating FP8 training performance with the NVIDIA NeMo framework":
 *           per-tensor and MXFP8 (blocks of 32 values) scaling recipes.
 *   [NVFP4] "NVIDIA developed a method to train neural networks in 4-bit precision",
 *           "How it works": 4-bit values, 16x16 random Hadamard transforms on gradient
 *           inputs, stochastic rounding.
 *
 * Conventions for every call:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never frees
 *     or keeps them.  BF16 inputs are raw bit patterns (uint16).  Matrices are row-major.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Every
 *     call is asynchronous on that stream: it validates its arguments on the host,
 *     enqueues its kernels and returns.
 *   - The return value reports host-side validation and launch only.  A kernel that gives
 *     up (a bounded wait that ran out) records a code in a per-device status word that
 *     fp8q_get_device_status() reads; faults surface as CUDA errors on the next sync.
 *   - Inputs are assumed finite; NaN/Inf inputs give unspecified codes but never fault.
 *   - The library allocates no device memory for tensors.  Calls that need a global amax
 *     (per-tensor and NVFP4 quantization) and the status word use a small per-device
 *     scratch pool the library allocates on first use and keeps until
 *     fp8q_release_scratch() or process exit.
 *
 * Quantization rules (the readings the pages leave open, shared by the CPU oracle):
 *   E4M3 is OCP "E4M3FN" (max 448), encoded round-to-nearest-even with saturation.
 *   1x128 / 128x128 / per-tensor: sf = 448 / amax (FP32 IEEE division; amax == 0 -> 1;
 *   overflow -> FLT_MAX), codes = E4M3(fp32(x * sf)), stored decode scale = 1 / sf.
 */
#ifndef FP8Q_H
#define FP8Q_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FP8Q_OK = 0,
  FP8Q_ERR_NULL = 1,        /* a required pointer is NULL                            */
  FP8Q_ERR_SHAPE = 2,       /* a size, stride or block-multiple requirement fails     */
  FP8Q_ERR_ALIGN = 3,       /* a pointer or leading dimension is not 16-byte aligned  */
  FP8Q_ERR_UNSUPPORTED = 4, /* valid request this build does not implement            */
  FP8Q_ERR_CUDA = 5,        /* a CUDA runtime/driver call or kernel launch failed     */
  FP8Q_ERR_TIMEOUT = 6,     /* (device status) a bounded wait inside a kernel ran out */
  FP8Q_ERR_DEVICE_ARG = 7   /* (device status) an argument read on the device was out of
                               range (grouped GEMM offsets); the kernel clamped it        */
} fp8q_status;

/* Byte layout of MX (E8M0) and NVFP4 (E4M3) scale factors. */
typedef enum {
  FP8Q_SF_ROWMAJOR = 0,  /* sf[r * n_sf_cols + c]                                     */
  FP8Q_SF_MMA_TILED = 1  /* per 128 rows x 4 scale columns, 512 contiguous bytes:
                            offset = ((r/128) * ceil(n_sf_cols/4) + c/4) * 512
                                     + (r%32) * 16 + ((r%128)/32) * 4 + c%4;
                            rows padded to 128 and scale columns to 4, padding bytes 0.
                            This is the image the block-scaled tensor-core MMA reads
                            into tensor memory; the MX and NVFP4 GEMMs require it.       */
} fp8q_sf_layout;

typedef enum {
  FP8Q_BLOCKWISE = 0,  /* [DSV3] 1x128 x 128x128 (or 1x128 x 1x128) FP32 scales, E4M3 */
  FP8Q_MXFP8 = 1,      /* [NeMo] E4M3 with E8M0 scales per 32 along K                  */
  FP8Q_PERTENSOR = 2,  /* [NeMo] E4M3 with one FP32 decode scale per operand           */
  FP8Q_NVFP4 = 3       /* [NVFP4] E2M1, E4M3 scales per 16 along K, FP32 tensor scale  */
} fp8q_recipe;

/* Selects how the blockwise B scales are indexed (the A scales are always 1x128). */
typedef enum {
  FP8Q_FPROP = 0,  /* B = W^T (N x K codes); sb[(n/128) * ld_sb + k/128]  (128x128)    */
  FP8Q_DGRAD = 1,  /* B = W   (N x K codes); sb[(k/128) * ld_sb + n/128]  (128x128)    */
  FP8Q_WGRAD = 2   /* B = dY^T (N x K codes, K = tokens); sb[(k/128) * ld_sb + n] (1x128)*/
} fp8q_layout;

/* FP8 element format of a per-tensor operand (OCP 8-bit floating point). */
typedef enum {
  FP8Q_E4M3 = 0,  /* max 448, the format of every other call                            */
  FP8Q_E5M2 = 1   /* max 57344, the gradient format of the delayed-scaling comparison  */
} fp8q_fp8_format;

/* NVFP4 per-direction flags for `rht` and `sr`. */
#define FP4Q_ROW 1  /* apply to the rowwise output (quantized along columns)           */
#define FP4Q_COL 2  /* apply to the colwise output (quantized along rows, transposed)  */

/* [DSV3] "Fine-grained quantization", "Online quantization": 1x128 tiles.
 * x: BF16 rows x cols, row stride ld_x elements (ld_x % 8 == 0, x 16-byte aligned).
 * Rowwise (needs cols % 128 == 0; any rows >= 0): one scale per 128 consecutive
 *   elements of a row -> q_row[r * cols + c] (E4M3, contiguous rows x cols) and
 *   s_row[(c/128) * ld_s_row + r] (FP32 decode scales, MN-major, ld_s_row >= rows,
 *   ld_s_row % 4 == 0).
 * Colwise (needs rows % 128 == 0; cols % 16 == 0): one scale per 128 consecutive
 *   elements of a column, output transposed: q_col[c * rows + r] (cols x rows,
 *   K-major in the row index: the wgrad operands) and s_col[(r/128) * ld_s_col + c]
 *   (ld_s_col >= cols, % 4 == 0).
 * Either output pair may be NULL (not produced); both NULL is FP8Q_ERR_NULL.
 * x is read once for both outputs.  rows == 0 or cols == 0 -> FP8Q_OK, nothing launched. */
fp8q_status fp8q_quantize_1x128(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                uint8_t* q_row, float* s_row, int64_t ld_s_row,
                                uint8_t* q_col, float* s_col, int64_t ld_s_col,
                                void* stream);

/* [DSV3] "Fine-grained quantization": 128x128 weight blocks.
 * w: BF16 K x N (K % 128 == 0, N % 128 == 0), row stride ld_w (% 8 == 0).
 * q_t: N x K codes (the FPROP B operand); q: K x N codes (the DGRAD B operand); the two
 * hold the same codes transposed; either may be NULL.  s: FP32 decode scales
 * [N/128][K/128] (s[(n/128) * (K/128) + k/128]), required. */
fp8q_status fp8q_quantize_128x128(const void* w, int64_t K, int64_t N, int64_t ld_w,
                                  uint8_t* q_t, uint8_t* q, float* s, void* stream);

/* [DSV3] "Fine-grained quantization" for a stack of weight matrices (the experts of a MoE
 * layer), in one launch: groups matrices w[g] = w + g * K * ld_w, each BF16 K x N with row
 * stride ld_w, quantized exactly as fp8q_quantize_128x128 quantizes one.  Outputs are
 * contiguous per matrix: q_t[g] = q_t + g * N * K (N x K codes, the grouped GEMM's B
 * operand), q[g] = q + g * K * N, s[g] = s + g * (N/128) * (K/128).  Same requirements as
 * fp8q_quantize_128x128; groups == 0 -> FP8Q_OK, nothing launched. */
fp8q_status fp8q_quantize_128x128_grouped(const void* w, int64_t groups, int64_t K, int64_t N, int64_t ld_w,
                                          uint8_t* q_t, uint8_t* q, float* s, void* stream);

/* [DSV3] "Fine-grained quantization", "Online quantization": several tensors in one launch.
 * Each item is one fp8q_quantize_1x128 call (kind FP8Q_ITEM_1X128: x is rows x cols, the
 * q_row / s_row / ld_s_row and q_col / s_col / ld_s_col outputs) or one
 * fp8q_quantize_128x128 call (kind FP8Q_ITEM_128X128: x is K x N with K = rows, N = cols,
 * outputs q_t, q and s), with exactly that call's requirements, layouts and results; the
 * fields of the other kind are ignored.  For 128x128 at least one of q_t and q is required.
 * Up to FP8Q_MAX_QUANT_ITEMS items; every item is validated before anything is launched
 * (the first failing item's status is returned and nothing runs).  One kernel quantizes
 * all items' 128x128 tiles, so the GPU is filled across tensors and the call pays one launch
 * and one partial last wave.  Items must not overlap each other's outputs.  Items with no
 * elements are skipped; n_items == 0 -> FP8Q_OK, nothing launched. */
#define FP8Q_MAX_QUANT_ITEMS 8
typedef enum { FP8Q_ITEM_1X128 = 0, FP8Q_ITEM_128X128 = 1 } fp8q_item_kind;
typedef struct fp8q_quant_item {
  int32_t kind;                   /* fp8q_item_kind */
  const void* x;                  /* BF16 input */
  int64_t rows, cols, ld_x;
  uint8_t* q_row;                 /* FP8Q_ITEM_1X128 outputs */
  float* s_row;
  int64_t ld_s_row;
  uint8_t* q_col;
  float* s_col;
  int64_t ld_s_col;
  uint8_t* q_t;                   /* FP8Q_ITEM_128X128 outputs */
  uint8_t* q;
  float* s;
} fp8q_quant_item;
fp8q_status fp8q_quantize_multi(const fp8q_quant_item* items, int32_t n_items, void* stream);

/* [NeMo] MXFP8: 32-element blocks, E8M0 scale = smallest e with amax <= 448 * 2^e
 * (amax == 0 -> e = -127; e clamped to [-127, 127]; byte e + 127), codes
 * E4M3(fp32(x * 2^-e)).
 * Rowwise (cols % 32 == 0): q_row rows x cols, e8m0_row for (rows, cols/32).
 * Colwise (rows % 32 == 0, cols % 16 == 0): transposed q_col cols x rows, e8m0_col for
 *   (cols, rows/32).
 * Scale bytes use `sf_layout`; size buffers with fp8q_sf_bytes(FP8Q_MXFP8, outer, inner,
 * layout) (outer = rows of the code matrix, inner = its columns).  Either pair may be NULL. */
fp8q_status fp8q_quantize_mx32(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                               uint8_t* q_row, uint8_t* e8m0_row,
                               uint8_t* q_col, uint8_t* e8m0_col,
                               fp8q_sf_layout sf_layout, void* stream);

/* [NeMo] per-tensor current scaling: amax of the whole tensor, then codes
 * q[r * cols + c] and one FP32 decode scale *s_dec (device).  cols % 8 == 0.
 * Two kernels (amax, cast) on `stream`; the amax lives in the library's scratch pool. */
fp8q_status fp8q_quantize_tensor(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                 uint8_t* q, float* s_dec, void* stream);

/* Per-tensor DELAYED scaling, the recipe [DSV3] "Online quantization" contrasts with its
 * own: the scale comes from the amaxes of earlier iterations instead of the tensor being
 * cast, so one pass over x both casts and measures.
 *   amax_history: device float[history_len] (1 <= history_len <= 1024), non-negative;
 *   sf = fmt_max / max(amax_history) (FP32 IEEE division; max 0 -> 1; overflow -> FLT_MAX),
 *   fmt_max = 448 (FP8Q_E4M3) or 57344 (FP8Q_E5M2); codes q[r * cols + c] =
 *   fmt(x * sf) rounded to nearest even and saturated (values beyond the historical range
 *   clip); *s_dec = fp32(1 / sf).  After the cast this tensor's amax is written to
 *   amax_history[history_pos] (0 <= history_pos < history_len; the caller rotates it),
 *   so it takes effect from the next call.  cols % 8 == 0. */
fp8q_status fp8q_quantize_tensor_delayed(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                         float* amax_history, int32_t history_len, int32_t history_pos,
                                         fp8q_fp8_format fmt, uint8_t* q, float* s_dec, void* stream);

/* Allocation-free variant of fp8q_quantize_tensor (no counterpart in the pages: it is a
 * library-integration entry point, not part of the method).  Same arguments, rules and
 * results as fp8q_quantize_tensor.
 * Who needs it: callers that cannot let a library allocate device memory - for example an
 * application whose allocator owns all device memory and forbids foreign cudaMalloc calls,
 * or one that runs under a fixed memory budget where a lazy allocation on first use could
 * fail at an arbitrary point (and cudaMalloc/cudaFree may synchronize the device).
 * fp8q_quantize_tensor allocates the library's scratch pool on its first call per device;
 * this entry point calls no cudaMalloc, cudaFree or allocating library routine.  Its
 * scratch is a fixed 256-byte array (64 words) in the library's device globals, present on
 * every GPU that loads the library until the process exits; one call needs 1 word (the
 * running amax), and a request needing more than the array holds is rejected with
 * FP8Q_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress,
 * with that device current); make that first call before any stream capture.
 * Every call shares the array and it keeps the last call's contents: each call clears the
 * amax word on `stream` before using it.  Calls that overlap on the GPU (different streams
 * without ordering, or different host threads) race on the array and may return wrong
 * scales; serialize them. */
fp8q_status fp8q_quantize_tensor_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                         uint8_t* q, float* s_dec, void* stream);

/* [NVFP4] 4-bit quantization with optional 16x16 random Hadamard transform and
 * stochastic rounding.
 *   G = amax of the (transformed) tensor; S_g = 2688 / G (G == 0 -> 1);
 *   per 16 elements along the quantized dim: sb = E4M3(fp32(amax_b / 6) * S_g),
 *   enc = S_g / decode(sb) (0 if sb == 0), y = x * enc, q = E2M1(y) by
 *   round-to-nearest-even or stochastic rounding; stored g_dec = 1 / S_g.
 *   RHT (per direction in `rht`, FP4Q_ROW / FP4Q_COL): 16 signs from Philox4x32-10
 *   (counter (0,0,0,0x52485431), key rht_seed, word 0 bits 0..15, 1 -> -1); each group of
 *   16 along the quantized dim is sign-flipped, passed through the butterflies h = 1, 2,
 *   4, 8 in FP32 and scaled by 1/4.
 *   SR (per direction in `sr`): random word = Philox4x32-10 output word (idx & 3) for
 *   counter (idx>>2 low, idx>>2 high, 0, tag), key sr_seed; idx = linear index of the
 *   element in that output; tag 0 rowwise, 1 colwise; u = (word >> 8) * 2^-24; round up
 *   iff u < (|y| - lo) / (hi - lo).
 * Rowwise (cols % 16 == 0): q_row rows x cols/2 bytes (even element in the low nibble),
 *   sf_row scale bytes for (rows, cols/16), *g_dec_row.
 * Colwise (rows % 16 == 0, cols % 16 == 0): transposed, q_col cols x rows/2, sf_col for
 *   (cols, rows/16), *g_dec_col.
 * Either triple may be NULL.  Two passes over x (global amax, then quantize). */
fp8q_status fp4q_rht16_quantize_sr(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                   int rht, uint64_t rht_seed, int sr, uint64_t sr_seed,
                                   uint8_t* q_row, uint8_t* sf_row, float* g_dec_row,
                                   uint8_t* q_col, uint8_t* sf_col, float* g_dec_col,
                                   fp8q_sf_layout sf_layout, void* stream);

/* NVFP4 weights with one E4M3 scale per 16x16 block, in both GEMM operand layouts, so that
 * the forward GEMM (weights read along one axis) and the backward-data GEMM (along the
 * other) use one quantized matrix.  The [NVFP4] page ("How it works") fixes the 4-bit
 * values, the per-16 E4M3 scales and the per-tensor FP32 scale; the 16x16 block shape of a
 * weight scale is this library's reading for that two-layout use.
 *   G = amax |x| over the tensor; S_g = 2688 / G (G == 0 -> 1);
 *   per 16x16 block: sb = E4M3(fp32(amax_b / 6) * S_g) over its 256 elements,
 *   enc = S_g / decode(sb) (0 if sb == 0), q = E2M1_RNE(x * enc); *g_dec = 1 / S_g.
 *   No transform and no stochastic rounding (weights, not gradient inputs).
 * x: BF16 rows x cols, row stride ld_x elements (ld_x % 8 == 0), 16-byte aligned;
 *   rows % 16 == 0 and cols % 16 == 0.
 * Rowwise (q_row, sf_row): q_row rows x cols/2 bytes (even element in the low nibble),
 *   sf_row scale bytes for (rows, cols/16), each block's code repeated over its 16 rows.
 * Colwise (q_col, sf_col): the same codes transposed, q_col cols x rows/2, sf_col for
 *   (cols, rows/16).  Either pair may be NULL, not both; g_dec (device float) is required.
 * Scale bytes in sf_layout (FP8Q_SF_MMA_TILED for the NVFP4 GEMM; padding bytes 0).
 * Two passes over x (global amax, then quantize); asynchronous on `stream`.
 * Errors: FP8Q_ERR_NULL, FP8Q_ERR_SHAPE, FP8Q_ERR_ALIGN (q pointers 16-byte aligned),
 *   FP8Q_ERR_UNSUPPORTED (sf_layout), FP8Q_ERR_CUDA. */
fp8q_status fp4q_quantize_2d16(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                               uint8_t* q_row, uint8_t* sf_row, uint8_t* q_col, uint8_t* sf_col,
                               float* g_dec, fp8q_sf_layout sf_layout, void* stream);

/* Arguments of fp8q_gemm_blockscaled: C[M x N] = A[M x K] . B[N x K]^T, both operands
 * K-major codes, C BF16 row-major (ldc >= N, ldc % 8 == 0, c 16-byte aligned) unless
 * c_fp32_accumulate is set (below).
 *   BLOCKWISE [DSV3] "Increased accumulation precision": for every 128-element K chunk the
 *     tensor cores form the E4M3 partial product in FP32 and CUDA cores add it into an
 *     FP32 accumulator with the chunk's scales applied:
 *       C[m,n] = bf16( sum_kb sa[kb * ld_sa + m] * sb(kb, n) * partial_kb[m,n] ),
 *     sb by `layout`.  K % 128 == 0.  a_scale/b_scale are float*.
 *   MXFP8: codes E4M3, scales E8M0 in FP8Q_SF_MMA_TILED layout for (M, K/32) and
 *     (N, K/32), applied by the hardware.  K % 128 == 0.
 *   PERTENSOR: codes E4M3, or E5M2 per operand (a_format / b_format, e.g. an E5M2
 *     gradient times E4M3 weights in dgrad); C = (*a_global) * (*b_global) * (A . B^T).
 *     K % 128 == 0.
 *   NVFP4: packed E2M1 (lda/ldb in BYTES, K/2 bytes per row), E4M3 scales in
 *     FP8Q_SF_MMA_TILED layout for (M, K/16) and (N, K/16), C scaled by
 *     (*a_global) * (*b_global).  K % 256 == 0.
 *   The K rules come from the kernels' pipeline: every stage moves 128 bytes of K per row
 *   (128 FP8 or 256 FP4 values) and there is no partial last stage; a K that breaks the
 *   rule returns FP8Q_ERR_SHAPE.  K == 0 is allowed (C = 0, or unchanged when
 *   accumulating).
 * lda/ldb: row strides in bytes (% 16 == 0).  a/b 16-byte aligned.
 * Grouped (MoE, BLOCKWISE/FPROP only) when num_groups > 0: m_offsets[0..G] (device int32,
 *   non-decreasing, m_offsets[0] == 0, m_offsets[G] == M) delimit each expert's rows of A
 *   and C; B is [G][N][K] (expert g at b + g * N * ldb) and b_scale [G][N/128][K/128]
 *   (expert g at g * (N/128) * ld_sb floats).  The kernel reads the offsets on the device
 *   and builds its tile schedule there (at most M/128 + G row tiles), so the host needs
 *   no copy of them.  Offsets that break the rule are clamped on the device to
 *   [previous offset, M] (no row outside C is ever written) and the device status word
 *   records FP8Q_ERR_DEVICE_ARG (read it with fp8q_get_device_status).
 * M, N >= 0 arbitrary (tails masked at the store).
 * c_fp32_accumulate (BLOCKWISE only; 0 for the other recipes): C is an FP32 row-major
 *   matrix (ldc % 4 == 0, c 16-byte aligned) that is updated in place,
 *     C[m,n] = fp32( C[m,n] + sum_kb ... )   (the FP32 sum above, before any BF16 rounding),
 *   the FP32 main-gradient accumulation that follows wgrad in training ([DSV3]
 *   "Mixed-precision framework": gradients and master weights stay in FP32).  K == 0
 *   leaves C unchanged.
 * q_out / s_out (BLOCKWISE with BF16 output, not grouped; both NULL otherwise): the GEMM
 *   also quantizes its BF16 output C in 1x128 tiles along N, as fp8q_quantize_1x128's
 *   rowwise output would from C ([DSV3] "Online quantization": the next layer's activation
 *   is quantized from its live amax), without a second pass over C:
 *     q_out[m * ld_q_out + n] = E4M3 codes (M x N bytes, ld_q_out >= N, % 16 == 0,
 *     q_out 16-byte aligned), s_out[(n / 128) * ld_s_out + m] = FP32 decode scales
 *     (ld_s_out >= M).  Needs N % 128 == 0 and K >= 384 (else FP8Q_ERR_SHAPE). */
typedef struct {
  fp8q_recipe recipe;
  fp8q_layout layout;
  int64_t M, N, K;
  const void* a;
  const void* a_scale;
  int64_t lda, ld_sa;
  const void* b;
  const void* b_scale;
  int64_t ldb, ld_sb;
  const float* a_global;
  const float* b_global;
  void* c;
  int64_t ldc;
  const int32_t* m_offsets;
  int32_t num_groups;
  int32_t c_fp32_accumulate;
  int32_t a_format, b_format;   /* fp8q_fp8_format of A / B codes (PERTENSOR; else 0) */
  uint8_t* q_out;               /* optional fused 1x128 quantization of C (see above) */
  float* s_out;
  int64_t ld_q_out, ld_s_out;
  void* workspace;              /* optional: split of the last wave (see fp8q_gemm_workspace_bytes) */
  int64_t workspace_bytes;
} fp8q_gemm_args;

fp8q_status fp8q_gemm_blockscaled(const fp8q_gemm_args* args, void* stream);

/* Workspace bytes that fp8q_gemm_blockscaled can use for `args` on the current device; 0 when
 * the call would use none.  Only BLOCKWISE GEMMs (BF16 output or FP32 accumulation), not
 * grouped and without the fused quantization, use one.  Their kernel keeps one CTA pair per
 * two SMs and walks the 256 x 256 output tiles wave by wave.  When the last wave would leave
 * more than half of the pairs idle for a whole tile and the cut saves at least 16 of its
 * chunks of 128, its tiles are cut into K ranges of at least 4 chunks (one range per pair at
 * most), run after the whole tiles in the same launch, each storing its FP32 partial sum (the
 * same promoted sum, over the range's chunks only) into the workspace; a second small launch
 * adds the ranges in order in FP32 and rounds the sum to BF16 into C (with
 * c_fp32_accumulate: adds it into C, still one addition per element).  The result is the same
 * FP32 sum, grouped by ranges, so it can differ from the unsplit schedule's by FP32 rounding,
 * and it is the same on every run.  workspace (device memory, 16-byte aligned, or NULL) with
 * workspace_bytes: a NULL workspace, fewer bytes than this function returns, or any other
 * kind of GEMM keeps the unsplit schedule (no error).  The library only uses the workspace in
 * kernels enqueued on the call's stream; the caller must not use it concurrently elsewhere
 * before they complete.  Returns 0 for NULL or invalid arguments. */
size_t fp8q_gemm_workspace_bytes(const fp8q_gemm_args* args);

/* Bytes of a scale-factor buffer: recipe MXFP8 (inner/32 scale columns) or NVFP4
 * (inner/16), `outer` rows, in `layout`.  Returns 0 for other recipes. */
size_t fp8q_sf_bytes(fp8q_recipe recipe, int64_t outer, int64_t inner, fp8q_sf_layout layout);

/* Synchronizes `stream`, returns and clears the current device's status word
 * (FP8Q_OK, or FP8Q_ERR_TIMEOUT if a kernel's bounded wait ran out since the last call). */
fp8q_status fp8q_get_device_status(void* stream);

/* Failure-detection self test (not part of the pages' method).  Launches one warp whose
 * first thread waits, with the same bounded mbarrier wait the GEMM kernels use, on a
 * shared-memory barrier that nothing ever arrives on.  After `limit_ns` nanoseconds of
 * wall time (1e3 .. 1e9) the wait gives up and records FP8Q_ERR_TIMEOUT in the device
 * status word, exactly as a GEMM role does before it winds down; the kernel then exits
 * with no copy or MMA in flight and the context stays usable.  Returns the launch status
 * (FP8Q_ERR_SHAPE for a limit out of range); read the outcome with
 * fp8q_get_device_status(). */
fp8q_status fp8q_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* Frees the current device's scratch pool (after a device sync).  Optional.  Must not
 * overlap any other fp8q call on that device (from another host thread): a call that
 * already holds the pool's address would use freed memory. */
fp8q_status fp8q_release_scratch(void);

const char* fp8q_status_string(fp8q_status s);

/* Library version, e.g. "fp8q 0.1.0 sm_100a". */
const char* fp8q_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8Q_H */
