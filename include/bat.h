/*
 * bat.h — C-ABI of the BATQuant W4A4 (MXFP4) linear layer for NVIDIA B200 (sm_100a).
 *
 * The operation (BATQuant note, en.papernotes.org, "Method > Key Designs 1-3";
 * nubint.ai review, "proposed method"):
 *
 *   Y = Q(X P) . Q(P^-1 W^T)
 *
 * X is M x K bf16 (tokens x in-features), W is N x K bf16 (out x in), P is
 * block-diagonal with one 32 x 32 block per 32-channel MXFP4 block b, and each
 * block is the Global-and-Private Kronecker product P_b = B_b (x) A: A is one
 * 8 x 8 factor shared by every block, B_b a private 4 x 4 factor. A block x of
 * 32 values read as the row-major 4 x 8 matrix X_r[i][p] = x[8i+p] maps to
 * y = x P_b = vec_row(B_b^T X_r A). Q is block-wise learnable clipping to
 * [sigma(g_lo_b) * min(y), sigma(g_hi_b) * max(y)] followed by MXFP4
 * quantization: E2M1 codes (grid 0, .5, 1, 1.5, 2, 3, 4, 6 and negatives),
 * one UE8M0 scale 2^e per 32 elements with e = floor(log2 amax) - 2,
 * round-to-nearest-even, saturating at +-6 ("Background & Motivation").
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller. The online entry
 *     points never allocate device memory; the offline bat_prepare_weight(_gpk)
 *     allocates (and frees, stream-ordered) one temporary of about
 *     4*s*s + 4*K*32/s bytes for the inverted factors. No state is kept between
 *     calls except a sticky device error word (see bat_device_error) and, per
 *     device, cached launch facts (kernel attributes set, how many clusters of a
 *     given size fit), which do not change results.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Calls are
 *     asynchronous on it unless stated otherwise.
 *   - Arguments are validated on the host before any CUDA call; a bad argument
 *     returns an error status and launches nothing. CUDA failures return
 *     BAT_ERR_CUDA. The device must be sm_100 (B200); other devices get
 *     BAT_ERR_UNSUPPORTED.
 *   - Calls are thread-safe (the per-device caches are atomics written with
 *     idempotent values).
 *   - Row limit: every operand has at most 2^30 rows (activations M, weights N,
 *     KV tokens x heads, cache slots x heads); more returns BAT_ERR_SHAPE. The
 *     tensor-memory copies address a tile by 32-bit signed coordinates.
 *   - Shapes and routing: activation batches of at most 64 rows are quantized on
 *     the CUDA cores, larger ones by the tensor-core prologue (the codes of one
 *     path are exact with respect to its own fp32 transformed values; the two
 *     paths' transformed values differ by fp32 rounding). A GEMM with one row of
 *     128-row tiles that leaves most SMs idle runs split-K over thread-block
 *     clusters, with a fixed summation order.
 *
 * Storage formats (bat_mxfp4_t):
 *   codes : [rows][k/2] bytes, row-major, two E2M1 codes per byte, element 2i in
 *           the low nibble and 2i+1 in the high nibble; sign in bit 3 of a code.
 *   scales: UE8M0 bytes (value 2^(byte-127)) in a tiled order the GEMM reads
 *           directly: rows padded to a multiple of 128, blocks (k/32) padded to a
 *           multiple of 4; the byte of (row m, block b) sits at
 *             ((m/128)*nbp4 + b/4)*512 + (m%32)*16 + ((m%128)/32)*4 + b%4,
 *           nbp4 = ceil((k/32)/4). Padding bytes are written as 0.
 */
#ifndef BAT_H_
#define BAT_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BAT_API __attribute__((visibility("default")))
#else
#define BAT_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BAT_OK = 0,
  BAT_ERR_INVALID_ARG = 1, /* null pointer, negative or zero size, bad enum */
  BAT_ERR_SHAPE = 2,       /* k % 32 != 0, operand shapes disagree, size over a limit */
  BAT_ERR_ALIGN = 3,       /* a pointer is not 16-byte aligned */
  BAT_ERR_SINGULAR = 4,    /* A or some B_b is singular or ill-conditioned */
  BAT_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  BAT_ERR_UNSUPPORTED = 6, /* device is not sm_100, or a feature outside this build */
  BAT_ERR_WORKSPACE = 7,   /* workspace pointer null or smaller than required */
  BAT_ERR_DEVICE = 8       /* a kernel reported a failure through the device error word */
} bat_status_t;

typedef enum { BAT_OUT_BF16 = 0, BAT_OUT_F32 = 1 } bat_out_dtype_t;

/* An MXFP4 matrix with `rows` rows of `k` elements; buffers owned by the caller. */
typedef struct {
  void* codes;  /* device, bat_mxfp4_codes_bytes(rows, k) bytes, 16-byte aligned */
  void* scales; /* device, bat_mxfp4_scales_bytes(rows, k) bytes, 16-byte aligned */
  int64_t rows;
  int64_t k;
} bat_mxfp4_t;

/*
 * An MXFP8 matrix (the W4A8 activations): the same struct, with
 *   codes : [rows][k] bytes, row-major, one OCP E4M3 code per element (sign in
 *           bit 7; largest finite 448, no infinities);
 *   scales: the tiled UE8M0 layout of bat_mxfp4_t (bat_mxfp4_scales_bytes).
 */
typedef bat_mxfp4_t bat_mxfp8_t;

/* Sizes of the two buffers of an MXFP4 matrix (0 if k % 32 != 0 or a size < 1). */
BAT_API size_t bat_mxfp4_codes_bytes(int64_t rows, int64_t k);
BAT_API size_t bat_mxfp4_scales_bytes(int64_t rows, int64_t k);

/* Human-readable name of a status code (static storage; "BAT_ERR_UNKNOWN" for a
 * value that is not a status). */
BAT_API const char* bat_status_string(bat_status_t status);

/* Library version, major*10000 + minor*100 + patch. */
BAT_API int bat_version(void);

/*
 * Online activation path: block transform, block clip, MXFP4 quantize + pack.
 * (Key Designs 2 "GPK decomposition" and 3 "Block-wise learnable clipping";
 * Method > "Overall Architecture": activation-side transforms run online.)
 *
 *   X     : bf16 [M][K] row-major, 16-byte aligned.
 *   A     : fp32 [8][8] row-major (shared factor).
 *   B     : fp32 [K/32][4][4] row-major (private factors, one per block).
 *   g_lo, g_hi : fp32 [K/32] clip logits, or both NULL for no clipping.
 *                Ratios are sigma(g) evaluated in fp64 and rounded to fp32;
 *                g = +inf gives ratio 1.
 *   Xq    : output; Xq->rows must equal M and Xq->k must equal K.
 * Requirements: 1 <= M <= 2^30, K >= 32, K % 32 == 0, K <= 262144.
 * Errors: BAT_ERR_INVALID_ARG (a NULL pointer, only one of g_lo/g_hi, M < 1 or
 * K < 32), BAT_ERR_SHAPE (K % 32, K or M over its limit, Xq's rows/k not M/K),
 * BAT_ERR_ALIGN (X, A, B, Xq->codes or Xq->scales not 16-byte aligned),
 * BAT_ERR_UNSUPPORTED (not an sm_100 device), BAT_ERR_CUDA (launch failure);
 * nothing is launched on an argument error.
 */
BAT_API bat_status_t bat_quantize_act(const void* X, int64_t M, int64_t K, const float* A, const float* B,
                              const float* g_lo, const float* g_hi, const bat_mxfp4_t* Xq,
                              void* stream);

/*
 * Same as bat_quantize_act, and also writes the fp32 transformed values y
 * (before clipping) to `y_out` (device fp32 [M][K]). For testing and
 * inspection; slower because of the extra 4 bytes per element.
 * Errors: as bat_quantize_act; also BAT_ERR_INVALID_ARG for a NULL y_out and
 * BAT_ERR_ALIGN for a y_out that is not 16-byte aligned.
 */
BAT_API bat_status_t bat_quantize_act_trace(const void* X, int64_t M, int64_t K, const float* A,
                                    const float* B, const float* g_lo, const float* g_hi,
                                    const bat_mxfp4_t* Xq, float* y_out, void* stream);

/*
 * The clip ratios the prologue uses: r[t] = fp32(1 / (1 + exp(-g[t]))) computed
 * in fp64 on the device (g = +inf gives 1; g == NULL gives all ones).
 * g, r: device fp32 [n].
 * Errors: BAT_ERR_INVALID_ARG (n < 1 or r NULL), BAT_ERR_UNSUPPORTED,
 * BAT_ERR_CUDA.
 */
BAT_API bat_status_t bat_clip_ratios(const float* g, int64_t n, float* r, void* stream);

/*
 * MXFP4 element conversion as the prologue performs it: codes[t] = E2M1 code of
 * v[t] (round-to-nearest-even, saturating at +-6, sign in bit 3), one code per
 * byte. Values are converted in pairs (2t, 2t+1) exactly as the prologue packs
 * them. v: device fp32 [n]; codes: device uint8 [n].
 * Errors: BAT_ERR_INVALID_ARG (n < 1 or a NULL pointer), BAT_ERR_UNSUPPORTED,
 * BAT_ERR_CUDA.
 */
BAT_API bat_status_t bat_e2m1_encode(const float* v, int64_t n, uint8_t* codes, void* stream);

/*
 * Offline weight side (Method > "Overall Architecture": the inverse transform is
 * fused into the weights once). Row n, block b of W becomes
 * w_b (B_b^-T (x) A^-T) = vec_row(B_b^-1 W_r A^-T), the rows of (P^-1 W^T)^T;
 * then optional per-(row, block) clipping and MXFP4 packing.
 *
 *   W      : bf16 [N][K] row-major, 16-byte aligned.
 *   A, B   : as in bat_quantize_act (device). They are copied to the host and
 *            inverted in fp64 with partial pivoting; a factor whose 1-norm
 *            condition number exceeds 1e6 returns BAT_ERR_SINGULAR.
 *   gw_lo, gw_hi : fp32 [N][K/32] weight clip logits, or both NULL (default: no clip).
 *   Wq     : output, Wq->rows == N, Wq->k == K.
 *   wt_out : optional device fp32 [N][K] for the transformed weights (NULL to skip).
 * This call synchronizes `stream` (it reads A and B on the host). It is meant to
 * run once per layer and is not on the timed path.
 */
BAT_API bat_status_t bat_prepare_weight(const void* W, int64_t N, int64_t K, const float* A,
                                const float* B, const float* gw_lo, const float* gw_hi,
                                const bat_mxfp4_t* Wq, float* wt_out, void* stream);

/*
 * The same two transforms with the 32 channels of a block split another way
 * (the shared/private size sweep of the BATQuant note, Key Designs 2 "GPK
 * decomposition", and the size study in the nubint.ai review): A is s x s and
 * shared by every block, each B_b is t x t with t = 32 / s, and
 *   P_b = B_b (x) A,  P_b[s i + p][s j + q] = B_b[i][j] * A[p][q],
 * so x P_b = vec_row(B_b^T X_r A) with X_r the t x s row-major view of the
 * block. s = 8 is bat_quantize_act / bat_prepare_weight; s = 32 is one shared
 * 32 x 32 transform scaled per block; s = 1 is a fully private 32 x 32 block.
 *
 *   shared : s, one of 1, 2, 4, 8, 16, 32 (anything else: BAT_ERR_UNSUPPORTED).
 *   A      : device fp32 [s][s] row-major, 16-byte aligned.
 *   B      : device fp32 [K/32][t][t] row-major, 16-byte aligned.
 *   y_out  : optional device fp32 [M][K] trace of the transformed values
 *            (NULL to skip), as in bat_quantize_act_trace.
 * All other arguments, requirements and errors are those of bat_quantize_act
 * and bat_prepare_weight (the weight side inverts A and every B_b in fp64 on
 * the host and synchronizes `stream`).
 */
BAT_API bat_status_t bat_quantize_act_gpk(const void* X, int64_t M, int64_t K, const float* A,
                                          int shared, const float* B, const float* g_lo,
                                          const float* g_hi, const bat_mxfp4_t* Xq, float* y_out,
                                          void* stream);
BAT_API bat_status_t bat_prepare_weight_gpk(const void* W, int64_t N, int64_t K, const float* A,
                                            int shared, const float* B, const float* gw_lo,
                                            const float* gw_hi, const bat_mxfp4_t* Wq,
                                            float* wt_out, void* stream);

/*
 * Factors of the block Hadamard rotation (the BRQ article, "Block Rotation"):
 * every 32-channel block is rotated by H_32 / sqrt(32), the normalised
 * Sylvester Hadamard matrix, which is H_t/sqrt(t) (x) H_s/sqrt(s) for any split
 * s t = 32. Writes A = H_s / sqrt(s) ([s][s]) and B_b = H_t / sqrt(t) for
 * b < nb ([nb][t][t]) to HOST buffers (H_n[i][j] = (-1)^popcount(i & j)). Feed
 * them (copied to the device) to the _gpk calls with the same s. Pure host code:
 * no CUDA call. Errors: BAT_ERR_UNSUPPORTED for another s, BAT_ERR_INVALID_ARG
 * for null buffers or nb < 1.
 */
BAT_API bat_status_t bat_block_hadamard_factors(int shared, int64_t nb, float* A, float* B);

/*
 * W4A8 activation side: the transform and clip of bat_quantize_act_gpk, then MXFP8
 * quantization (the W4A8 settings of the BATQuant note, Loss & Training: "MXFP8
 * uses E4M3"). Per 32-element block, e = floor(log2 amax) - 8 (8 is E4M3's largest
 * exponent), clamped to [-127, 127]; elements v * 2^-e rounded to the nearest E4M3
 * (ties to even), saturating at +-448; an exact zero is +0.
 *   Xq : output, Xq->rows == M, Xq->k == K, codes of bat_mxfp8_codes_bytes(M, K).
 * Other arguments, requirements and errors as bat_quantize_act_gpk (shared = 8 with
 * 8 x 8 / [K/32][4][4] factors is the default split).
 */
BAT_API size_t bat_mxfp8_codes_bytes(int64_t rows, int64_t k);
BAT_API bat_status_t bat_quantize_act_mxfp8(const void* X, int64_t M, int64_t K, const float* A,
                                            int shared, const float* B, const float* g_lo,
                                            const float* g_hi, const bat_mxfp8_t* Xq,
                                            float* y_out, void* stream);

/*
 * E4M3 element conversion exactly as the MXFP8 prologue performs it (values
 * converted in groups of four, round to nearest even, saturating at +-448).
 * v: device fp32 [n]; codes: device uint8 [n].
 * Errors: BAT_ERR_INVALID_ARG (n < 1 or a NULL pointer), BAT_ERR_UNSUPPORTED,
 * BAT_ERR_CUDA.
 */
BAT_API bat_status_t bat_e4m3_encode(const float* v, int64_t n, uint8_t* codes, void* stream);

/*
 * W4A8 GEMM: Y = Xq . Wq^T with MXFP8 (E4M3) activations and MXFP4 weights from
 * bat_prepare_weight(_gpk), on tcgen05 kind::mxf8f6f4 (fp32 accumulation).
 *   Y[m][n] = sum_b 2^(eX[m][b] + eW[n][b]) * sum_{j<32} x[m][32b+j] * w[n][32b+j]
 * Requirements beyond bat_mxfp4_gemm's: K % 128 == 0 and Wq->codes 32-byte
 * aligned (the weights' codes are unpacked to one byte per element by the TMA
 * load); otherwise BAT_ERR_SHAPE / BAT_ERR_ALIGN.
 */
BAT_API bat_status_t bat_w4a8_gemm(const bat_mxfp8_t* Xq, const bat_mxfp4_t* Wq, void* Y,
                                   bat_out_dtype_t out_dtype, void* stream);

/*
 * KV-cache path (the BATQuant note, Key Designs 4 "Equivalent Transformer
 * integration": transform sets on the per-head key and value cache paths; the KV8
 * and KV4 settings of Loss & Training store the cache in MXFP8 / MXFP4).
 *
 * Every head vector of D = head_dim channels (D % 32 == 0, 32 <= D <= 256) goes
 * through the block transform x_b (B_b (x) A) with the same factors for every head
 * (A: device fp32 [s][s]; B: device fp32 [D/32][32/s][32/s], one per 32-channel
 * block of the head; s as in bat_quantize_act_gpk), the block clip with logits
 * g_lo, g_hi (device fp32 [D/32], shared by heads and tokens; both NULL for no
 * clip), and MX quantization (reading of bat_quantize_act for KV4, of
 * bat_quantize_act_mxfp8 for KV8). The transform is computed in fp32.
 *
 * Cache layout (caller-owned device buffers of num_slots rows):
 *   codes : [num_slots][H][D] E4M3 bytes (BAT_KV_MXFP8) or [num_slots][H][D/2]
 *           packed E2M1 (BAT_KV_MXFP4, element 2i in the low nibble), 16-byte aligned;
 *   scales: [num_slots][H][D/32] UE8M0 bytes, plain row-major.
 * A paged cache is the same buffers indexed by slot = page * page_size + offset.
 */
typedef enum { BAT_KV_MXFP8 = 0, BAT_KV_MXFP4 = 1 } bat_kv_format_t;

/* Buffer sizes of a cache of num_slots rows (0 for an invalid shape or format). */
BAT_API size_t bat_kv_codes_bytes(int64_t num_slots, int64_t H, int64_t D, bat_kv_format_t fmt);
BAT_API size_t bat_kv_scales_bytes(int64_t num_slots, int64_t H, int64_t D);

/*
 * Quantize T new tokens' K (or V) into the cache.
 *   kv    : device bf16 [T][H][D], 16-byte aligned.
 *   slots : device int64 [T], 8-byte aligned: cache row of token t; -1 skips the
 *           token. A slot >= num_slots is skipped and sets the device error word
 *           (bat_device_error), since it cannot be checked on the host without a copy.
 *   y_out : optional device fp32 [T][H][D] trace of the transformed values (NULL to skip).
 * Errors: BAT_ERR_UNSUPPORTED (s), BAT_ERR_SHAPE (D), BAT_ERR_INVALID_ARG (null
 * pointers, sizes < 1, one clip logit array only), BAT_ERR_ALIGN.
 */
BAT_API bat_status_t bat_kv_quantize(const void* kv, int64_t T, int64_t H, int64_t D,
                                     const float* A, int shared, const float* B,
                                     const float* g_lo, const float* g_hi, const int64_t* slots,
                                     bat_kv_format_t fmt, void* cache_codes, void* cache_scales,
                                     int64_t num_slots, float* y_out, void* stream);

/*
 * Read T cache rows back: out[t][h][:] = the dequantized values of row slots[t]
 * (E4M3 / E2M1 element times 2^(scale - 127)), and, when A and B are given, those
 * values multiplied per 32-channel block by B_b (x) A (pass the inverse factors
 * A^-1 and B_b^-1, split s, to undo the transform). out: device [T][H][D] in
 * out_dtype, 16-byte aligned. A slot outside [0, num_slots) gives zeros and sets
 * the device error word. Errors as bat_kv_quantize.
 */
BAT_API bat_status_t bat_kv_dequantize(const void* cache_codes, const void* cache_scales,
                                       int64_t num_slots, int64_t H, int64_t D,
                                       bat_kv_format_t fmt, const int64_t* slots, int64_t T,
                                       const float* A, int shared, const float* B, void* out,
                                       bat_out_dtype_t out_dtype, void* stream);

/*
 * Block-scaled MXFP4 GEMM on the 5th-generation tensor cores (tcgen05,
 * kind::mxf4, fp32 accumulation in tensor memory):
 *   Y[m][n] = sum_b 2^(eX[m][b] + eW[n][b]) * sum_{j<32} x[m][32b+j] * w[n][32b+j]
 * (the low-bit product Q(XP) . Q(P^-1 W^T) of Key Designs 1).
 *
 *   Xq : M x K MXFP4 activations; Wq : N x K MXFP4 weights (Xq->k == Wq->k).
 *   Y  : device [M][N] row-major, bf16 or fp32 per `out_dtype`, 16-byte aligned.
 * Kernels: M > 128 runs on CTA pairs (256 x 256 tiles); M <= 64 (and K <= 16384) on the
 * decode kernel, Y^T = Wq . Xq^T with K split over a cluster of up to 8 CTAs; otherwise
 * on one SM per tile (split K over a cluster when one row of tiles leaves SMs idle).
 * Every summation order is fixed: the result does not depend on timing.
 * Errors: BAT_ERR_INVALID_ARG (a NULL pointer, an unknown out_dtype, rows < 1 or
 * k < 32), BAT_ERR_SHAPE (Xq->k != Wq->k, k % 32, k or rows over their limits),
 * BAT_ERR_ALIGN (codes, scales or Y not 16-byte aligned), BAT_ERR_UNSUPPORTED (also:
 * the decode kernel's clusters cannot be resident on this device), BAT_ERR_CUDA;
 * nothing is launched on an argument error.
 */
BAT_API bat_status_t bat_mxfp4_gemm(const bat_mxfp4_t* Xq, const bat_mxfp4_t* Wq, void* Y,
                            bat_out_dtype_t out_dtype, void* stream);

/* Workspace bytes bat_linear needs for M rows of K inputs (the quantized X and, for
 * M <= 64 or M > 128, the completion flags the two kernels synchronise on); 0 for an
 * invalid shape. */
BAT_API size_t bat_linear_workspace_bytes(int64_t M, int64_t K);

/*
 * The whole online linear layer Y = Q(XP) . Q(P^-1 W^T): bat_quantize_act into
 * `workspace`, then bat_mxfp4_gemm, on one stream (BATQuant note, en.papernotes.org,
 * Method > Key Designs 1 for the product, 2 and 3 for the transform and the clip).
 *   X  : bf16 [M][K]; Wq from bat_prepare_weight (Wq->k == K); A, B, g_lo, g_hi
 *        as in bat_quantize_act; Y: [M][Wq->rows] in `out_dtype`.
 *   workspace : device, >= bat_linear_workspace_bytes(M, K) bytes, 256-byte aligned.
 *   fused : 0 or 1. With 1 and M > 128 the two kernels overlap at tile granularity:
 *        the quantizer publishes each 128-row token tile's block pairs as it stores
 *        them, and the GEMM starts on a token tile as soon as that tile is complete
 *        instead of after the whole quantizer. Codes and Y are the same bytes as with 0
 *        (the same kernels; only their synchronisation changes). For M <= 128, fused
 *        changes nothing (at M <= 64 the GEMM always starts on the quantizer's
 *        completion flags).
 * Errors: those of bat_quantize_act and bat_mxfp4_gemm, and BAT_ERR_WORKSPACE
 * (workspace NULL or smaller than needed) or BAT_ERR_ALIGN (workspace not
 * 256-byte aligned).
 */
BAT_API bat_status_t bat_linear(const void* X, int64_t M, const bat_mxfp4_t* Wq, const float* A,
                        const float* B, const float* g_lo, const float* g_hi, void* Y,
                        bat_out_dtype_t out_dtype, void* workspace, size_t workspace_bytes,
                        int fused, void* stream);

/*
 * Allocation-free variant of bat_linear. There is no counterpart on the pages:
 * the method's linear layer is bat_linear; this entry point exists only for
 * callers that cannot hand the library a workspace.
 *
 * Who needs it: code that may not call cudaMalloc, and cannot get a device
 * buffer from its host framework either. Examples are plugins run under an
 * allocator that has already reserved all device memory, and serving loops
 * that must not allocate (or make the implicit device synchronization an
 * allocation can cause) once they are running.
 *
 * Instead of a caller workspace, the quantized activations go into a scratch
 * array of BAT_NOALLOC_SCRATCH_BYTES that the library defines in device memory
 * (a static __device__ array). Every GPU that loads the library holds that
 * array until the process exits. Nothing here calls cudaMalloc, cudaFree or any
 * other allocating routine.
 *   - Limit: bat_linear_workspace_bytes(M, Wq->k) must be at most
 *     BAT_NOALLOC_SCRATCH_BYTES (for example M = 2048 at K = 4096, M = 512 at
 *     K = 12288); larger calls return BAT_ERR_WORKSPACE and launch nothing.
 *   - The first call on each device looks up the array's device address with
 *     that device current (cudaGetSymbolAddress) and caches it. Make that first
 *     call before any stream capture. The cached address assumes the device's
 *     primary context lives until the process exits: after cudaDeviceReset (or
 *     anything else that destroys and recreates that context) the address is
 *     stale, so do not call this entry point again in that process.
 *   - All calls share the one array, and it keeps the last call's contents.
 *     Every byte a call reads is written by that same call first, so nothing
 *     needs clearing. Calls that overlap on the GPU (other streams, other host
 *     threads) race on the array: the caller must order them.
 * Other arguments, results and errors are exactly those of bat_linear.
 */
#define BAT_NOALLOC_SCRATCH_BYTES (8u << 20)
BAT_API bat_status_t bat_linear_noalloc(const void* X, int64_t M, const bat_mxfp4_t* Wq,
                                        const float* A, const float* B, const float* g_lo,
                                        const float* g_hi, void* Y, bat_out_dtype_t out_dtype,
                                        void* stream);

/*
 * Self-test of the failure path every kernel wait uses: one thread waits on an
 * mbarrier that nothing arrives on, gives up after `limit_ns` nanoseconds
 * (1 .. 2e9), records the stall in the device error word (bat_device_error then
 * returns a non-zero code) and sets *waited_out (device uint32) to 1. No trap and
 * no endless wait; the context stays usable.
 */
BAT_API bat_status_t bat_selftest_bounded_wait(uint64_t limit_ns, unsigned int* waited_out,
                                               void* stream);

/*
 * Text of the last CUDA error that made a call on this host thread return
 * BAT_ERR_CUDA ("no CUDA error" if none). Static storage; per thread.
 */
BAT_API const char* bat_last_cuda_error(void);

/*
 * Reads and clears the sticky device error word the kernels set when a bounded
 * wait runs out (a pipeline stall that should never happen). Returns 0 if no
 * kernel reported a failure since the last call; synchronizes the device.
 */
BAT_API int bat_device_error(void);

#ifdef __cplusplus
}
#endif

#endif /* BAT_H_ */
