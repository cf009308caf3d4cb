/*
 * svdq.h — C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (devpress.csdn.net SVDQuant paper walkthrough, eq. (5)):
 *
 *     X W  =  X_hat W_hat  ~=  (X_hat L1) L2  +  Q(X_hat) Q(R)
 *
 *   X_hat = X diag(lambda)^-1                smoothed activation
 *   W_hat = diag(lambda) W = L1 L2 + R       16-bit rank-r branch + residual
 *   Q(.)  = NVFP4: E2M1 codes, one E4M3 scale per 16 K-elements (eq. (1), q_max = 6)
 *
 * Conventions used by every entry point:
 *
 *   Orientation.  X is [M][K] (M tokens, K input channels). The weight is given
 *     in nn.Linear orientation W_lin [N][K]; the paper's W is W_lin^T. Y is [M][N].
 *   Memory.  Every pointer is a DEVICE pointer to memory the caller owns, aligned
 *     to 16 bytes (SVDQ_ERR_MISALIGNED otherwise). The library allocates nothing
 *     on the per-call path; svdq_prepare_weights works inside the caller's
 *     workspace. All matrices are dense row-major with no padding between rows.
 *   Streams.  `stream` is a cudaStream_t (NULL = legacy default stream). Calls
 *     are asynchronous with respect to the host unless stated otherwise.
 *   Shapes.  M >= 0 (M == 0 is a no-op), K >= 128 and K % 128 == 0,
 *     N >= 128 and N % 128 == 0, rank % 16 == 0 and 0 <= rank <= 128;
 *     anything else returns SVDQ_ERR_UNSUPPORTED_SHAPE.
 *   Errors.  No entry point aborts or throws. Launch failures return
 *     SVDQ_ERR_CUDA (details in svdq_last_error()). A kernel that gives up on a
 *     bounded wait records a device error word; svdq_check() reads it
 *     (SVDQ_ERR_TIMEOUT) and clears it.
 *   Device.  A device other than compute capability 10.0 returns
 *     SVDQ_ERR_NO_DEVICE. There is no CPU fallback.
 *
 * Buffer formats (byte sizes come from svdq_act_sizes / svdq_weight_sizes):
 *
 *   codes   uint8 [rows][K/2]: E2M1 nibbles, element 2i in the low nibble.
 *   scales  E4M3 bytes in the native tile layout: for row block rb (128 rows)
 *           and K block kb (64 elements) a 512-byte atom at offset
 *           (rb * K/64 + kb) * 512; inside it, row 32q + i and group j (0..3)
 *           of the block sit at byte 16*i + 4*q + j. Rows past the end of the
 *           matrix hold zero. svdq_scales_to_canonical() gives [rows][K/16].
 *   L1p     bf16 [rank][K]: the down-projection factor with the smoothing folded
 *           in, L1p[k][j] = bf16(L1[j][k] / lambda_j), so that X L1p^T == X_hat L1.
 *   L2t     bf16 [N][rank]: the up-projection factor, L2t[n][k] = bf16(L2[k][n]).
 *   T       bf16 [M][rank]: the down-projection X_hat L1.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SVDQ_API __attribute__((visibility("default")))
#else
#define SVDQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer where one is required, bad enum, alpha out of range */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* shape outside the conventions above */
  SVDQ_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
  SVDQ_ERR_BUFFER_TOO_SMALL = 4,   /* workspace smaller than svdq_weight_sizes() asks for */
  SVDQ_ERR_NO_DEVICE = 5,          /* no CUDA device, or not compute capability 10.0 */
  SVDQ_ERR_CUDA = 6,               /* a CUDA runtime call or kernel launch failed */
  SVDQ_ERR_TIMEOUT = 7,            /* a kernel gave up on a bounded wait (see svdq_check) */
  SVDQ_ERR_INTERNAL = 8
} svdq_status;

typedef enum {
  SVDQ_FUSED = 0,    /* low-rank down-projection inside the quantize pass, up-projection
                        inside the 4-bit GEMM's accumulator (walkthrough Fig. 6) */
  SVDQ_UNFUSED = 1   /* the same arithmetic as separate passes: the down-projection
                        re-reads X, the up-projection re-reads and re-writes Y */
} svdq_variant;

/* Problem shape. The quantization group is fixed at 16. */
typedef struct {
  int64_t M;
  int64_t K;
  int64_t N;
  int32_t rank;
} svdq_shape;

/* Flags of svdq_prepare_weights. */
#define SVDQ_PREPARE_GIVEN_FACTORS 1u  /* L1p and L2t are inputs: use the caller's factors */

/* Human-readable name of a status code (static storage; never NULL). */
SVDQ_API const char* svdq_status_string(int status);

/* Last error message of the calling host thread (static thread-local storage). */
SVDQ_API const char* svdq_last_error(void);

/* Library ABI version: 100 * major + minor. */
SVDQ_API int svdq_version(void);

/* Byte sizes of the per-call buffers for `shape`: codes Qx, native scales Sx,
 * and T (0 when rank == 0). Any output pointer may be NULL. Host only. */
SVDQ_API svdq_status svdq_act_sizes(svdq_shape shape, size_t* qx_bytes, size_t* sx_bytes, size_t* t_bytes);

/* Byte sizes of the prepared-weight buffers (Qr codes, native Sr scales, L1p,
 * L2t) and of the workspace svdq_prepare_weights needs. Any output pointer may
 * be NULL. Host only. */
SVDQ_API svdq_status svdq_weight_sizes(svdq_shape shape, size_t* qr_bytes, size_t* sr_bytes, size_t* l1p_bytes,
                              size_t* l2t_bytes, size_t* workspace_bytes);

/* Per-channel activation maximum for the smoothing rule (calibration):
 * amax[j] = max_m |X[m][j]|. X bf16 [M][K], amax fp32 [K] (overwritten).
 * K % 8 == 0 suffices here; M >= 1.
 * (anrans.github.io AI-infra handbook, Quantization chapter, SmoothQuant.) */
SVDQ_API svdq_status svdq_channel_amax(int64_t M, int64_t K, const void* X, float* amax, void* stream);

/* Offline weight preparation (not on the per-call path):
 *   1. smoothing factors: lambda_j = amax_j^alpha / max_n|W_lin[n][j]|^(1-alpha),
 *      lambda_j = 1 where either maximum is 0; lambda = fp32(.), inv_lambda =
 *      fp32(1/lambda)  (handbook SmoothQuant section);
 *   2. W_hat = diag(lambda) W_lin^T and its top-rank SVD split W_hat ~= L1 L2 with
 *      the singular values in L1 (walkthrough: SVD paragraph after eq. (8);
 *      handbook SVDQuant section). Without SVDQ_PREPARE_GIVEN_FACTORS the library
 *      computes it on the device (randomized subspace iteration in fp32,
 *      deterministic: a fixed seed and fixed reduction orders) and writes
 *      L1p = bf16(L1 / lambda)^T [rank][K] and L2t = bf16(L2)^T [N][rank]; with
 *      the flag, L1p and L2t are read as given;
 *   3. residual R = fp32(W_hat - sum_k (lambda * L1p[k]) L2t[:,k]) in fp64, in
 *      increasing k, no fused multiply-add (eq. (5));
 *   4. NVFP4 encoding of R grouped along K: codes Qr [N][K/2], native scales Sr.
 * W_lin bf16 [N][K]; act_amax fp32 [K]; alpha in [0, 1]; lambda, inv_lambda fp32
 * [K] (written); workspace of at least svdq_weight_sizes()'s workspace_bytes
 * (may be NULL when that size is 0). Stream-ordered; the caller's buffers are
 * ready when the stream reaches the end of the call. */
SVDQ_API svdq_status svdq_prepare_weights(svdq_shape shape, const void* W_lin, const float* act_amax, float alpha,
                                 unsigned int flags, void* L1p, void* L2t, void* Qr, void* Sr,
                                 float* lambda, float* inv_lambda, void* workspace, size_t workspace_bytes,
                                 void* stream);

/* Size of the library's own device scratch used by svdq_prepare_weights_static. */
#define SVDQ_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* svdq_prepare_weights without a workspace argument and without any
 * allocation: the device SVD runs in one fixed scratch array of
 * SVDQ_STATIC_SCRATCH_BYTES (32 MiB) that is part of the library's device
 * image. The paper has no counterpart: this is a deployment convenience for
 * callers that cannot hand out workspace memory. Same arguments, flags,
 * arithmetic and outputs as svdq_prepare_weights (bit-identical results).
 *   Limit.  Shapes whose SVD workspace (svdq_weight_sizes' workspace_bytes)
 *     exceeds SVDQ_STATIC_SCRATCH_BYTES are refused with
 *     SVDQ_ERR_BUFFER_TOO_SMALL and a message naming both sizes; use
 *     svdq_prepare_weights with a caller workspace for those. The FLUX
 *     projections at rank 32 need about 14 MB.
 *   Set-up.  The first call on a device looks up the scratch's device address
 *     (and sets kernel attributes) with that device current; make that first
 *     call before capturing a stream into a CUDA graph.
 *   Zero.  Nothing in the scratch needs to start at zero: every byte a call
 *     reads was written earlier in the same call.
 *   Concurrency.  There is one scratch per device and process. Calls whose
 *     work overlaps on the device (other streams, other host threads) race on
 *     it and corrupt each other's factors; serialize them. */
SVDQ_API svdq_status svdq_prepare_weights_static(svdq_shape shape, const void* W_lin, const float* act_amax,
                                                 float alpha, unsigned int flags, void* L1p, void* L2t, void* Qr,
                                                 void* Sr, float* lambda, float* inv_lambda, void* stream);

/* Per-call activation quantization with the low-rank down-projection.
 * X bf16 [M][K]; inv_lambda fp32 [K]; L1p bf16 [rank][K].
 * Writes Qx codes [M][K/2], Sx native scales, T bf16 [M][rank]:
 *   x_hat = fp32(fp32(x) * inv_lambda[k]);
 *   per 16-group: s = E4M3_rne_satfinite(fp32(max|x_hat| / 6)),
 *                 q = E2M1_rne_satfinite(x_hat / s) of the exact real quotient
 *                     (ties to even), all +0 if s == 0;
 *   T = bf16(X L1p^T)  (fp32 accumulation)
 * (eq. (1), Table 3's NVFP4 microscaling, Fig. 6's fused down-projection).
 * variant SVDQ_FUSED reads X once; SVDQ_UNFUSED runs the down-projection as a
 * second pass over X. rank == 0: L1p and T may be NULL. */
SVDQ_API svdq_status svdq_quantize_act(svdq_shape shape, const void* X, const float* inv_lambda, const void* L1p,
                              void* Qx, void* Sx, void* T, int variant, void* stream);

/* Per-call W4A4 GEMM with the low-rank up-projection:
 *   Y = bf16( deq(Qx) deq(Qr)^T + T L2t^T )   (fp32 accumulation)
 * (eq. (2), eq. (5)). Qx/Sx as written by svdq_quantize_act, Qr/Sr/L2t as
 * written by svdq_prepare_weights, Y bf16 [M][N]. variant SVDQ_FUSED adds T L2
 * into the GEMM's tensor-memory accumulator; SVDQ_UNFUSED runs the GEMM with
 * no branch, then a second kernel reads Y, adds T L2 in fp32 and writes Y.
 * rank == 0: T and L2t may be NULL. */
SVDQ_API svdq_status svdq_linear(svdq_shape shape, const void* Qx, const void* Sx, const void* T, const void* Qr,
                        const void* Sr, const void* L2t, void* Y, int variant, void* stream);

/* svdq_linear whose output feeds another W4A4 layer directly: Y, quantized
 * for the NEXT layer (whose K equals this layer's N). The codes and scales are
 * bit-identical to those of the two calls
 *     svdq_linear(shape, ..., Y);
 *     svdq_quantize_act({M, N, *, next_rank}, Y, next_inv_lambda, next_L1p,
 *                       next_Qx, next_Sx, next_T, SVDQ_FUSED, stream);
 * i.e. next_Qx codes [M][N/2], next_Sx native scales of Y's 16-groups along N
 * and, when next_rank > 0, next_T bf16 [M][next_rank] ~= Y next_L1p^T.
 * Routes (walkthrough eq. (1) and Fig. 6's activation quantization, moved into
 * the producer of the activation):
 *   - next_rank == 0 and the shape runs on 256 x 256 CTA-pair tiles: the GEMM's
 *     epilogue encodes the accumulator tile directly; Y is written only if
 *     asked for.
 *   - next_rank 16 or 32 on 256 x 256 pair tiles, with SVDQ_NEXT_FUSE_LOWRANK
 *     in `flags`: the epilogue also forms the next layer's down-projection with
 *     tcgen05 MMAs on the staged Y tile; each tile's fp32 partial of next_T
 *     goes to the workspace and a second kernel adds them in tile order (next_T
 *     then agrees with the two calls within bf16 rounding, not bit for bit).
 *     Measured slower than the two calls on the FLUX projections, so it is
 *     opt-in.
 *   - otherwise Y is formed (in Y, or in the workspace when Y is NULL) and
 *     quantized by svdq_quantize_act's kernel (next_T then bit-identical).
 * Inputs as for svdq_linear, plus next_inv_lambda fp32 [N] and next_L1p bf16
 * [next_rank][N] of the next layer (next_rank in {0, 16, ..., 128}; next_L1p and
 * next_T may be NULL when it is 0). Y bf16 [M][N] is written only if non-NULL.
 * flags: 0 or SVDQ_NEXT_FUSE_LOWRANK; other bits are SVDQ_ERR_INVALID_ARG.
 * workspace / workspace_bytes: at least svdq_linear_quantize_next_workspace()'s
 * size for the same flags -- 0 on the rank-0 fused route, N/256*M*next_rank*4
 * on the low-rank fused route, M*N*2 otherwise (needed there only when Y is
 * NULL); SVDQ_ERR_BUFFER_TOO_SMALL if smaller. Its contents on return are
 * unspecified. Stream-ordered. */
#define SVDQ_NEXT_FUSE_LOWRANK 1u
SVDQ_API svdq_status svdq_linear_quantize_next(svdq_shape shape, const void* Qx, const void* Sx, const void* T,
                                               const void* Qr, const void* Sr, const void* L2t, int32_t next_rank,
                                               const float* next_inv_lambda, const void* next_L1p, void* next_Qx,
                                               void* next_Sx, void* next_T, void* Y, void* workspace,
                                               size_t workspace_bytes, unsigned int flags, void* stream);

/* Workspace bytes svdq_linear_quantize_next needs for `shape`, next_rank and
 * flags on the current device (the route depends on the device's SM count). */
SVDQ_API svdq_status svdq_linear_quantize_next_workspace(svdq_shape shape, int32_t next_rank, unsigned int flags,
                                                         size_t* bytes);

/* LoRA as part of the low-rank branch (walkthrough, Figure 9 and Figure 16: a
 * LoRA runs in, or is merged into, the independent 16-bit branch, with no
 * re-quantization of the residual). A LoRA update Y += X A^T B^T acts on the raw
 * activation, exactly like the stored down-projection L1p (which already has
 * lambda folded in), so the branch of rank r + extra is the concatenation
 *   L1p_out [r + extra][K] = [L1p ; A],   L2t_out [N][r + extra] = [L2t , B].
 * shape.K, shape.N, shape.rank = r describe the prepared layer (shape.M unused);
 * L1p bf16 [r][K], L2t bf16 [N][r] (may be NULL when r == 0), A bf16 [extra][K],
 * B bf16 [N][extra]. extra > 0, multiple of 16, r + extra <= 128
 * (SVDQ_ERR_UNSUPPORTED_SHAPE otherwise). Outputs must not overlap the inputs.
 * Qr/Sr are unchanged; use the layer with rank r + extra afterwards.
 * Stream-ordered device copies only. */
SVDQ_API svdq_status svdq_append_lowrank(svdq_shape shape, int32_t extra, const void* L1p, const void* L2t,
                                         const void* A, const void* B, void* L1p_out, void* L2t_out,
                                         void* stream);

/* ---------------------------------------------------------------- INT4 variant
 * The same layer with INT4 in place of NVFP4 (the pages' path for GPUs without
 * FP4 tensor cores: walkthrough eq. (1) with q_max = 2^(4-1) - 1 = 7; handbook,
 * Quantization chapter: one fp16 scale per 64 elements). Per 64-element group
 * along K:  s = fp16_rne(min(fp32(max|v| / 7), 65504)),
 *           q = clamp(rint(v / s), -7, 7) of the exact real quotient (ties to
 *               even; all 0 when s == 0),
 * and Y = bf16( sum_g sx[m,g] sw[n,g] sum_{k in g} qx[m,k] qr[n,k] + T L2 ).
 * Smoothing, L1p, L2t and T are those of the NVFP4 layer (svdq_prepare_weights);
 * only the residual and the activation are encoded differently.
 *
 * Buffer formats (sizes from svdq_int4_act_sizes / svdq_int4_weight_sizes):
 *   int4 codes   uint8 [rows][K]: one byte per code, the E4M3 encoding of the
 *                integer (0x00 for 0, 0x38 for 1, ..., 0x4E for 7, sign bit 0x80
 *                for negatives). sm_100a has no 4-bit integer MMA; E4M3 holds
 *                every code exactly and feeds the FP8 tensor cores, at twice
 *                the bytes of packed nibbles.
 *   int4 scales  fp32 [K/64][rows_pad], group-major: scale of (row r, group g)
 *                at g * rows_pad + r. Every value is an fp16 value. rows_pad =
 *                ceil(M/128)*128 for the activation (rows past M hold 0) and N for
 *                the weight.
 * Shapes as for the NVFP4 entry points. */
SVDQ_API svdq_status svdq_int4_act_sizes(svdq_shape shape, size_t* qx, size_t* sx, size_t* t);
SVDQ_API svdq_status svdq_int4_weight_sizes(svdq_shape shape, size_t* qr, size_t* sr);

/* INT4 codes and scales of the residual R = W_hat - (lambda L1p^T) L2 (eq. (5);
 * fp64 with every product exact, rounded to fp32 once, exactly as
 * svdq_prepare_weights forms it), grouped along K for every output channel.
 * W_lin bf16 [N][K], lambda fp32 [K], L1p bf16 [rank][K], L2t bf16 [N][rank]
 * as written by svdq_prepare_weights (L1p and L2t may be NULL when rank == 0).
 * Writes Qr uint8 [N][K] and Sr fp32 [K/64][N]. Stream-ordered. */
SVDQ_API svdq_status svdq_int4_quantize_residual(svdq_shape shape, const void* W_lin, const float* lambda,
                                                 const void* L1p, const void* L2t, void* Qr, void* Sr, void* stream);

/* Hot path, step 1 (INT4): one read of X bf16 [M][K] -> smoothing, INT4 codes
 * Qx uint8 [M][K] and scales Sx fp32 [K/64][ceil(M/128)*128], and the fused
 * down-projection T bf16 [M][rank] = bf16(X L1p^T) (same kernel as
 * svdq_quantize_act, INT4 encoder). Async on stream. */
SVDQ_API svdq_status svdq_int4_quantize_act(svdq_shape shape, const void* X, const float* inv_lambda,
                                            const void* L1p, void* Qx, void* Sx, void* T, void* stream);

/* Hot path, step 2 (INT4): Y bf16 [M][N]. Each group's integer products run on
 * FP8 tensor cores into fp32 tensor memory (exact); the group's scale product
 * fp32(sx * sw) (exact) is applied with one fused multiply-add per element into
 * fp32 accumulators; T L2 is added from a bf16 MMA; Y = bf16_rne of the sum.
 * Qx/Sx from svdq_int4_quantize_act, Qr/Sr from svdq_int4_quantize_residual,
 * T and L2t as for svdq_linear (NULL allowed when rank == 0). Async on stream. */
SVDQ_API svdq_status svdq_int4_linear(svdq_shape shape, const void* Qx, const void* Sx, const void* T,
                                      const void* Qr, const void* Sr, const void* L2t, void* Y, void* stream);

/* ---------------------------------------------------------------- DeltaQuant
 * Core + delta encoding of video activations (libaedu.com article on 4-bit
 * diffusion-model quantization, DeltaQuant paragraphs: tokens of a local 3-D
 * spatio-temporal block share a core token, their mean, kept in FP8; each
 * token's difference to it is quantized to 4 bits). The article gives the
 * method in outline only; the readings here:
 *   X        bf16 [F*H*W][C]: the tokens of an F-frame, H x W video latent in
 *            frame, row, column order; C % 64 == 0.
 *   blocks   2 x 2 x 2 tokens tiled from the origin, numbered in (frame, row,
 *            column) order of the block grid ceil(F/2) x ceil(H/2) x ceil(W/2);
 *            blocks at a ragged edge hold the tokens that exist.
 *   core     uint8 [blocks][C]: E4M3 (fn, saturating at 448) of the block's
 *            exact mean per channel, rounded once to nearest even; a negative
 *            mean rounding to zero keeps the sign bit (0x80), a zero sum is 0x00.
 *   Qd, Sd   the NVFP4 codes [F*H*W][C/2] and native-layout scales of the
 *            deltas fp32(x - core), grouped by 16 channels, in the format of
 *            svdq_quantize_act's Qx / Sx (rows past the last token of the last
 *            128-row scale atom hold zero).
 * Sizes of the three outputs from svdq_deltaquant_sizes. Shapes: F, H, W >= 1,
 * F*H*W < 2^31, 64 <= C <= 2^20 with C % 64 == 0; otherwise
 * SVDQ_ERR_UNSUPPORTED_SHAPE. Pointers as everywhere (device, 16-byte aligned,
 * caller-owned). Async on stream. */
SVDQ_API svdq_status svdq_deltaquant_sizes(int64_t F, int64_t H, int64_t W, int64_t C, size_t* core_bytes,
                                           size_t* qd_bytes, size_t* sd_bytes);
SVDQ_API svdq_status svdq_deltaquant_encode(int64_t F, int64_t H, int64_t W, int64_t C, const void* X, void* core,
                                            void* Qd, void* Sd, void* stream);

/* Diagnostic of the failure path (the pages have no counterpart): one thread
 * waits, with the library's bounded wait, on a barrier phase that nothing
 * completes; after the wait limit (2 s) it records the device error word and
 * returns -- no fault, no hang, the context stays usable. The next svdq_check()
 * on the stream returns SVDQ_ERR_TIMEOUT and clears the word. */
SVDQ_API svdq_status svdq_selftest_timeout(void* stream);

/* Native scale layout -> canonical [rows][K/16] bytes (inspection helper). */
SVDQ_API svdq_status svdq_scales_to_canonical(int64_t rows, int64_t K, const void* native, void* canonical,
                                     void* stream);

/* Synchronize `stream`, then read and clear the device error word of the
 * current device. Returns SVDQ_ERR_TIMEOUT if a kernel gave up on a bounded
 * wait since the last check, SVDQ_ERR_CUDA on an asynchronous CUDA error. */
SVDQ_API svdq_status svdq_check(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
