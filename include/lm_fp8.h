/*
 * lm_fp8.h -- C ABI of libfp8lm.so: FP8 training GEMMs with dynamic
 * tensorwise scaling for a non-gated relu^2 MLP and plain linears, written for
 * NVIDIA B200 (sm_100a).
 *
 * The method (little-lm write-up, decomputer.nl, "Het trainen van een 3.8B
 * LLM tot 0.384 CORE voor $998", section "Vroege experimenten" item 4 and
 * section "Doorvoer (Throughput) verhogen", FP8 bullet; simpleprog.com,
 * "Training a 3.8B LLM to 0.384 CORE for $998", "Five Changes That Mattered"):
 * all three GEMMs of every linear layer -- forward Y = X W^T, dgrad
 * dX = dY W, wgrad dW = dY^T X -- run in FP8, each operand quantised with one
 * fp32 scale computed from that tensor's current amax.  The MLP is the
 * non-gated relu^2 MLP at 4x ("Niet-gated MLPs" bullet; "Appendix: De
 * configuratie": hidden 3072, intermediate 12288, hidden_act relu2).
 *
 * Formats: e4m3 (OCP E4M3, max 448, no infinities) for activations and
 * weights, e5m2 (OCP E5M2, max 57344) for gradients.  Codes are raw bytes.
 *
 * Conventions for every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory.  bf16 tensors are passed as `const void*` /
 *    `void*` holding IEEE bfloat16 bits.  Scales are device fp32.
 *  - Matrices are row-major.  "K-major" means the reduction dimension is the
 *    contiguous one: A [M x K] and B [N x K] for D = A B^T.
 *  - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is
 *    the legacy default stream).  No entry point synchronises the host, and
 *    no scale ever travels to the host.
 *  - Argument, alignment and shape checks run on the host before any launch
 *    and return a non-zero status without enqueuing anything.  A failed launch
 *    returns LM_ERR_CUDA.  Device-side failures (a bounded wait that ran out)
 *    are recorded in a per-device error word read by lm_get_error().
 *  - No C++ exception crosses this interface.
 */
#ifndef LM_FP8_H
#define LM_FP8_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define LM_API __attribute__((visibility("default")))
#else
#define LM_API
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* lm_stream_t;

typedef enum {
    LM_OK = 0,
    LM_ERR_INVALID_ARG = 1,        /* null pointer, negative size, workspace too small */
    LM_ERR_ALIGNMENT = 2,          /* a pointer or row pitch not 16-byte aligned */
    LM_ERR_UNSUPPORTED_SHAPE = 3,  /* a dimension violates the documented multiple */
    LM_ERR_UNSUPPORTED_FORMAT = 4, /* e5m2 x e5m2, or an unknown format/epilogue */
    LM_ERR_CUDA = 5,               /* a CUDA runtime/driver call or launch failed */
    LM_ERR_TIMEOUT = 6,            /* a device-side bounded wait ran out */
    LM_ERR_NONFINITE = 7           /* a cast met a NaN or infinite amax (lm_get_error) */
} lm_status;

typedef enum { LM_FP8_E4M3 = 0, LM_FP8_E5M2 = 1 } lm_fp8_format;

typedef enum {
    LM_EPI_NONE = 0,      /* D = bf16(acc * s) */
    LM_EPI_RELU2_FWD = 1, /* D = H = bf16(acc * s); amax of h = bf16(relu(H)^2) */
    LM_EPI_RELU2_BWD = 2, /* g = bf16(acc * s); D = dH = bf16(g * 2 * relu(aux)) */
    LM_EPI_ACCUM_F32 = 3  /* D is fp32: D += fp32(acc * s) (gradient accumulation) */
} lm_epilogue;

/* Flags of lm_relu2_mlp_fwd_ex / lm_relu2_mlp_bwd_ex (gradient accumulation
 * over micro-batches: decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384
 * CORE voor $998", section "Vroege experimenten" item 2 and "Appendix: De
 * configuratie", total_batch_size = 20 x 2048 x 7 grad_accum x 8 GPUs). */
#define LM_MLP_REUSE_WEIGHT_CASTS 1u /* fwd: the W_up/W_down codes and scales already in
                                        `saved` are current; their casts are skipped */
#define LM_MLP_ACCUMULATE_WGRAD 2u   /* bwd: dW_up and dW_down are fp32 accumulators;
                                        this micro-batch's weight gradients are added */

/*
 * Dynamic tensorwise scaling cast (amax -> scale -> saturating RNE cast).
 *
 *   amax  = max |x|                      (relu2_input: max h, h = bf16(relu(x)^2))
 *   scale = fp32(fmax / max(amax, 1e-12)),  fmax = 448 (e4m3) or 57344 (e5m2)
 *   inv   = fp32(1 / scale)
 *   q[r][c] = sat_rne_fp8(fp32(x_or_h[r][c] * scale)),  qT[c][r] = q[r][c]
 *
 * x: bf16 [rows x cols] with leading dimension ld (elements).
 * amax_in: if non-NULL, a device fp32 already holding the amax of the tensor
 *   to be cast (for example written by lm_fp8_gemm's epilogue); no reduction
 *   pass runs.  If NULL, a reduction pass computes it.
 * amax_out, scale_out, inv_scale_out: device fp32, written (amax_out may
 *   alias amax_in).  When amax_in is NULL, amax_out is also the reduction's
 *   accumulator and is overwritten.
 * q: [rows x cols] codes, qT: [cols x rows] codes (the K-major copy that
 *   dgrad/wgrad consume); either may be NULL to skip it.
 * Requirements: cols % 16 == 0, ld % 8 == 0, ld >= cols; rows % 16 == 0 when
 *   qT != NULL; x, q, qT 16-byte aligned.  rows == 0 or cols == 0 writes the
 *   amax (0) and scales only.
 */
LM_API lm_status lm_fp8_amax_scale_cast(const void* x, int64_t rows, int64_t cols, int64_t ld,
                                 lm_fp8_format fmt, int relu2_input, const float* amax_in,
                                 float* amax_out, float* scale_out, float* inv_scale_out,
                                 uint8_t* q, uint8_t* qT, lm_stream_t stream);

/*
 * FP8 GEMM on the 5th-generation tensor cores (tcgen05, TMEM accumulators):
 *
 *   acc[m][n] = sum_k A[m][k] * B[n][k]      (fp32 accumulation of the FP8 products)
 *   s = inv_scale_a * inv_scale_b
 *   D[m][n] = epilogue(acc * s) as bf16     (see lm_epilogue)
 *
 * A: [M x K] codes of format fa, B: [N x K] codes of format fb, both K-major.
 * inv_scale_a / inv_scale_b: device fp32 dequantisation factors (1/scale).
 * aux: bf16 [M x N], the saved pre-activation H, required for
 *   LM_EPI_RELU2_BWD, ignored otherwise.
 * D: bf16 [M x N], row-major; for LM_EPI_ACCUM_F32 an fp32 [M x N] accumulator
 *   that is added to (each element receives exactly one add per call, so the
 *   result does not depend on scheduling).
 * amax_out: device fp32 or NULL.  If non-NULL it is max-reduced (atomically,
 *   order independent) with the amax of the tensor the next cast consumes:
 *   max|D| (NONE), max bf16(relu(D)^2) (RELU2_FWD), max|D| (RELU2_BWD); unused
 *   for ACCUM_F32.  The caller zeroes it before the first GEMM that feeds it.
 * Formats: (e4m3, e4m3), (e5m2, e4m3), (e4m3, e5m2); e5m2 x e5m2 returns
 *   LM_ERR_UNSUPPORTED_FORMAT.
 * Requirements: K % 16 == 0, N % 8 == 0; A, B, D, aux 16-byte aligned.
 *   M and N need not be multiples of the tile; K == 0 writes D = 0.
 */
LM_API lm_status lm_fp8_gemm(const uint8_t* A, lm_fp8_format fa, const uint8_t* B, lm_fp8_format fb,
                      int64_t M, int64_t N, int64_t K, const float* inv_scale_a,
                      const float* inv_scale_b, lm_epilogue epi, const void* aux, void* D,
                      float* amax_out, lm_stream_t stream);

/* Operand storage flags of lm_fp8_gemm_ex. */
#define LM_GEMM_A_MN_MAJOR 1u /* A stored as [K x M] row-major (M contiguous), i.e. A^T */
#define LM_GEMM_B_MN_MAJOR 2u /* B stored as [K x N] row-major (N contiguous), i.e. B^T */

/*
 * lm_fp8_gemm with the storage of each operand chosen by `flags`: the same
 * D = epilogue(A B^T s), where an MN-major operand is read as the transpose
 * of the matrix stored.  This lets dgrad and wgrad consume the row-major codes
 * of a cast directly: the tensor cores read 8-bit operands in either order
 * from shared memory, so no transposed copy of the codes is needed
 * (tcgen05.mma instruction descriptor, "transpose A/B" bits).
 * Additional requirements: M % 16 == 0 with LM_GEMM_A_MN_MAJOR, N % 16 == 0
 * with LM_GEMM_B_MN_MAJOR (each stored row starts on a 16-byte boundary);
 * unknown flag bits return LM_ERR_INVALID_ARG.  With flags == 0 and no
 * workspace this is lm_fp8_gemm.
 *
 * workspace (device, 16-byte aligned, >= lm_fp8_gemm_workspace_size() bytes,
 * or NULL): scratch for a split-K tail.  The persistent grid gives tiles out
 * round-robin, so a last wave with fewer tiles than CTA pairs leaves pairs
 * idle.  Each tile of that wave may instead be computed as S units over S
 * ranges of K (lm_fp8_gemm_split_plan gives S for a shape): the last unit of
 * a tile adds the others' fp32 sums, exchanged through the workspace, before
 * the epilogue.  The result then differs from the unsplit one only by fp32
 * summation order; it is the same from call to call.  Calls that share a
 * workspace must not overlap on the GPU.  With NULL (ws_bytes 0) no tile is
 * split.
 * Operands stored MN-major give bit-identical results to lm_fp8_gemm on the
 * transposed copies (with the same workspace choice).
 */
LM_API lm_status lm_fp8_gemm_ex(const uint8_t* A, lm_fp8_format fa, const uint8_t* B,
                         lm_fp8_format fb, int64_t M, int64_t N, int64_t K, uint32_t flags,
                         const float* inv_scale_a, const float* inv_scale_b, lm_epilogue epi,
                         const void* aux, void* D, float* amax_out, void* workspace,
                         size_t ws_bytes, lm_stream_t stream);

/* Workspace bytes that let lm_fp8_gemm_ex split the last wave of any shape
 * (a fixed size: 128 partial tiles' fp32 sums and flags, about 32 MB). */
LM_API size_t lm_fp8_gemm_workspace_size(void);

/* The split-K tail lm_fp8_gemm_ex (with a workspace) uses for an M x N x K
 * GEMM on a GPU of sm_count multiprocessors.  Host arithmetic only; nothing
 * is launched and no GPU is needed.  *parts: the K ranges each tile of the
 * last wave runs as (1: no split); *tail_tiles: how many tiles are split.
 *  - A last wave of at most half as many tiles as CTA pairs is halved.
 *  - Otherwise the wave's tiles are split only when a time model of the tail
 *    says that more parts are clearly faster.
 *  - Shapes with M <= 128 (a single-CTA kernel) are never split.
 * Returns LM_ERR_INVALID_ARG for null outputs, negative sizes or sm_count < 2. */
LM_API lm_status lm_fp8_gemm_split_plan(int64_t M, int64_t N, int64_t K, int sm_count,
                                        int* parts, int* tail_tiles);

/*
 * The producer of a GEMM input: RMSNorm, then the dynamic FP8 cast of its
 * output (the model's pre-norm; decomputer.nl, "Het trainen van een 3.8B
 * LLM tot 0.384 CORE voor $998", "Appendix: De configuratie", rms_norm_eps
 * 1e-6, PyTorch's F.rms_norm):
 *
 *   X[r][c] = bf16( R[r][c] / sqrt(mean_c R[r][c]^2 + eps) * weight[c] )
 *   then amax / scale / q / qT of X exactly as lm_fp8_amax_scale_cast.
 *
 * The normalising pass also max-reduces |X|, so the cast needs no reduction
 * pass of its own.  R: bf16 [rows x cols] (contiguous); weight: bf16 [cols] or
 * NULL (no weight); X: bf16 [rows x cols] output; amax_out, scale_out,
 * inv_scale_out, q, qT as in lm_fp8_amax_scale_cast.  The norm accumulates in
 * fp32 (sum of squares, one IEEE sqrt and division).  Requirements as for
 * the cast, plus R, weight, X 16-byte aligned and eps >= 0.
 */
LM_API lm_status lm_rmsnorm_fp8_cast(const void* R, const void* weight, int64_t rows,
                                     int64_t cols, float eps, lm_fp8_format fmt, void* X,
                                     float* amax_out, float* scale_out, float* inv_scale_out,
                                     uint8_t* q, uint8_t* qT, lm_stream_t stream);

/*
 * Tensors the relu^2 MLP forward saves for its backward.  Every pointer is a
 * caller-owned device buffer (see lm_relu2_mlp_saved_carve).  Shapes for
 * X [M x d], W_up [f x d], W_down [d x f]:
 */
typedef struct lm_mlp_saved {
    uint8_t* Xq;   /* [M x d] e4m3; wgrad of W_up reads it MN-major */
    uint8_t* Wuq;  /* [f x d] e4m3, B of the up GEMM; dgrad reads it MN-major */
    uint8_t* Wdq;  /* [d x f] e4m3, B of the down GEMM; dgrad reads it MN-major */
    void* H;       /* [M x f] bf16 pre-activation X W_up^T */
    uint8_t* hq;   /* [M x f] e4m3 codes of h = bf16(relu(H)^2); wgrad reads it MN-major */
    float* scales; /* 16 device floats: {amax, scale, inv_scale, unused} for X, W_up, W_down, h */
} lm_mlp_saved;

/* Bytes needed to hold every buffer of lm_mlp_saved (each 256-byte aligned). */
LM_API size_t lm_relu2_mlp_saved_bytes(int64_t M, int64_t d, int64_t f);

/* Host-only pointer arithmetic: carve a caller-allocated device buffer `base`
 * of `bytes` (>= lm_relu2_mlp_saved_bytes) into `out`.  Launches nothing. */
LM_API lm_status lm_relu2_mlp_saved_carve(void* base, size_t bytes, int64_t M, int64_t d, int64_t f,
                                   lm_mlp_saved* out);

/* Bytes of scratch lm_relu2_mlp_bwd needs.  Its first
 * lm_fp8_gemm_workspace_size() bytes are the GEMMs' split-K scratch, which is
 * all lm_relu2_mlp_fwd uses of it (optionally). */
LM_API size_t lm_relu2_mlp_workspace_size(int64_t M, int64_t d, int64_t f);

/*
 * relu^2 MLP forward, Y = relu(X W_up^T)^2 W_down^T, every GEMM in FP8:
 *   cast X, W_up, W_down to e4m3 (one amax launch for the three, one cast
 *     launch for X and W_up; W_down's codes are written by extra warps of
 *     the up GEMM's launch, which does not read them)
 *   H = up GEMM with the RELU2_FWD epilogue (bf16 H + amax of h)
 *   cast h = bf16(relu(H)^2) to e4m3 using that amax
 *   Y = down GEMM (bf16)
 * Only row-major codes are made: the backward's GEMMs read them MN-major
 * (lm_fp8_gemm_ex), so no transposed copy is written or saved.
 * X: bf16 [M x d], W_up: bf16 [f x d], W_down: bf16 [d x f], Y: bf16 [M x d].
 * workspace: NULL (ws_bytes 0), or 256-byte-aligned device scratch of at least
 * lm_fp8_gemm_workspace_size() bytes (e.g. the backward's workspace), which
 * lets the GEMMs split an under-filled last wave (see lm_fp8_gemm_ex).  With
 * a workspace and M > 128, the cast of h runs inside the down GEMM's launch
 * (extra warps cast it in 256 x 128 blocks just before the GEMM's tiles read
 * them; the workspace also holds one ready bit per block); otherwise it is its
 * own launch before the down GEMM.  The codes are the same either way.
 * Requirements: M, d, f multiples of 16.  M may be 0 (an empty micro-batch):
 * X and Y may then be NULL, the weights are still cast, and the scale blocks
 * of X and h are those of amax 0.
 */
LM_API lm_status lm_relu2_mlp_fwd(const void* X, const void* W_up, const void* W_down, int64_t M,
                           int64_t d, int64_t f, void* Y, lm_mlp_saved* saved, void* workspace,
                           size_t ws_bytes, lm_stream_t stream);

/*
 * relu^2 MLP backward from the forward's saved tensors:
 *   cast dY to e5m2
 *   dH = dgrad of W_down with the RELU2_BWD epilogue: bf16(bf16(dY W_down) * 2 relu(H))
 *   dW_down = dY^T h   (wgrad, K = M)
 *   cast dH to e5m2 using the epilogue's amax (by extra warps of the dW_down
 *     GEMM's launch, which does not read dH)
 *   dX = dH W_up;  dW_up = dH^T X
 * (W_down and W_up as dgrad B operands, and dY, h, dH, X as wgrad operands,
 * are read MN-major from their row-major codes.)
 * dY: bf16 [M x d]; outputs bf16 dX [M x d], dW_up [f x d], dW_down [d x f].
 * workspace: device scratch of >= lm_relu2_mlp_workspace_size bytes,
 * 256-byte aligned.  Requirements as for the forward.  With M == 0, dY and dX
 * may be NULL, and dW_up and dW_down are zero.
 */
LM_API lm_status lm_relu2_mlp_bwd(const void* dY, const lm_mlp_saved* saved, int64_t M, int64_t d,
                           int64_t f, void* dX, void* dW_up, void* dW_down, void* workspace,
                           size_t ws_bytes, lm_stream_t stream);

/*
 * relu^2 MLP backward that allocates nothing (no counterpart on the pages:
 * the method itself says nothing about memory ownership).  For callers that
 * cannot hand the library a workspace: plugins whose host framework owns all
 * device memory and forbids allocation in its execute callback, and loops that
 * cannot absorb the device-wide synchronisation of cudaMalloc/cudaFree.
 * Computes exactly what lm_relu2_mlp_bwd computes, using as its workspace a
 * 64 MiB device array owned by the library (lm_relu2_mlp_bwd_noalloc_max_bytes).
 *  - A shape fits when lm_relu2_mlp_workspace_size(M, d, f) is at most that
 *    size: the GEMMs' split-K scratch (lm_fp8_gemm_workspace_size, about
 *    32 MiB) plus M*d + 3*M*f bytes, each part rounded up to 256 bytes.  At
 *    the model's d = 3072, f = 12288 that is M <= 832 tokens (M = 512 fits,
 *    M = 1024 does not); the 256 x 256 x 1024 block fits.  Larger shapes
 *    return LM_ERR_UNSUPPORTED_SHAPE with nothing enqueued.
 *  - The first call on a device looks up the array's device address with that
 *    device current; make that first call before any stream capture begins.
 *    The looked-up address is not valid after cudaDeviceReset on that device.
 *    Every GPU that loads the array keeps it until the process exits.
 *  - All calls on a device share the array, which keeps the previous call's
 *    contents (the backward re-zeroes what must start at zero).  Calls whose
 *    work overlaps on the GPU (e.g. on two unordered streams) race; calls on
 *    one stream are safe.
 * Other arguments, layouts and errors as lm_relu2_mlp_bwd.
 */
LM_API lm_status lm_relu2_mlp_bwd_noalloc(const void* dY, const lm_mlp_saved* saved, int64_t M,
                                          int64_t d, int64_t f, void* dX, void* dW_up,
                                          void* dW_down, lm_stream_t stream);

/* Size in bytes of the array lm_relu2_mlp_bwd_noalloc uses as its workspace. */
LM_API size_t lm_relu2_mlp_bwd_noalloc_max_bytes(void);

/*
 * Gradient-accumulation forms of the MLP forward and backward (flags above).
 * With flags == 0 they are lm_relu2_mlp_fwd / lm_relu2_mlp_bwd.
 *  - LM_MLP_REUSE_WEIGHT_CASTS (fwd): skip the casts of W_up and W_down and
 *    use the codes and scales `saved` holds from an earlier
 *    forward of the same weights (once per optimizer step is enough).
 *  - LM_MLP_ACCUMULATE_WGRAD (bwd): dW_up [f x d] and dW_down [d x f] are fp32;
 *    each wgrad GEMM adds fp32(acc * s) into them (LM_EPI_ACCUM_F32); dX stays
 *    bf16.  The caller zeroes the accumulators at the start of an optimizer step.
 */
LM_API lm_status lm_relu2_mlp_fwd_ex(const void* X, const void* W_up, const void* W_down,
                                     int64_t M, int64_t d, int64_t f, void* Y, lm_mlp_saved* saved,
                                     void* workspace, size_t ws_bytes, uint32_t flags,
                                     lm_stream_t stream);
LM_API lm_status lm_relu2_mlp_bwd_ex(const void* dY, const lm_mlp_saved* saved, int64_t M,
                                     int64_t d, int64_t f, void* dX, void* dW_up, void* dW_down,
                                     void* workspace, size_t ws_bytes, uint32_t flags,
                                     lm_stream_t stream);

/*
 * Plain FP8 linear layer, Y = X W^T, with its dgrad and wgrad (the attention
 * projections and the LM head of the model; decomputer.nl, "Het trainen van
 * een 3.8B LLM tot 0.384 CORE voor $998", section "Vroege experimenten" item
 * 4: all three GEMMs of a linear in FP8 with dynamic tensorwise scaling):
 *   forward:  cast X, W to e4m3 (one amax launch, one cast launch);  Y = Xq Wq^T
 *   backward: cast dY to e5m2;  dX = dYq Wq;  dW = dYq^T Xq   (K of the wgrad = M)
 * Only row-major codes are made; the dgrad reads Wq and the wgrad reads dYq
 * and Xq MN-major (lm_fp8_gemm_ex), so no transposed copy is written.
 * X: bf16 [M x K]; W: bf16 [N x K]; Y, dY: bf16 [M x N]; dX: bf16 [M x K];
 * dW: bf16 [N x K], or an fp32 accumulator with LM_LINEAR_ACCUMULATE_WGRAD.
 * Requirements: M, K, N multiples of 16 (M may be 0).
 */
typedef struct lm_linear_saved {
    uint8_t* Xq;   /* [M x K] e4m3 codes of X; the wgrad reads them MN-major */
    uint8_t* Wq;   /* [N x K] e4m3 codes of W; the dgrad reads them MN-major */
    float* scales; /* 8 device floats: {amax, scale, inv_scale, unused} for X, then W */
} lm_linear_saved;

#define LM_LINEAR_REUSE_WEIGHT_CAST 1u /* fwd: W's codes and scale block in `saved` are
                                          current; W's cast is skipped (W may be NULL) */
#define LM_LINEAR_ACCUMULATE_WGRAD 2u  /* bwd: dW is an fp32 [N x K] accumulator; this
                                          call's weight gradient is added to it */

/* Bytes of every buffer of lm_linear_saved (each 256-byte aligned); 0 for an
 * unsupported shape. */
LM_API size_t lm_fp8_linear_saved_bytes(int64_t M, int64_t K, int64_t N);

/* Host-only pointer arithmetic: carve a caller-allocated, 256-byte-aligned
 * device buffer `base` of `bytes` (>= lm_fp8_linear_saved_bytes) into `out`. */
LM_API lm_status lm_fp8_linear_saved_carve(void* base, size_t bytes, int64_t M, int64_t K,
                                           int64_t N, lm_linear_saved* out);

/* Bytes of scratch lm_fp8_linear_bwd needs: the GEMMs' split-K scratch
 * (lm_fp8_gemm_workspace_size bytes, all the forward uses of it), then dY's
 * codes and scale block; 0 for an unsupported shape. */
LM_API size_t lm_fp8_linear_workspace_size(int64_t M, int64_t K, int64_t N);

/* Forward.  workspace: NULL (ws_bytes 0) or 256-byte-aligned scratch of at least
 * lm_fp8_gemm_workspace_size() bytes, which lets the GEMM split an under-filled
 * last wave.  flags: 0 or LM_LINEAR_REUSE_WEIGHT_CAST; other bits return
 * LM_ERR_INVALID_ARG. */
LM_API lm_status lm_fp8_linear_fwd(const void* X, const void* W, int64_t M, int64_t K,
                                   int64_t N, void* Y, lm_linear_saved* saved, void* workspace,
                                   size_t ws_bytes, uint32_t flags, lm_stream_t stream);

/* Backward from the forward's saved codes.  dX may be NULL (no dgrad, e.g. for a
 * layer whose input needs no gradient).  workspace: >= lm_fp8_linear_workspace_size
 * bytes, 256-byte aligned.  flags: 0 or LM_LINEAR_ACCUMULATE_WGRAD. */
LM_API lm_status lm_fp8_linear_bwd(const void* dY, const lm_linear_saved* saved, int64_t M,
                                   int64_t K, int64_t N, void* dX, void* dW, void* workspace,
                                   size_t ws_bytes, uint32_t flags, lm_stream_t stream);

/*
 * Gated (SwiGLU) MLP, the comparison workload of the non-gated relu^2 MLP
 * (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998",
 * section "Doorvoer (Throughput) verhogen", bullet "Niet-gated MLPs": three
 * matmuls instead of two; intermediate ratio 2.75).  Same FP8 tensorwise
 * scaling, e4m3 activations and weights, e5m2 gradients.
 *
 *   G = X W_gate^T, U = X W_up^T, h = bf16(silu(G) U), Y = h W_down^T
 *   backward: g = dY W_down; dG = bf16(g U silu'(G)); dU = bf16(g silu(G));
 *   dX = dG W_gate + dU W_up; dW_gate = dG^T X; dW_up = dU^T X; dW_down = dY^T h
 *
 * Layout: W_gu is [2f x d] with the rows of W_gate and W_up interleaved in
 * blocks of 128 (rows 256b..256b+127 = W_gate rows 128b.., the next 128 =
 * W_up rows 128b..); dW_gu comes back in the same order.  f % 128 == 0,
 * d % 16 == 0, M % 16 == 0.  Buffers, workspace and errors as for the relu^2
 * MLP, M = 0 included (an empty micro-batch: tensors with M rows may be NULL,
 * the weights are still cast, the weight gradients are zero); the saved GU
 * holds G and U in the same interleaved column order.
 */
typedef struct lm_swiglu_saved {
    uint8_t* Xq;           /* [M x d] e4m3 (read MN-major by the wgrad of W_gu) */
    uint8_t* Wguq;         /* [2f x d] e4m3, interleaved gate/up */
    uint8_t* Wdq;          /* [d x f] e4m3 */
    void* GU;              /* [M x 2f] bf16 pre-activations, interleaved */
    void* h;               /* [M x f] bf16 silu(G) U */
    uint8_t* hq;           /* [M x f] e4m3 (read MN-major by the wgrad of W_down) */
    float* scales;         /* 16 floats: {amax, scale, inv_scale, 0} for X, W_gu, W_down, h */
} lm_swiglu_saved;

LM_API size_t lm_swiglu_mlp_saved_bytes(int64_t M, int64_t d, int64_t f);
LM_API lm_status lm_swiglu_mlp_saved_carve(void* base, size_t bytes, int64_t M, int64_t d,
                                           int64_t f, lm_swiglu_saved* out);
LM_API size_t lm_swiglu_mlp_workspace_size(int64_t M, int64_t d, int64_t f);
LM_API lm_status lm_swiglu_mlp_fwd(const void* X, const void* W_gu, const void* W_down,
                                   int64_t M, int64_t d, int64_t f, void* Y, lm_swiglu_saved* saved,
                                   void* workspace, size_t ws_bytes, lm_stream_t stream);
LM_API lm_status lm_swiglu_mlp_bwd(const void* dY, const lm_swiglu_saved* saved, int64_t M,
                                   int64_t d, int64_t f, void* dX, void* dW_gu, void* dW_down,
                                   void* workspace, size_t ws_bytes, lm_stream_t stream);

/*
 * The LM head in FP8 inside a chunked, softcapped fused linear cross-entropy
 * (decomputer.nl, "Het trainen van een 3.8B LLM tot 0.384 CORE voor $998",
 * section "Doorvoer (Throughput) verhogen", fused linear cross-entropy
 * bullet, and "Appendix: De configuratie": loss with softcap 15.0).  Forward
 * and backward in one call; the M x V logits are never held in full:
 *
 *   z = softcap * tanh(logits / softcap),  logits = X W^T (FP8 GEMM, bf16)
 *   loss_out = mean over the M tokens of (logsumexp(z) - z[label])
 *   dX  = dlogits W              (FP8 dgrad, e5m2 x e4m3, bf16 out)
 *   dW += fp32(dlogits^T X)      (FP8 wgrad accumulated into the caller's fp32 dW)
 *   dlogits = (softmax(z) - onehot(label)) (1 - (z/softcap)^2) / M
 *
 * X and W are quantised once (X's per-chunk codes use X's whole-tensor
 * scale); each chunk's dlogits gets its own tensorwise e5m2 scale.  All V
 * columns take part in the softmax.
 * X: bf16 [M x d]; W: bf16 [V x d]; labels: device int32 [M], each in [0, V);
 * loss_out: device fp32 scalar; dX: bf16 [M x d]; dW: fp32 [V x d] (added to);
 * chunk: tokens per chunk; workspace: >= lm_fp8_lmhead_ce_workspace_size bytes,
 * 256-byte aligned.  M, d, V, chunk multiples of 16.  M may be 0: X, labels
 * and dX may then be NULL, W is still cast, the loss is 0 and dW is unchanged.
 */
LM_API size_t lm_fp8_lmhead_ce_workspace_size(int64_t M, int64_t d, int64_t V, int64_t chunk);
LM_API lm_status lm_fp8_lmhead_ce(const void* X, const void* W, const int32_t* labels, int64_t M,
                                  int64_t d, int64_t V, int64_t chunk, float softcap,
                                  float* loss_out, void* dX, float* dW, void* workspace,
                                  size_t ws_bytes, lm_stream_t stream);

/* Synchronises `stream`, then returns and clears the current device's error
 * word (the first code recorded since the last call wins):
 *  - LM_ERR_TIMEOUT if a kernel's bounded wait ran out;
 *  - LM_ERR_INVALID_ARG if a kernel met invalid device-side data (code 0x401:
 *    a label outside [0, V) in lm_fp8_lmhead_ce, treated as having no target);
 *  - LM_ERR_NONFINITE if a cast's amax was NaN or infinite (code 0x501: the
 *    tensor held a NaN or an infinity; its scales and codes follow the formulas
 *    and are NaN or zero, and everything computed from them is meaningless);
 *  - LM_ERR_CUDA if the synchronisation itself failed; else LM_OK.
 * If where_out is non-NULL it receives the code (0 if none). */
LM_API lm_status lm_get_error(lm_stream_t stream, uint32_t* where_out);

/*
 * Kernel-boundary timing, for benchmarks (no counterpart on the pages).
 * lm_timing_attach(events, capacity) makes every kernel launch that the
 * calling host thread enqueues through this library first record
 * events[i] (each a cudaEvent_t created by the caller) on the launch's
 * stream, i = 0, 1, ... up to capacity; the interval from events[i] to the
 * next recorded event therefore brackets launch i.  lm_timing_detach()
 * stops recording and returns the number of events recorded.
 * lm_timing_kinds() copies one character per recorded launch ('a' amax
 * reduction, 'c' cast, 's' scales only, 'g' GEMM, 'n' RMSNorm, 'w'
 * SwiGLU backward elementwise, 'e' softcapped CE, 'l' mean loss) into out[0..cap) and
 * returns how many it wrote; labels are kept for the first 4096 launches
 * after an attach.  State is per host thread.
 */
LM_API void lm_timing_attach(void* const* events, int capacity);
LM_API int lm_timing_detach(void);
LM_API int lm_timing_kinds(char* out, int cap);

/*
 * Self-test of the device-side failure path (no counterpart on the pages).
 * Enqueues one small kernel whose single thread waits, for at most limit_ms
 * milliseconds (1..5000), on a shared-memory barrier that nothing ever
 * arrives at.  The wait runs out, the kernel records code 0x301 in the
 * device error word and exits normally, so the next lm_get_error() returns
 * LM_ERR_TIMEOUT with where = 0x301 and the CUDA context stays usable.  Every
 * wait in the GEMM and cast kernels takes this same bounded path.
 */
LM_API lm_status lm_selftest_bounded_wait(uint32_t limit_ms, lm_stream_t stream);

/* Static, human-readable name of a status. */
LM_API const char* lm_status_string(lm_status status);

/* Library version, as major*10000 + minor*100 + patch. */
LM_API int lm_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LM_FP8_H */
