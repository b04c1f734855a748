/*
 * ttq.h -- C ABI of the TTQ linear-layer library (libttq.so, sm_100a).
 *
 * TTQ (activation-aware test-time quantization, arXiv:2603.19296) quantises
 * a linear layer's weight on the fly from the activations of the current
 * call.  For X with d input channels and T tokens and W of shape d' x d:
 *
 *   D_ii  = (||X_i,:||_p + lambda)^alpha                         (1)
 *   W_hat = Q[W D^{1/2}] D^{-1/2}                                (2)
 *   Y     = W_hat X  (+ B (A X) when a static low-rank pair is given)  (3)
 *
 * (1) and (2): gist.science/zh/paper/2603.19296, section 2.1 (online AWQ);
 * also gist.science/nl/paper/2603.19296, section 2 "Kerncomponenten" 1 and
 * gist.science/it/paper/2603.19296, section 2 "Concetti Chiave".
 * (3): gist.science/zh/paper/2603.19296, sections 2.2 (low-rank W ~ W_q + BA)
 * and 2.3 (projection cost O[d'dT]).  Q is the affine scale + zero-point
 * quantiser of blog.lo0.es "Test-time quantization without calibration
 * dataset", section "The maths that matter", applied group-wise along the
 * input dimension.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Layouts are row-major.  X is [T][d] (token-major: the pages' d x T
 *    matrix stored column by column), W is [d'][d], A is [r][d], B is [d'][r],
 *    Y is [T][d'].  D, D_rsqrt are float32 [d].
 *  - Quantised weights: codes are uint32 [d'][d*bits/32]; each row is a
 *    little-endian bit stream in which code i occupies bits [bits*i,
 *    bits*i + bits).  scales and zeros are IEEE binary16 (as uint16 bit
 *    patterns) [d'][d/group]; group k of row j covers input channels
 *    [k*group, (k+1)*group).  The weight of row j, channel i is
 *    recovered as  scales[j][k] * (code - zeros[j][k]) * D_rsqrt[i].
 *  - The quantiser runs in binary32 in this order (bit-exact contract):
 *      h = sqrtf(D_i);  x = W_ji * h;  m = min(0, min_group x);
 *      M = max(0, max_group x);  s32 = (M - m) / (2^bits - 1), floored at
 *      2^-14;  s = binary16(s32) rounded toward +inf;  inv = 1 / s;
 *      z = clamp(rint(-m * inv), 0, 2^bits - 1);
 *      q = clamp(rint(x * inv) + z, 0, 2^bits - 1);  rint rounds the
 *      exact product (no binary32 rounding before it) half to even.
 *      D == NULL means D = I (plain round-to-nearest).
 *  - All tensor pointers are DEVICE pointers, allocated and owned by the
 *    caller, and must be 16-byte aligned.  The library never allocates
 *    device memory and keeps no per-call state.  Temporary storage is the
 *    caller's workspace `ws` of `ws_bytes` >= ttq_workspace_size(...) bytes
 *    (256-byte aligned); its header (the first 20480 bytes, or all of a
 *    smaller workspace) holds a device status word and internal counters.
 *    Initialise a fresh workspace once with ttq_workspace_init.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *    only enqueues work on that stream and returns; the library never
 *    synchronises.  Calls sharing one workspace must be ordered on the GPU
 *    (same stream, or synchronised by the caller).
 *  - Errors: invalid arguments are reported synchronously by the return
 *    value and nothing is enqueued.  Conditions found on the device
 *    (non-finite input or statistic, a scale beyond binary16, an internal
 *    wait that gave up) set bits of the workspace status word and never trap
 *    or abort the context; read them with ttq_get_status after synchronising
 *    the stream.  Flags accumulate until ttq_workspace_init clears them.
 *  - No function throws; every function is safe to call from C.
 */
#ifndef TTQ_H_
#define TTQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ttq_status {
  TTQ_OK = 0,
  TTQ_ERR_INVALID_ARG = 1, /* a size, pointer, alignment or parameter is out of range */
  TTQ_ERR_UNSUPPORTED = 2, /* valid for the method but not built here (e.g. bits = 5) */
  TTQ_ERR_CUDA = 3,        /* a CUDA runtime call or kernel launch failed */
  TTQ_ERR_NONFINITE = 4,   /* device flag: NaN/Inf input, D_ii not in (0, inf), scale overflow,
                              or an activation beyond the binary16 range */
  TTQ_ERR_TIMEOUT = 5,     /* device flag: an internal pipeline wait gave up (kernel returned early) */
  TTQ_ERR_WORKSPACE = 6    /* workspace smaller than ttq_workspace_size(...) */
} ttq_status;

typedef enum ttq_dtype {
  TTQ_F32 = 0,  /* X, W, A, B and Y are float32 */
  TTQ_BF16 = 1, /* X, W, A, B and Y are bfloat16 */
  TTQ_F16 = 2   /* binary16: only for X of ttq_scale_activations and ttq_dequant_gemm */
} ttq_dtype;

/* The quantiser's code scheme (blog.lo0.es "Test-time quantization ...",
 * section "The maths that matter").  TTQ_QSCHEME_ASYMMETRIC: the range
 * [min(0, min x), max(0, max x)] over 2^bits - 1 steps with an integer zero
 * point (the default everywhere).  TTQ_QSCHEME_SYMMETRIC: levels
 * +-(2^(bits-1) - 1) with scale max|x| / (2^(bits-1) - 1); the codes are
 * stored as level + 2^(bits-1), and the zero point 2^(bits-1) is stored in
 * `zeros`, so both schemes dequantise as scales * (code - zeros).
 * TTQ_QSCHEME_FP8_E4M3 (blog.lo0.es, the comparison with FP8 end to end:
 * TTQ derives s, the code format is free): bits must be 8; the code is the
 * E4M3 value (OCP 8-bit floating point: bias 7, 3 fraction bits, largest
 * 448) nearest to the binary32 product x * (1/s), ties to even, saturating,
 * with s = binary16 round-up of max|x| / 448 per group; one byte per weight
 * (four per word, weight i in bits 8 (i mod 4) of word i / 4), zeros +0,
 * reconstruction scales * e4m3(code).  For T <= 16 tokens and d a
 * multiple of 64 the forward's product reads the 8-bit codes themselves
 * (E4M3 pairs converted to binary16 in registers), and ttq_dequant_gemm
 * takes them there; otherwise the forward materialises the binary16
 * s * e4m3(q) and multiplies by that.  INT schemes take bits 2..4. */
typedef enum ttq_qscheme {
  TTQ_QSCHEME_ASYMMETRIC = 0,
  TTQ_QSCHEME_SYMMETRIC = 1,
  TTQ_QSCHEME_FP8_E4M3 = 2
} ttq_qscheme;

/* Device status word bits (ttq_get_status). */
#define TTQ_FLAG_NONFINITE 0x1u
#define TTQ_FLAG_SCALE_OVERFLOW 0x2u
#define TTQ_FLAG_TIMEOUT 0x4u
#define TTQ_FLAG_X_RANGE 0x8u /* an activation beyond the binary16 range (|x| > 65504) */
#define TTQ_FLAG_RANK_DEFICIENT 0x10u /* ttq_lowrank_init: W's sampled range had fewer than
                                         r + oversample independent directions (a Cholesky
                                         pivot was not positive and was floored) */

/* Byte offsets of the workspace regions for one problem shape (all 256-byte
 * aligned); `total` equals ttq_workspace_size(...).  After
 * ttq_linear_forward the regions hold that call's intermediates: D and
 * D_rsqrt as float32 [d], A X as bf16 [T][ax_ld], and the codes/scales/
 * zeros of W_hat where the product read them (INT codes at 17 to 256
 * tokens and with a non-bf16 or symmetric layer at up to 16; FP8 codes at
 * up to 16 tokens).  Where the product read the materialised binary16 W_hat
 * (wq: more than 256 tokens; FP8 above 16) that alone is kept, no codes;
 * the single-pass product (bf16, asymmetric, up to 16 tokens) keeps
 * neither.  Offsets of regions the shape does not use are 0 with
 * size 0.  Returns TTQ_ERR_INVALID_ARG for an unsupported shape. */
typedef struct ttq_workspace_layout {
  size_t status;  /* uint32 status word, then internal counters */
  size_t D;       /* float32 [d]   D_ii                          */
  size_t D_rsqrt; /* float32 [d]   D_ii^(-1/2)                   */
  size_t partial; /* float64 [splits][d] partial sums of |x|^p   */
  size_t codes;   /* uint32 [d'][d*bits/32]                      */
  size_t scales;  /* uint16 [d'][d/group]                        */
  size_t zeros;   /* uint16 [d'][d/group]                        */
  size_t ax;      /* bf16 [T][ax_ld]  A X                        */
  size_t xh;      /* binary16 [T][d] X D^{-1/2} for the product   */
  size_t xb;      /* bf16 [T][d] copy of float32 X (TTQ_F32, r > 0) */
  size_t ab;      /* bf16 copies of float32 A and B (TTQ_F32, r > 0) */
  size_t wq;      /* binary16 [d'][d] s (q - z) (s e4m3(q) for 8-bit codes)
                     that ttq_linear_forward's product reads when T > 256, or
                     for 8-bit codes beyond the decode product's reach
                     (T > 16 or d % 64 != 0); 0: not in this layout */
  size_t total;
  int64_t splits; /* number of token splits of the statistic pass */
  int64_t ax_ld;  /* row stride (elements) of A X                 */
  size_t axp;     /* float32 [ax_splits][T][r] partial sums of A X split along d
                     (0 when A X is not split) */
  size_t D_sqrt;  /* float32 [d] sqrtf(D_ii) for the single-pass decode product */
  size_t ypart;   /* float32 partial output tiles of the single-pass decode product
                     (T <= 16), or float32 [splits][T][d'] partial sums of the
                     product on wq when it is split along K (T > 256 and few
                     output tiles); 0: not in this layout */
  size_t tickets; /* uint32 arrival tickets of its 256-row tiles (inside the
                     zeroed header; 0: not in this layout) */
  int64_t ax_splits; /* K splits of the A X product (1: none; 0 when r == 0) */
} ttq_workspace_layout;

/* Workspace bytes needed by every entry point below for this shape
 * (d' = dp, rank r; r = 0 means no low-rank term).  0 if the shape is
 * unsupported. */
size_t ttq_workspace_size(int64_t d, int64_t dp, int64_t T, int64_t r, int bits,
                          int group, ttq_dtype dtype);

ttq_status ttq_workspace_get_layout(int64_t d, int64_t dp, int64_t T, int64_t r,
                                    int bits, int group, ttq_dtype dtype,
                                    ttq_workspace_layout* out);

/* Clears the header of a workspace: the status word and internal counters,
 * the first min(ws_bytes, 20480) bytes (enqueued on `stream`; ws_bytes must
 * be at least 4096).  Call once after allocating a workspace, to reset flags,
 * and after TTQ_ERR_TIMEOUT. */
ttq_status ttq_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Step (1), the per-channel activation statistic
 * (gist.science/zh/paper/2603.19296, section 2.1):
 *   D[i] = (||X[:, i]||_p + lambda)^alpha,  D_rsqrt[i] = D[i]^(-1/2).
 * X [T][d] (dtype), d % 8 == 0, T >= 0, p >= 1, lambda >= 0, alpha >= 0.
 * The L_p norm is taken over the T tokens of this call (no 1/T factor).
 * |x|^p is summed in fp64, split over tokens and merged in a fixed order,
 * so the result is deterministic; n, D and D^{-1/2} are formed in fp64 and
 * rounded once to binary32.  D or D_rsqrt may be NULL (then they are still written
 * to the workspace).  Flags NONFINITE if any D[i] is not finite and > 0. */
ttq_status ttq_act_norm(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                        float p, float lambda, float alpha, float* D,
                        float* D_rsqrt, void* ws, size_t ws_bytes, void* stream);

/* Step (1) together with the B operand of the product, in one pass over X:
 * D and D_rsqrt exactly as ttq_act_norm computes them
 * (gist.science/zh/paper/2603.19296, section 2.1), and
 *   Xs[t][i] = binary16(X[t][i] * D_rsqrt[i])
 * exactly as ttq_scale_activations computes it (the D^{-1/2} factor of
 * W_hat = Q[W D^{1/2}] D^{-1/2}, carried by X).  X [T][d] in TTQ_F32 or
 * TTQ_BF16, d % 8 == 0; Xs binary16 [T][d] (uint16 bit patterns), required
 * when T > 0; D and D_rsqrt float32 [d] or NULL (then written to the
 * workspace only).  The token splits are those of ttq_act_norm (the
 * layout's `splits`): for T <= 2048, enough for about two 128-channel
 * blocks per SM and for at most 256 rows each, at most 8; for longer T,
 * at most 16.  When there are at most 8 splits of at most 256 rows (128 for
 * float32 X), this is one kernel that reads X from HBM once and keeps it in
 * registers, the splits of a column block forming one thread-block cluster;
 * otherwise it is the two kernels of ttq_act_norm and
 * ttq_scale_activations.  The results are the same bits either way.  The
 * workspace is the one ttq_act_norm needs (it must have been cleared by
 * ttq_workspace_init once; the call leaves its counters at zero).  Flags as
 * ttq_act_norm and ttq_scale_activations (NONFINITE, X_RANGE). */
ttq_status ttq_act_norm_scale(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                              float p, float lambda, float alpha, float* D,
                              float* D_rsqrt, uint16_t* Xs, void* ws, size_t ws_bytes,
                              void* stream);

/* ttq_act_norm without a workspace, for callers that cannot allocate device
 * memory: for example a plug-in that runs inside another framework's memory
 * manager and may neither call cudaMalloc nor reserve a buffer of its own,
 * or a real-time loop that must not allocate once it has started.  The
 * method has no counterpart to this entry point (an interface choice of this
 * library, not a step of the paper).
 *   Same inputs, outputs and results as ttq_act_norm, except that D and
 * D_rsqrt are required.  The scratch memory (fp64 partial sums, merge
 * tickets, a status word) is one array compiled into the library: every GPU
 * that loads the library holds 2 MiB + 4 KiB for it until the process exits,
 * and d may be at most 16384 (larger d returns TTQ_ERR_UNSUPPORTED).
 *   The first call on a device looks up the array's device address on the
 * current device; make that first call before any stream capture.  Every
 * later call checks that the cached address still names device memory of
 * that device and looks it up again if not (after cudaDeviceReset, or once
 * the primary context was released and created anew, the array may sit
 * elsewhere; make the first call after such a reset outside a capture too).  All calls
 * share the one array, so calls whose work overlaps on the GPU (other
 * streams, other threads) race: order them on one stream.  Each call clears
 * the array's status word and tickets first; device flags are not reported
 * (a non-finite input shows up as a non-finite D).  The array keeps the last
 * call's partial sums. */
ttq_status ttq_act_norm_noalloc(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                                float p, float lambda, float alpha, float* D,
                                float* D_rsqrt, void* stream);

/* Step (2) without the rescale: codes, scales and zeros of Q[W D^{1/2}]
 * (gist.science/zh/paper/2603.19296, section 2.1; quantiser of blog.lo0.es
 * "The maths that matter"), in the binary32 order stated above.
 * W [dp][d] (dtype); D float32 [d] or NULL (identity).  bits in {2, 3, 4};
 * group in {32, 64, 128, 256} with d % group == 0.  Outputs as described
 * above.  Flags NONFINITE for a non-finite W*sqrt(D) and SCALE_OVERFLOW
 * (with NONFINITE) for a group whose scale, or scale * (2^bits - 1), exceeds
 * binary16. */
ttq_status ttq_quantize_weight(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                               const float* D, int bits, int group, uint32_t* codes,
                               uint16_t* scales, uint16_t* zeros, void* ws,
                               size_t ws_bytes, void* stream);

/* ttq_quantize_weight with a choice of code scheme and an optional
 * dequantised binary16 weight (as ttq_quantize_dequant_weight writes it;
 * W_hat may be NULL).  With W_hat given, codes, scales and zeros may all
 * be NULL: then W_hat alone is written (the same values; the flags as
 * with the codes).  With TTQ_QSCHEME_SYMMETRIC the binary32 order is
 *   h = sqrtf(D_i); x = W_ji * h; M = max_group |x|;
 *   s32 = M / (2^(bits-1) - 1), floored at 2^-14; s = binary16 round-up;
 *   inv = 1 / s; level = clamp(rint(x * inv), -(2^(bits-1)-1), 2^(bits-1)-1)
 *   (exact product, half to even); code = level + 2^(bits-1);
 *   zeros = 2^(bits-1)
 * (a finite group never needs the clamp).  Flags as ttq_quantize_weight
 * (SCALE_OVERFLOW when s * (2^(bits-1) - 1) exceeds binary16). */
ttq_status ttq_quantize_weight_ex(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                                  const float* D, int bits, int group, ttq_qscheme scheme,
                                  uint32_t* codes, uint16_t* scales, uint16_t* zeros,
                                  uint16_t* W_hat, void* ws, size_t ws_bytes, void* stream);

/* ttq_quantize_weight that also writes the dequantised weight
 *   W_hat[j][i] = binary16(s[j][k] * (q[j][i] - z[j][k]))
 * (binary16 bit patterns, [dp][d] row-major, 16-byte aligned; required
 * when dp > 0): W_hat of the paper (gist.science/zh/paper/2603.19296,
 * section 2.1) without its D^{-1/2} factor, which the product's other
 * operand X D^{-1/2} carries.  q - z is exact and the product is rounded
 * once, so these are the operand values ttq_dequant_gemm forms from the
 * codes.  codes, scales and zeros may all be NULL (W_hat alone is written,
 * as the forward does when it materialises the weight).  Everything else
 * as ttq_quantize_weight. */
ttq_status ttq_quantize_dequant_weight(const void* W, ttq_dtype dtype, int64_t dp, int64_t d,
                                       const float* D, int bits, int group, uint32_t* codes,
                                       uint16_t* scales, uint16_t* zeros, uint16_t* W_hat,
                                       void* ws, size_t ws_bytes, void* stream);

/* The B operand of the product: Xs[t][i] = binary16(X[t][i] * D_rsqrt[i])
 * (the D^{-1/2} factor of W_hat = Q[W D^{1/2}] D^{-1/2}, carried by X;
 * gist.science/zh/paper/2603.19296, section 2.1).  X [T][d] in dtype (F32,
 * BF16 or F16), D_rsqrt float32 [d] or NULL (identity), Xs binary16 [T][d]
 * (uint16 bit patterns); d % 8 == 0.  Each product is rounded once to
 * binary16; flags X_RANGE if some |Xs| > 65504.  Needs a workspace of at
 * least 4096 bytes (status word). */
ttq_status ttq_scale_activations(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                                 const float* D_rsqrt, uint16_t* Xs, void* ws,
                                 size_t ws_bytes, void* stream);

/* Steps (2)-(3) from already quantised weights: Y = W_hat X (+ B (A X)),
 * with W_hat[j][i] = scales[j][k] (codes[j][i] - zeros[j][k]) D_rsqrt[i],
 * on the tensor cores as (s (q - z)) x (X D^{-1/2}): binary16 operands (the
 * first formed in shared memory, the second written to the workspace;
 * |x D^{-1/2}| and s (2^bits - 1) must not exceed 65504, else flag
 * X_RANGE / SCALE_OVERFLOW), fp32 accumulation; the low-rank term B (A X)
 * uses bf16 operands with fp32 accumulation, A X held in bf16.
 * D_rsqrt == NULL means D = I.  A [r][d] and B [dp][r] (dtype) may be NULL
 * when r == 0; r % 8 == 0.  dtype TTQ_F16 means X is binary16 and already
 * holds X D^{-1/2} when D_rsqrt is NULL (as written by
 * ttq_scale_activations): then only the product runs; it needs r == 0.
 * Y [T][dp] is written in y_dtype (TTQ_F32 or TTQ_BF16): TTQ_F32 keeps the
 * fp32 accumulator as is, TTQ_BF16 rounds it to nearest-even once.
 * bits = 8 takes FP8 (E4M3) codes (TTQ_QSCHEME_FP8_E4M3, zeros ignored)
 * for T <= 16 and d a multiple of 64 only (else TTQ_ERR_UNSUPPORTED). */
ttq_status ttq_dequant_gemm(const uint32_t* codes, const uint16_t* scales,
                            const uint16_t* zeros, const float* D_rsqrt,
                            const void* X, const void* A, const void* B,
                            ttq_dtype dtype, int64_t d, int64_t dp, int64_t T,
                            int64_t r, int bits, int group, void* Y,
                            ttq_dtype y_dtype, void* ws, size_t ws_bytes,
                            void* stream);

/* Step (3) on a dequantised weight: Y[t][j] = sum_i W_hat[j][i] Xs[t][i]
 * (gist.science/zh/paper/2603.19296, section 2.3), on the tensor cores
 * with binary16 operands and fp32 accumulation.  W_hat binary16 [dp][d]
 * (as written by ttq_quantize_dequant_weight), Xs binary16 [T][d] (X
 * D^{-1/2}, as written by ttq_scale_activations); d % 8 == 0; all pointers
 * 16-byte aligned.  Y [T][dp] in y_dtype (TTQ_F32 or TTQ_BF16, rounded
 * once).  No low-rank term.  Needs a workspace of at least 4096 bytes
 * (status word).  For more than 256 tokens and a shape with few output
 * tiles (d' small against T and d: a long K), the product is split along K
 * exactly as ttq_linear_forward splits it: the splits' float32 partial sums
 * go to the workspace after its 20480-byte header and are added in split
 * order, rounded once.  It does so when the workspace spans
 * ttq_dequantized_gemm_workspace_size(d, dp, T) bytes, and then gives the
 * forward's bits; with a smaller workspace it runs unsplit (the same
 * product, its fp32 sums in another order). */
ttq_status ttq_dequantized_gemm(const uint16_t* W_hat, const uint16_t* Xs, int64_t d,
                                int64_t dp, int64_t T, void* Y, ttq_dtype y_dtype, void* ws,
                                size_t ws_bytes, void* stream);

/* Workspace bytes at which ttq_dequantized_gemm takes the forward's K split
 * for this shape (4096 when it never splits); 0 for an invalid shape.  An
 * interface query of this library; the method has no counterpart. */
size_t ttq_dequantized_gemm_workspace_size(int64_t d, int64_t dp, int64_t T);

/* The whole TTQ linear layer, (1) -> (2) -> (3), on `stream`:
 *   Y = Q[W D^{1/2}] D^{-1/2} X + B (A X).
 * X [T][d], W [dp][d], A [r][d], B [dp][r] in `dtype`; Y [T][dp] in
 * `y_dtype` (TTQ_F32: the fp32 accumulator; TTQ_BF16: rounded once to
 * nearest-even).  A and B may be NULL when r == 0.  W is taken to be the
 * residual that the static low-rank pair complements (gist.science/zh,
 * section 2.2).  The workspace keeps D and D_rsqrt of this call and the
 * quantised weight in the form the product read (see ttq_workspace_layout).
 * For T > 256 the quantiser writes the dequantised weight s (q - z) in
 * binary16 to the workspace (layout field wq) instead of the codes, and the
 * product reads it as a plain tensor-core operand, so that no 256-token
 * tile dequantises the codes again (where few output tiles would leave
 * most SMs to one long K loop, that product is split along K and the
 * float32 partial sums are added in split order, layout field ypart); for
 * 17 <= T <= 256 the product
 * dequantises the codes itself (as ttq_dequant_gemm does); for T <= 16
 * (bf16, asymmetric codes) one kernel quantises W in registers and
 * multiplies (as ttq_quantize_gemm).  All give the same operand values. */
ttq_status ttq_linear_forward(const void* X, const void* W, const void* A,
                              const void* B, ttq_dtype dtype, int64_t d, int64_t dp,
                              int64_t T, int64_t r, float p, float lambda, float alpha,
                              int bits, int group, void* Y, ttq_dtype y_dtype, void* ws,
                              size_t ws_bytes, void* stream);

/* ttq_linear_forward with a choice of code scheme (TTQ_QSCHEME_ASYMMETRIC
 * is exactly ttq_linear_forward). */
ttq_status ttq_linear_forward_ex(const void* X, const void* W, const void* A,
                                 const void* B, ttq_dtype dtype, int64_t d, int64_t dp,
                                 int64_t T, int64_t r, float p, float lambda, float alpha,
                                 int bits, int group, ttq_qscheme scheme, void* Y,
                                 ttq_dtype y_dtype, void* ws, size_t ws_bytes, void* stream);

/* Number of kernels one ttq_linear_forward_ex call with these sizes and
 * this code scheme enqueues on the current device (host query; no device
 * work), in *kernels: the statistic pass (fused with the scaling of X when
 * it fits, see ttq_act_norm_scale), the quantiser and the product (one
 * kernel together where the forward takes the single-pass decode product,
 * see ttq_quantize_gemm; plus the reduction of its K splits where the
 * product on the materialised weight is split), and for r > 0 the A X
 * product (plus the
 * reduction of its K splits, and two bf16 conversions of a float32 A and
 * B).  An interface query of this library; the method has no counterpart. */
ttq_status ttq_linear_forward_kernels(ttq_dtype dtype, int64_t d, int64_t dp, int64_t T,
                                      int64_t r, float p, int bits, int group,
                                      ttq_qscheme scheme, int* kernels);

/* Steps (2)-(3) in one pass over the weight, for a few tokens: reads bf16 W
 * once, forms Q[W D^{1/2}] group by group in the binary32 order stated at
 * the top of this file, and multiplies it with the binary16 X D^{-1/2} on
 * the tensor cores, so that the codes never travel through memory
 * (gist.science/zh/paper/2603.19296, section 2.1 for W_hat, section 2.3 for
 * the cost it attacks: at decode the 3d'd test-time term outweighs the
 * d'dT product, and reading W once is its floor).
 *   Y [T][d'] (y_dtype) = sum_i s (q - z) Xs[t][i]  (+ B (A X) when r > 0),
 * accumulated in fp32 (each group's sum of (q - z) Xs is scaled by s once).
 * W bf16 [dp][d]; D float32 [d]; Xs binary16 [T][d] = X D^{-1/2} as
 * ttq_act_norm_scale writes it; A [r][d], B [dp][r] and X [T][d] bf16 (only
 * for r > 0).  codes, scales, zeros: NULL, or all three given and filled
 * exactly as ttq_quantize_weight fills them (same bits).
 *   Limits: 1 <= T <= 16, d a multiple of 128, bits 2..4, group 32, 64 or
 * 128, dp <= 1048576 (else TTQ_ERR_UNSUPPORTED).  Workspace as for
 * ttq_linear_forward (TTQ_BF16) of the same sizes; its tile tickets start at
 * zero (ttq_workspace_init) and every call leaves them at zero.  Flags as
 * ttq_quantize_weight, and TIMEOUT (then re-initialise the workspace).
 * ttq_linear_forward takes this product itself for bf16 layers with the
 * asymmetric codes and at most 16 tokens (without storing codes). */
ttq_status ttq_quantize_gemm(const void* W, const float* D, const uint16_t* Xs, const void* A,
                             const void* B, const void* X, int64_t d, int64_t dp, int64_t T,
                             int64_t r, int bits, int group, uint32_t* codes, uint16_t* scales,
                             uint16_t* zeros, void* Y, ttq_dtype y_dtype, void* ws,
                             size_t ws_bytes, void* stream);

/* Reads the workspace status word (a blocking device-to-host copy; the caller
 * synchronises its stream first).  *flags receives the raw TTQ_FLAG_* bits
 * (may be NULL).  Returns ttq_status_from_flags of those bits.
 *   After TTQ_ERR_TIMEOUT the workspace must be reset with
 * ttq_workspace_init before its next use: a statistic pass whose barrier
 * among its blocks gave up leaves that barrier's counter off zero, and the
 * next call would otherwise start from it. */
ttq_status ttq_get_status(const void* ws, uint32_t* flags);

/* The status that a set of TTQ_FLAG_* bits stands for (host only, no device
 * work): TTQ_ERR_TIMEOUT if the timeout flag is set; else TTQ_ERR_NONFINITE
 * if any other bit except TTQ_FLAG_RANK_DEFICIENT is set (a non-finite
 * value, a binary16 scale overflow, an activation beyond binary16, or a bit
 * this version does not define); else TTQ_OK.  TTQ_FLAG_RANK_DEFICIENT is a
 * warning: a weight of rank below r + oversample is a valid input to
 * ttq_lowrank_init, whose outputs stay finite. */
ttq_status ttq_status_from_flags(uint32_t flags);

/* ---------------------------------------------------------------------
 * Static low-rank initialisation (the step before the path).
 *
 * gist.science/zh/paper/2603.19296, section 2.2 (and gist.science/nl/paper/
 * 2603.19296, section 2 "Kerncomponenten", item 3): W ~ W_q + B A, with the
 * static factors B, A initialised by PCA and W_q the quantised residual.
 * PCA of W is read as W's uncentred truncated SVD: B = U_r S_r [dp][r] and
 * A = V_r^T [r][d] (A's rows orthonormal, B = W A^T), computed by a
 * randomised range finder with `power_iters` subspace iterations (Halko,
 * Martinsson, Tropp 2011) on the caller's Gaussian test matrix Omega
 * [d][r + oversample] (float32, row-major; the random draws are an input).
 * The closer the spectrum of W is to having a gap after r, and the more
 * iterations, the closer B A is to the exact truncated SVD.
 *
 * W, B, A and W_res share `dtype` (TTQ_F32 or TTQ_BF16), row-major.
 * W_res = W - B A (with B, A as stored, i.e. rounded to dtype) [dp][d] is
 * written when non-NULL; it is the weight to pass to ttq_linear_forward
 * together with A and B.  Requirements: 1 <= r, oversample >= 0,
 * r + oversample <= min(96, dp, d), 0 <= power_iters <= 16, ws of at least
 * ttq_lowrank_workspace_size(dp, d, r, oversample) bytes, initialised with
 * ttq_workspace_init.  Device-side conditions set TTQ_FLAG_RANK_DEFICIENT
 * or TTQ_FLAG_NONFINITE in the workspace status word.  Asynchronous on
 * `stream`; deterministic for given inputs. */
size_t ttq_lowrank_workspace_size(int64_t dp, int64_t d, int64_t r, int64_t oversample);
ttq_status ttq_lowrank_init(const void* W, ttq_dtype dtype, int64_t dp, int64_t d, int64_t r,
                            int64_t oversample, int power_iters, const float* Omega, void* B,
                            void* A, void* W_res, void* ws, size_t ws_bytes, void* stream);

/* Static description of a status code. */
const char* ttq_status_string(ttq_status s);

/* Library version, e.g. "0.1.0". */
const char* ttq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TTQ_H_ */
