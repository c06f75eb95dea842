/*
 * kq.h -- W4A4 quantized linear layer for diffusion Transformers on NVIDIA B200 (sm_100a).
 *
 * The layer computes Y = X W (row-vector convention: X [M, K] tokens x features,
 * W [K, N]) through a 4-bit x 4-bit contraction:
 *
 *   mu_m  = mean_k X[m, k]                      (optional per-token centring)
 *   Xt    = (X - mu 1^T) P                      (invertible block transform on 32-blocks)
 *   Y     = deq(Q(Xt)) deq(Q(R)) + U L2 + mu s  (MXFP4 GEMM + low-rank + rank-1 branches)
 *
 * with, prepared once per layer: W' = P^-1 W, W' ~ L1 L2 (rank r, bf16 factors),
 * R = W' - L1 L2 in MXFP4, s = 1^T W, and online U = Xt L1. The low-rank branch runs in
 * 16 bits: U is held as fp16 (saturated at +-65504, which the device error word reports)
 * and multiplied with L2 (bf16 values, held as fp16) on the tensor cores with fp32
 * accumulation.
 *
 * Sources (commentary pages on the methods):
 *   - KroQuant: Kronecker-Structured Block Transforms for Efficient Post-Training
 *     Quantization of Diffusion Transformers -- section 01 (Y = (X P)(P^-1 W)),
 *     section 02 (P = A (x) B on 32-element blocks), section 03 (MXFP4).
 *   - OrbitQuant (data-free quantization for image and video DiTs) -- section 03,
 *     equation RPBH(X) = X P H D and the offline fold W' = R^-1 W.
 *   - CentriQ: Calibration-Free Quantization of Diffusion Transformers via Exact
 *     Mean Centering -- abstract (centre each token before the rotation, restore the
 *     mean exactly through a rank-1 full-precision branch).
 *   - SVDQuant explainer -- section 3 (SVD of the updated weight; top-r part kept in
 *     16 bits, residual quantized to 4 bits; low-rank work fused into the 4-bit kernel).
 *   MXFP4 itself follows the OCP Microscaling Formats v1.0 rule: E2M1 elements, one
 *   E8M0 scale 2^e per 32 elements along K, e = floor(log2(amax)) - 2 clamped to
 *   [-127, 127], round to nearest even, saturate at +-6.
 *
 * Conventions for every call:
 *   - Ownership: the caller allocates and owns every device buffer (for example as
 *     torch tensors). The library never calls cudaMalloc. Host arrays reached through
 *     descriptors are read during the call only.
 *   - Streams: work is enqueued asynchronously on `stream` (0 = legacy default stream).
 *     Buffers must stay alive until that work completes.
 *   - Errors: argument, shape and alignment problems are found on the host and
 *     returned before anything is launched. CUDA launch errors return KQ_ERR_CUDA.
 *     Device-side problems (a bounded wait that ran out, a low-rank activation outside
 *     the fp16 range) set bits of an error word in the activation workspace;
 *     kq_last_device_error() reports and clears it. Nothing aborts or traps.
 *   - Alignment: device pointers 16-byte aligned (what TMA needs of a global address);
 *     K % 32 == 0, N % 16 == 0, M >= 1 arbitrary; rank <= 64.
 *   - Determinism: outputs are bitwise reproducible run to run.
 */
#ifndef KQ_H_
#define KQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (same type as cudaStream_t). */
typedef struct CUstream_st *kq_stream_t;

typedef enum {
  KQ_OK = 0,
  KQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad enum */
  KQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 32 != 0, N % 16 != 0, rank > 64, ... */
  KQ_ERR_ALIGNMENT = 3,          /* a device pointer is not 16-byte aligned */
  KQ_ERR_SINGULAR_TRANSFORM = 4, /* A or B of the Kronecker transform is not invertible */
  KQ_ERR_WORKSPACE_TOO_SMALL = 5,/* a caller buffer is smaller than the size query says */
  KQ_ERR_CUDA = 6,               /* a CUDA runtime/driver/library call failed */
  KQ_ERR_DEVICE_TIMEOUT = 7,     /* a device-side bounded wait ran out (see kq_last_device_error) */
  KQ_ERR_NO_SM100 = 8,           /* the current device is not compute capability 10.0 */
  KQ_ERR_LOWRANK_RANGE = 9       /* a low-rank activation U lay outside the fp16 range and was
                                    saturated at +-65504 (or was not a number); the output
                                    of that call is not to be trusted */
} kq_status;

typedef enum { KQ_T_NONE = 0, KQ_T_KRON = 1, KQ_T_RPBH = 2 } kq_transform_kind;
typedef enum { KQ_OUT_F32 = 0, KQ_OUT_BF16 = 1 } kq_out_dtype;

/* Activation format.
 *   KQ_CB_MXFP4: MXFP4 (OCP E2M1 elements, one E8M0 scale per 32 along K), contracted by
 *     the block-scaled FP4 tensor-core MMA (KroQuant section 03).
 *   KQ_CB_LLOYDMAX: OrbitQuant's single 16-level Lloyd-Max codebook of N(0, 1) for the
 *     rotated coordinates (OrbitQuant section 03) with CentriQ's closed-form per-token
 *     scale (abstract): sigma_m = RMS of the rotated (centred) token, each value the
 *     level nearest to Xt / sigma_m (magnitude by midpoint thresholds, a magnitude on a
 *     threshold taking the larger level; sign of Xt). The tensor cores have no codebook
 *     format, so the decoded operand fp16(fp32(sigma_m) * fp32(level)) is stored and the
 *     weights' MXFP4 residual is decoded to fp16 offline: the contraction is an fp16
 *     tensor-core GEMM (a quarter of the FP4 rate, four times the operand bytes). Needs
 *     the RPBH transform (whose coordinates the codebook is designed for) or none, and
 *     no LayerNorm front-end. */
typedef enum { KQ_CB_MXFP4 = 0, KQ_CB_LLOYDMAX = 1 } kq_act_format;

/* The online block transform P (KroQuant section 02; OrbitQuant section 03).
 * All pointers are HOST memory, read during the call.
 *   KQ_T_KRON: P = blockdiag(A (x) B) over the K/32 blocks, A a_dim x a_dim and
 *              B b_dim x b_dim row-major float32, a_dim = 4, b_dim = 8. Within a block
 *              element 8 i + j has (A (x) B)[(i,j),(k,l)] = A[i,k] B[j,l].
 *   KQ_T_RPBH: P = Pi blockdiag(H32 / sqrt(32)) D: x -> x[perm[j]] (gather), then a
 *              Sylvester Hadamard on each 32-block, then multiply by sign[j] (+1/-1).
 *              perm: int32 [K], a permutation of 0..K-1; sign: int8 [K].
 *   KQ_T_NONE: P = I. */
typedef struct {
  int32_t kind;          /* kq_transform_kind */
  const float *A;        /* KRON: host [a_dim * a_dim] */
  int32_t a_dim;
  const float *B;        /* KRON: host [b_dim * b_dim] */
  int32_t b_dim;
  const int32_t *perm;   /* RPBH: host [K] */
  const int8_t *sign;    /* RPBH: host [K] */
} kq_transform_desc;

/* Optional LayerNorm front-end, fused into the online half (the KroQuant commentary,
 * section 01: normalisation layers between the blocks are why the transform runs online).
 * Per token, over the K channels:  y = (x - m) / sqrt(v + eps) * gamma + beta  with
 * m the mean and v the biased variance; then the layer runs on y (centring, transform,
 * MXFP4, low-rank branch, mean restore). Requires center == 1 (the normalised token is
 * centred); not available to kq_smooth_quantize_act. gamma and beta are read only by
 * kq_prepare_weights / kq_weights_pack, which copy them into the prepared weights with
 * the low-rank map diag(gamma) L1' and the sums gamma^T L1', beta^T L1' (KQ_ERR_INVALID_ARG
 * there if a pointer is null or a value is not finite); later calls need on and eps only.
 * The activation workspace then also holds each token's m and 1/sqrt(v + eps) (0 for a
 * token with zero variance, which normalises to beta exactly).
 * Conditioning: the low-rank input is formed from raw x as
 * rstd (x diag(gamma) L1' - m gamma^T L1') + beta^T L1' - mean(y) c1, so its absolute error
 * is about 2^-24 (|m| / sqrt(v + eps)) sum_k |gamma_k L1'_k| from fp32 accumulation: small
 * for tokens whose mean is within a few standard deviations of zero (DiT residual streams),
 * large for nearly constant tokens with a large mean. */
typedef struct {
  int32_t on;            /* 1: front-end on */
  float eps;             /* > 0 */
  const float *gamma;    /* host [K], per-channel scale */
  const float *beta;     /* host [K], per-channel shift */
} kq_layernorm_desc;

/* One linear layer. The same descriptor (same values) must be passed to
 * kq_prepare_weights and to every later call that uses the prepared weights. */
typedef struct {
  int32_t K;             /* input features, K % 32 == 0 */
  int32_t N;             /* output features, N % 16 == 0 */
  int32_t rank;          /* low-rank branch rank r, 0..64 */
  int32_t center;        /* 1: per-token mean centring with rank-1 restore (CentriQ) */
  kq_transform_desc t;
  kq_layernorm_desc ln;  /* zero-initialised: no front-end */
  int32_t codebook;      /* kq_act_format; 0 (MXFP4) when zero-initialised */
} kq_layer_desc;

/* ---------------------------------------------------------------------------------
 * Sizes. Both return 0 for an invalid descriptor.
 * ------------------------------------------------------------------------------- */

/* Bytes of the prepared-weights buffer for this layer (residual codes and scales,
 * low-rank factors, column sums, transform tables). */
size_t kq_weights_bytes(const kq_layer_desc *desc);

/* Bytes of the activation workspace for M tokens: MXFP4 codes, block scales in the
 * tensor-core layout, token means, low-rank activations U (fp16), and a small header
 * holding the device error word. */
size_t kq_act_bytes(const kq_layer_desc *desc, int32_t M);

/* ---------------------------------------------------------------------------------
 * Offline weight preparation (once per layer). OrbitQuant section 03 (fold the
 * inverse transform into the weight offline), SVDQuant explainer section 3 (SVD
 * low-rank branch in 16 bits, 4-bit residual), CentriQ abstract (s = 1^T W for the
 * rank-1 mean restore).
 *   W_bf16:  device, bf16 [K, N] row-major (Y = X W).
 *   weights: device, kq_weights_bytes(desc) bytes, written.
 *   ws:      device scratch of at least kq_prepare_ws_bytes(desc) bytes.
 * Computes s = 1^T W, W' = P^-1 W (float64), the rank-r truncated SVD of W'
 * (float64, through cuSOLVER), L1 = bf16(U_r S_r^1/2), L2 = bf16(S_r^1/2 V_r^T),
 * R = W' - L1 L2 rounded to float32 and MXFP4-encoded along K, L1' = P L1 and
 * c1 = 1^T L1'. Synchronous on `stream` (it waits for the solver).
 * Errors: KQ_ERR_SINGULAR_TRANSFORM if A or B cannot be inverted. */
size_t kq_prepare_ws_bytes(const kq_layer_desc *desc);
kq_status kq_prepare_weights(const kq_layer_desc *desc, const void *W_bf16, void *weights,
                             void *ws, size_t ws_bytes, kq_stream_t stream);

/* kq_prepare_weights with the residual's MXFP4 block scales fitted under a robust l_p
 * objective (CentriQ summary and abstract: weights fitted with an l_p objective that tracks
 * each group's dense mode while discounting heavy tails). Per 32-element block of R the
 * candidates are the OCP exponent and the three below it; the codes at each are the usual
 * round-to-nearest-even, saturating ones; the block keeps the candidate with the smallest
 * sum |r - deq|^p (float64), ties to the larger exponent. Everything else is as in
 * kq_prepare_weights (same buffers, same sizes). p in (0, 2], else KQ_ERR_INVALID_ARG. */
kq_status kq_prepare_weights_lp(const kq_layer_desc *desc, double p, const void *W_bf16,
                                void *weights, void *ws, size_t ws_bytes, kq_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Online activation quantization (every denoising step, every layer; KroQuant
 * section 01 explains why it must run online). CentriQ abstract (centring),
 * KroQuant section 02 / OrbitQuant section 03 (block transform), KroQuant
 * section 03 (MXFP4), SVDQuant section 3 (low-rank input U = Xt L1).
 *   X_bf16: device, bf16 [M, K] row-major.
 *   act:    device workspace of kq_act_bytes(desc, M) bytes, written.
 * ------------------------------------------------------------------------------- */
kq_status kq_quantize_act(const kq_layer_desc *desc, const void *weights, const void *X_bf16,
                          int32_t M, void *act, size_t act_bytes, kq_stream_t stream);

/* Comparator of KroQuant section 02 (the SmoothQuant channel-wise scaling its
 * quantization kernel is measured against): the activation is multiplied per channel by
 * inv_s (fp32, device, [K]; inv_s[k] = 1/s_k with SmoothQuant's s_k = max|X_k|^a /
 * max|W_k|^(1-a)), each product rounded to fp32, then MXFP4-encoded along K into the
 * activation workspace (codes and scales in the layout kq_gemm reads; means set to 0).
 * Same kernel and pipeline as kq_quantize_act, only the transform differs. The layer
 * descriptor must have no transform, no centring and rank 0 (else KQ_ERR_INVALID_ARG);
 * the matching weights are kq_prepare_weights of diag(s) W for that descriptor.
 * inv_s must be 16-byte aligned. Async on `stream`. */
kq_status kq_smooth_quantize_act(const kq_layer_desc *desc, const float *inv_s,
                                 const void *X_bf16, int32_t M, void *act, size_t act_bytes,
                                 kq_stream_t stream);

/* The whole layer: kq_quantize_act followed by the block-scaled FP4 GEMM with the
 * low-rank (U L2) and rank-1 (mu s) branches fused into its accumulator/epilogue
 * (SVDQuant section 3: low-rank work fused into the 4-bit kernel).
 *   Y: device, [M, N] row-major, float32 or bf16 per out_dtype, written. */
kq_status kq_linear(const kq_layer_desc *desc, const void *weights, const void *X_bf16,
                    int32_t M, void *Y, int32_t out_dtype, void *act, size_t act_bytes,
                    kq_stream_t stream);

/* The same layer from HOST buffers: copies X (pinned host, bf16 [M, K]) to the device
 * buffer X_dev [M, K], runs the layer, and copies Y back into Y_host (pinned host) from
 * Y_dev [M, N]. For M >= 1024 the rows go in up to 8 chunks (a multiple of 128 rows,
 * >= 512 each): the copy-in of a chunk, the kernels of the previous one and the copy-out
 * of the one before run at the same time, the copies on two streams the library keeps
 * per device (created on first use), ordered against `stream` with events. All work is
 * ordered after the work already on `stream`, and work enqueued on `stream` after this
 * call runs after all of it; the call returns without waiting. The device error word
 * (kq_last_device_error) covers every chunk. */
kq_status kq_linear_host(const kq_layer_desc *desc, const void *weights, const void *X_host,
                         void *X_dev, int32_t M, void *Y_host, void *Y_dev, int32_t out_dtype,
                         void *act, size_t act_bytes, kq_stream_t stream);

/* kq_linear without a caller-supplied workspace. This call has no counterpart in the
 * method's description; it exists for callers that cannot allocate device memory on the
 * path where the layer runs: a C or C++ host with no caching allocator, a serving loop
 * that must not call cudaMalloc/cudaFree there (they are slow and can synchronise the
 * whole device), or a process whose device memory is already handed out to another
 * allocator. It allocates nothing: the activation workspace is a fixed array of
 * KQ_NOALLOC_WORKSPACE_BYTES bytes inside this library's device image, created when
 * the library's module is loaded on a device.
 *   Limit: kq_act_bytes(desc, M) must not exceed KQ_NOALLOC_WORKSPACE_BYTES, else the
 *     call returns KQ_ERR_WORKSPACE_TOO_SMALL and enqueues nothing (about 22,000
 *     tokens for K = 1152, 9,500 for K = 3072, 2,500 for K = 12288 with a low-rank
 *     branch). Use kq_linear with your own workspace for larger M.
 *   Set-up: the first call made with a given device current looks up the array's
 *     address on that device (cudaGetSymbolAddress) and caches it with the id of the
 *     current context; later calls in the same context only read the cache, and a call
 *     in another context (for example after cudaDeviceReset) looks the address up again.
 *     Make the first call in a context before any stream capture begins.
 *   Sharing: every call on a device uses the same array, and it keeps what the last
 *     call wrote. Each call clears the error word at its head and rewrites everything
 *     else it reads. Calls whose work can overlap on the GPU (different streams, or
 *     different host threads, without ordering between them) race on the array and
 *     give wrong results: order them on one stream, or use kq_linear.
 *   The device error word is not exposed; a device-side timeout is not reported here
 *     (use kq_linear with your own workspace and kq_last_device_error for that).
 * Arguments, output and errors are otherwise those of kq_linear. */
#define KQ_NOALLOC_WORKSPACE_BYTES ((size_t)16 << 20)
kq_status kq_linear_noalloc(const kq_layer_desc *desc, const void *weights, const void *X_bf16,
                            int32_t M, void *Y, int32_t out_dtype, kq_stream_t stream);

/* GEMM half only, on an activation workspace already filled by kq_quantize_act or
 * kq_act_pack. */
kq_status kq_gemm(const kq_layer_desc *desc, const void *weights, const void *act, int32_t M,
                  void *Y, int32_t out_dtype, kq_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Canonical <-> internal layouts (tests, checkpoints, imported weights).
 * Canonical layouts: codes uint8 [rows, K/2] with element 2j in the low nibble of
 * byte j; scales uint8 [rows, K/32] row-major (E8M0 bytes); all device pointers.
 * ------------------------------------------------------------------------------- */

/* Write a prepared-weights buffer from canonical parts:
 *   r_codes [N, K/2], r_scales [N, K/32]   residual R^T in MXFP4 (blocks along K)
 *   L1p_f32 float32 [K, rank]              L1' = P L1 (stored internally as a bf16
 *                                          hi/lo pair; c1 = 1^T L1' is derived from it)
 *   L2_bf16 [rank, N]                      low-rank factor L2 as bf16
 *   s float32 [N]                          column sums of the original weight
 * plus the transform tables from the descriptor. */
kq_status kq_weights_pack(const kq_layer_desc *desc, const void *r_codes, const void *r_scales,
                          const float *L1p_f32, const void *L2_bf16, const float *s,
                          void *weights, kq_stream_t stream);

/* Read a prepared-weights buffer back into canonical parts (any pointer may be null
 * to skip that part). L1p_f32 receives hi + lo of the stored L1'. */
kq_status kq_weights_unpack(const kq_layer_desc *desc, const void *weights, void *r_codes,
                            void *r_scales, float *L1p_f32, void *L2_bf16, float *c1, float *s,
                            kq_stream_t stream);

/* Fill an activation workspace from canonical parts (mu may be null when centring is
 * off; U_f16, the low-rank activations as fp16 [M, rank], may be null when rank == 0).
 * For a KQ_CB_LLOYDMAX layer, codes is the fp16 operand [M, K] and scales the fp32
 * per-token sigma [M]. */
kq_status kq_act_pack(const kq_layer_desc *desc, const void *codes, const void *scales,
                      const float *mu, const void *U_f16, int32_t M, void *act,
                      size_t act_bytes, kq_stream_t stream);

/* Read an activation workspace back into canonical parts (null pointers skip).
 * U_f16 receives fp16 [M, rank]. For a KQ_CB_LLOYDMAX layer, codes receives the fp16
 * operand [M, K] and scales the fp32 per-token sigma [M]. */
kq_status kq_act_unpack(const kq_layer_desc *desc, const void *act, int32_t M, void *codes,
                        void *scales, float *mu, void *U_f16, kq_stream_t stream);

/* The library's 16-level Lloyd-Max codebook of N(0, 1) (host memory, no device work):
 * levels8 = the 8 positive levels ascending, thresholds7 = the midpoints between them,
 * computed once by Lloyd's alternation in float64. Either pointer may be null. */
kq_status kq_lloydmax_codebook(double *levels8, double *thresholds7);

/* ---------------------------------------------------------------------------------
 * Debug entry points (each runs one stage of the online half in isolation).
 * ------------------------------------------------------------------------------- */

/* Centring + block transform only: Xt float32 [M, K] and mu float32 [M] (device). */
kq_status kq_debug_transform(const kq_layer_desc *desc, const void *weights,
                             const void *X_bf16, int32_t M, float *Xt, float *mu,
                             kq_stream_t stream);

/* MXFP4 encoder only, on float32 values V [M, K] (device): canonical codes
 * [M, K/2] and scales [M, K/32] (device). */
kq_status kq_debug_encode_f32(const float *V, int32_t M, int32_t K, void *codes, void *scales,
                              kq_stream_t stream);

/* The robust l_p block-scale fit alone (as kq_prepare_weights_lp applies it to R), on
 * float32 rows V [M, K] (device), canonical outputs as kq_debug_encode_f32. p in (0, 2]. */
kq_status kq_debug_encode_lp_f32(const float *V, int32_t M, int32_t K, double p, void *codes,
                                 void *scales, kq_stream_t stream);

/* Synchronises `stream`, then maps the workspace's device error word to a status and
 * clears it: KQ_ERR_DEVICE_TIMEOUT if a bounded device-side wait ran out (it takes
 * precedence), else KQ_ERR_LOWRANK_RANGE if a low-rank activation was saturated, else
 * KQ_OK. */
kq_status kq_last_device_error(const kq_layer_desc *desc, void *act, int32_t M,
                               kq_stream_t stream);

/* Exercises the bounded-wait path without a fault: one warp waits up to limit_us
 * microseconds (1 .. 1,000,000) on a barrier that nothing completes, records the timeout
 * in the error word of `act` (kq_act_bytes(desc, M) bytes, device) and returns. The
 * next kq_last_device_error on that workspace then reports KQ_ERR_DEVICE_TIMEOUT; the
 * context stays usable. Every wait in the library's kernels is bounded the same way
 * (2 s), so a pipeline stage that never fills ends the kernel instead of hanging the GPU.
 * This entry has no counterpart in the method's description. Async on `stream`. */
kq_status kq_debug_wait_timeout(const kq_layer_desc *desc, void *act, int32_t M,
                                uint32_t limit_us, kq_stream_t stream);

/* Static string for a status code. */
const char *kq_status_string(kq_status s);

/* Library build/version string. */
const char *kq_version(void);

#ifdef __cplusplus
}
#endif
#endif /* KQ_H_ */
