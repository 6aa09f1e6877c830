/*
 * svdq.h -- C ABI of the B200 (sm_100a) SVDQuant W4A4 / AWQ W4A16 linear library.
 *
 * The layer (Nunchaku README, "Method": SVDQuant's three stages; "Engine design":
 * the 16-bit low-rank branch beside the 4-bit GEMM):
 *
 *     Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 + bias,   X_hat = X diag(smooth_inv)
 *
 * Q is NVFP4 (E2M1 codes, one unsigned E4M3 scale per 16 values along K) or
 * INT4 (symmetric, one FP16 scale per 64 values along K) -- the Diffusers blog,
 * "quantization_config": svdq_w4a4 {precision, group_size, rank} and awq_w4a16
 * {precision int4, group_size 64}.
 *
 * Calls: the activation quantizer with the fused down-projection
 * (svdq_quantize_act, svdq_quantize_act_noalloc), the 4-bit GEMM with the fused
 * up-projection (svdq_w4a4_linear), NVFP4 with a per-tensor second scale level
 * (svdq_tensor_scale, svdq_quantize_act_two_level, svdq_w4a4_linear_two_level),
 * the fused QKV projection with head norm and rotation
 * (svdq_w4a4_linear_qkv_norm_rope), the fused MLP's fc1 (svdq_mlp_fc1), the AWQ W4A16 linear (awq_w4a16_linear),
 * layout conversion (svdq_pack, svdq_unpack, svdq_pack_lowrank), offline weight
 * preparation (svdq_column_absmax, svdq_smoothing, svdq_lowrank_factors,
 * svdq_residual, awq_quantize_weight), buffer sizes, and the device status word
 * (svdq_check_device_status).
 *
 * Conventions for every call:
 *  - Memory: the caller allocates and owns every buffer. Pointers named as device
 *    pointers must be device memory, 16-byte aligned. The library allocates
 *    nothing, frees nothing and synchronises nothing (svdq_check_device_status
 *    is the one call that synchronises its stream).
 *  - Streams: `stream` is a cudaStream_t (NULL = the legacy default stream). All
 *    work is enqueued on it; calls return before the GPU work finishes.
 *  - Errors: argument errors are detected on the host before any launch and
 *    returned synchronously; nothing is launched then. A failed launch returns
 *    SVDQ_ERR_CUDA. A kernel whose bounded wait ran out records it in a device
 *    status word, read (and cleared) by svdq_check_device_status; the outputs
 *    of every call enqueued since the previous check are then undefined.
 *  - Matrices are row-major. bf16/fp16 are IEEE-style 16-bit patterns.
 *  - Shapes: M >= 1; K % 64 == 0; N % 16 == 0; r == 0 or (r % 16 == 0 and r <= 256).
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* svdq_stream_t; /* a cudaStream_t */

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1, /* a shape, pointer or enum is out of contract */
  SVDQ_ERR_ALIGNMENT = 2,   /* a pointer or leading dimension is not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED = 3, /* valid request this build does not implement */
  SVDQ_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  SVDQ_ERR_TIMEOUT = 5      /* a kernel's bounded wait ran out (device status word) */
} svdq_status;

typedef enum {
  SVDQ_NVFP4_G16 = 0, /* E2M1 codes, UE4M3 scale per 16 along K */
  SVDQ_INT4_G64 = 1   /* int4 codes in [-7, 7], FP16 scale per 64 along K */
} svdq_format;

typedef enum { SVDQ_OUT_BF16 = 0, SVDQ_OUT_F32 = 1 } svdq_out;

typedef enum {
  SVDQ_PACK_ACT = 0,    /* activation codes + scales */
  SVDQ_PACK_WEIGHT = 1, /* residual-weight codes + scales (same layouts as ACT) */
  SVDQ_PACK_AWQ = 2     /* AWQ qweight + scales + zeros */
} svdq_pack_kind;

/* Human-readable name of a status code (static storage). */
const char* svdq_status_str(svdq_status status);

/* Library ABI version (major * 100 + minor). */
int svdq_version(void);

/*
 * Buffer sizes in bytes of the storage formats below. Codes are row-major
 * packed nibbles, K contiguous, element 2j in the low nibble, 2j+1 in the high
 * nibble: rows * K / 2 bytes. NVFP4 codes are E2M1 and INT4 values (-7..7) are
 * two's complement nibbles, in both the plain and the tiled form (the same
 * bytes).
 * Scales ("tiled"):
 *  - NVFP4: rows padded to 128; for row m and scale column j = k/16 the byte sits
 *    in 512-byte atom a = (m/128) * (K/64) + j/4 at offset
 *    (m%32)*16 + ((m%128)/32)*4 + j%4. This is the order tcgen05.cp copies into
 *    tensor memory for the block-scaled MMA, so the kernels read it unchanged.
 *  - INT4: FP16 at [K/64][rows padded to 128] (group-major), padding 0.
 * Returns 0 for an invalid request.
 */
size_t svdq_codes_bytes(svdq_format format, int rows, int K);
size_t svdq_scales_bytes(svdq_format format, int rows, int K);

/* AWQ storage (see svdq_pack): fragment-ordered qweight and interleaved (scale, zero). */
size_t awq_qweight_bytes(int N, int K);
size_t awq_sz_bytes(int N, int K);

/*
 * svdq_xl1_splits -- S, the number of [M, r] slices of the xl1 buffer that
 * svdq_quantize_act needs for an M x K activation with rank r (it splits K into
 * S ranges): the largest power of two <= 8 (and <= K/64) that keeps
 * ceil(M/128) * S within the 148 SMs of a B200; 1 when r == 0. A pure function
 * of its arguments; 0 for an invalid request.
 */
int svdq_xl1_splits(int M, int K, int r);

/*
 * svdq_quantize_act -- steps a1..a4: smooth, group-scale, quantize + pack the
 * activations, and the rank-r down-projection of the smoothed activations, in
 * one pass over X (Nunchaku README, "Engine design" (b): the down projection and
 * the quantizer read the same input).
 *
 *   x_hat[m,k] = RN32(X[m,k] * smooth_inv[k])             (smooth_inv NULL -> x_hat = X)
 *   NVFP4: s = UE4M3(RN32(amax16 / 6)), q = E2M1(RN32(x_hat * RN32(1 / s)))
 *   INT4:  s = FP16(RN32(amax64 / 7)),  q = clamp(rint(RN32(x_hat * RN32(1 / s))), -7, 7)
 *   a group whose decoded scale is 0 stores scale 0 and codes 0
 *   xl1[m,:] = x_hat[m,:] @ L1                            (float32 output)
 *
 * X          device, bf16 [M, ldx] (first K columns used), ldx % 8 == 0
 * smooth_inv device, float32 [K], or NULL
 * L1s        device, the down-projection operand from svdq_pack_lowrank: bf16
 *            [2][r][K] = diag(smooth_inv) L1, transposed, as hi and lo planes;
 *            NULL iff r == 0
 * codes      device, svdq_codes_bytes(format, M, K) bytes, written (tiled form)
 * scales     device, svdq_scales_bytes(format, M, K) bytes, written (padding rows too)
 * xl1        device, float32 [S][M][r] with S = svdq_xl1_splits(M, K, r): on
 *            return its first [M, r] slice holds x_hat L1; the other S - 1
 *            slices are the call's working space (the down-projections of S
 *            ranges of K, added in order into the first); NULL iff r == 0
 * Codes and scales are bit-exact functions of the inputs. xl1 is computed on the
 * tensor cores as X (hi + lo) with float32 accumulation, which equals x_hat L1 to
 * about 2^-17 relative per term. The K ranges let every SM work on the pass
 * without any CTA waiting for another. This call also serves as the weight quantizer
 * (residual R given as bf16, smooth_inv NULL, r 0).
 */
svdq_status svdq_quantize_act(svdq_format format, int M, int K, int r, const void* X, int ldx,
                              const float* smooth_inv, const void* L1s, void* codes,
                              void* scales, float* xl1, svdq_stream_t stream);

/*
 * svdq_quantize_act_noalloc -- svdq_quantize_act with no working space from the
 * caller: xl1 is only float32 [M, r] (same contents on return), and the partial
 * down-projections of K splits 1 .. S-1 go to a working array the library
 * holds in device memory for each device (one static array of 2^21 float32,
 * 8 MiB; nothing is allocated or freed at any time). The pages describe no
 * counterpart of this call. It exists for callers that cannot allocate device
 * memory at the point where they quantize: a serving runtime or a plugin of a
 * host framework whose allocator owns all device memory and sizes it before the
 * first request, so that a cudaMalloc mid-step would go around that budget, may
 * block or synchronise the device, and may fail under memory pressure. Such a
 * caller passes only the inputs and outputs it already holds.
 *
 * Set-up: the first call of any entry point of this library on a device (this
 * one included) looks up that device's copy of the array (cudaGetSymbolAddress
 * with the device current) and sets kernel attributes, once per device; make
 * that first call before any stream capture begins on the device.
 *
 * Limit: (S - 1) * M * r <= 2^21 with S = svdq_xl1_splits(M, K, r); a larger
 * request returns SVDQ_ERR_UNSUPPORTED before anything is launched (r == 0 always
 * fits). Nothing in the array needs to start at zero: each call writes every
 * element it reads. The array is shared by all calls on a device and keeps
 * the last call's partial sums, so two of these calls that overlap on the GPU
 * (e.g. in flight on different streams) race on it; calls ordered on one
 * stream do not. Other arguments, layouts and errors as for svdq_quantize_act.
 */
svdq_status svdq_quantize_act_noalloc(svdq_format format, int M, int K, int r, const void* X,
                                      int ldx, const float* smooth_inv, const void* L1s,
                                      void* codes, void* scales, float* xl1,
                                      svdq_stream_t stream);

/*
 * svdq_w4a4_linear -- steps a5..a6: the 4-bit GEMM with the low-rank
 * up-projection and bias accumulated into the same tensor-memory accumulator
 * (Nunchaku README, "Engine design" (b): the up projection and the 4-bit
 * compute share the output).
 *
 *   Y[m,n] = sum_g s_a[m,g] s_w[n,g] sum_{k in g} q_a[m,k] q_w[n,k]
 *          + sum_j xl1[m,j] L2[j,n] + bias[n]
 *
 * a_codes, a_scales  device, activation codes/scales from svdq_quantize_act (M rows)
 * xl1                device, float32 [M, r] (the first slice of svdq_quantize_act's
 *                    xl1); NULL iff r == 0
 * w_codes, w_scales  device, weight codes/scales in the same formats (N rows)
 * L2                 device, bf16 [r, N]; NULL iff r == 0
 * bias               device, bf16 [N], or NULL
 * Y                  device, [M, ldy] bf16 (out = SVDQ_OUT_BF16) or float32, ldy >= N,
 *                    ldy * element size % 16 == 0
 * The low-rank product uses xl1 split into two bf16 terms; accumulation is float32.
 * NVFP4 runs on the block-scaled FP4 MMA. INT4 has no 4-bit integer MMA on
 * sm_100a: both operands are dequantized on chip to FP16 values fp16(s q) (one
 * rounding, relative error <= 2^-12; exact for power-of-two scales) and
 * multiplied on the FP16 tensor cores with float32 accumulation. |s q| must fit
 * FP16 (group absolute maxima below 65504).
 */
svdq_status svdq_w4a4_linear(svdq_format format, int M, int N, int K, int r, const void* a_codes,
                             const void* a_scales, const float* xl1, const void* w_codes,
                             const void* w_scales, const void* L2, const void* bias, void* Y,
                             int ldy, svdq_out out, svdq_stream_t stream);

/*
 * Two-level NVFP4. NVFP4 as named on the pages (Diffusers blog,
 * "quantization_config": precision nvfp4, group_size 16: E2M1 values with one
 * E4M3 scale per 16) has a second scale level above the group scales: one
 * float32 factor s_t per tensor, which lets a tensor whose range E4M3 group
 * scales cannot cover (amax / 6 above 448 or below 2^-9) keep the format's
 * relative precision. The pages state no formula for it; this library uses
 *
 *   s_t = RN32(amax / (6 * 448)) if that is a normal float32, else 1
 *   codes and group scales of x' = RN32(x_hat * RN32(1 / s_t)), exactly as
 *   svdq_quantize_act does for x_hat
 *   Y = RN32(s_t,a * s_t,w) * sum_g s_a s_w sum_k q_a q_w + xl1 L2 + bias
 *
 * svdq_tensor_scale -- scale[0] = s_t and scale[1] = RN32(1 / s_t) of
 *   x_hat = RN32(X * smooth_inv) (smooth_inv NULL: x_hat = X).
 *   X device bf16 [M, ldx], ldx % 8 == 0; smooth_inv device float32 [K] or NULL;
 *   scale device float32 [2], 8-byte aligned, written. Enqueues a 4-byte memset
 *   of scale[0] and two kernels (an absolute-maximum pass over X, then one thread).
 *
 * svdq_quantize_act_two_level -- svdq_quantize_act in NVFP4 with the codes and
 *   group scales of x' = RN32(x_hat * scale[1]); xl1 = x_hat L1 is unchanged
 *   (unscaled). scale: device float32 [2] as svdq_tensor_scale writes it (for the
 *   same tensor, or a calibrated [s_t, RN32(1 / s_t)]), 8-byte aligned. Residual
 *   weights are quantized the same way with smooth_inv NULL, r 0 and their own
 *   scale. Other arguments as for svdq_quantize_act.
 *
 * svdq_w4a4_linear_two_level -- svdq_w4a4_linear in NVFP4 for codes from
 *   svdq_quantize_act_two_level: a_tensor_scale and w_tensor_scale are the device
 *   scale pairs of the activation and the weight (element 0, s_t, is read); alpha =
 *   RN32(a_tensor_scale[0] * w_tensor_scale[0]). The low-rank term shares the
 *   tensor-memory accumulator with the 4-bit product, so it enters as
 *   RN32(xl1 * RN32(1 / alpha)) and the epilogue computes alpha * acc + bias (one
 *   extra rounding of the low-rank term, relative 2^-24). Other arguments as for
 *   svdq_w4a4_linear.
 */
svdq_status svdq_tensor_scale(int M, int K, const void* X, int ldx, const float* smooth_inv,
                              float* scale, svdq_stream_t stream);
svdq_status svdq_quantize_act_two_level(int M, int K, int r, const void* X, int ldx,
                                        const float* smooth_inv, const float* scale,
                                        const void* L1s, void* codes, void* scales, float* xl1,
                                        svdq_stream_t stream);
svdq_status svdq_w4a4_linear_two_level(int M, int N, int K, int r, const void* a_codes,
                                       const void* a_scales, const float* a_tensor_scale,
                                       const float* xl1, const void* w_codes, const void* w_scales,
                                       const float* w_tensor_scale, const void* L2, const void* bias,
                                       void* Y, int ldy, svdq_out out, svdq_stream_t stream);

/*
 * svdq_mlp_fc1 -- the first half of the fused MLP (Diffusers blog, "From SVDQuant
 * to Nunchaku Lite": the original engine runs GELU/MLP as one fused path, where
 * Lite runs the two SVDQ linears apart). fc1's NVFP4 layer, and in its epilogue
 * everything fc2 needs from the hidden activation, so the [M, N1] activation never
 * reaches HBM in 16 bits:
 *
 *   y1     = the fc1 layer as svdq_w4a4_linear computes it, float32 in tensor memory
 *   h_hat  = RN32(RN32(GELU(RN32(y1))) * smooth_inv2[n]),
 *            GELU(y) = 0.5 y (1 + tanh(u)), u = sqrt(2/pi) (y + 0.044715 y^3), evaluated in
 *            float32 as y / (1 + exp(-2u)) (the same function; a few float32 ulps)
 *   codes2, scales2 = NVFP4 codes and scales of h_hat (steps a2, a3 of fc2, groups of 16
 *            along N1, the layouts svdq_quantize_act writes)
 *   xl1_2  = h_hat L1_2 (step a4 of fc2; h_hat as a bf16 hi + lo pair on the tensor
 *            cores, float32 accumulation)
 *
 * Then svdq_w4a4_linear(NVFP4, M, N2, K = N1, r2, codes2, scales2, xl1_2, ...) is fc2.
 *
 * a_codes, a_scales, xl1_1  fc1's input from svdq_quantize_act (M rows, K1)
 * w_codes, w_scales         fc1's weight codes/scales (N1 rows)
 * L2_1                      device, bf16 [r1, N1]; NULL iff r1 == 0
 * bias1                     device, bf16 [N1] or NULL
 * smooth_inv2               device, float32 [N1] (fc2's smoothing) or NULL (1)
 * L1t_2                     device, bf16 [r2, N1]: fc2's factor L1_2 [N1, r2] transposed
 *                           (row j holds column j of L1_2); NULL iff r2 == 0
 * codes2, scales2           device, svdq_codes_bytes / svdq_scales_bytes(NVFP4, M, N1), written
 * xl1_2                     device, float32, svdq_mlp_splits(M, N1) * M * r2 elements of
 *                           working space; on return its first M * r2 hold xl1_2 [M, r2].
 *                           NULL iff r2 == 0
 * hhat                      device, float32 [M, N1] receiving h_hat, or NULL (for tests)
 * Shapes: N1 % 128 == 0, K1 % 64 == 0, r1 as for svdq_w4a4_linear, r2 in {0, 32, 64, 96, 128}.
 * INVALID_ARG / ALIGNMENT before any launch otherwise.
 */
int svdq_mlp_splits(int M, int N1);
svdq_status svdq_mlp_fc1(int M, int N1, int K1, int r1, int r2, const void* a_codes, const void* a_scales,
                         const float* xl1_1, const void* w_codes, const void* w_scales, const void* L2_1,
                         const void* bias1, const float* smooth_inv2, const void* L1t_2, void* codes2,
                         void* scales2, float* xl1_2, float* hhat, svdq_stream_t stream);

/*
 * svdq_w4a4_linear_qkv_norm_rope -- the fused QKV projection of an attention
 * block with its head normalisation and rotary embedding in the GEMM's epilogue
 * (Diffusers blog, the fused QKV section: to_q, to_k, to_v joined along the
 * output dimension in the order Q, K, V into one SVDQ linear, whose output goes
 * through norm_q / norm_k per head and then the rotary embedding in one fused
 * call). svdq_w4a4_linear in NVFP4, then on each row m of Y:
 *   heads of 128 columns, H = N / 384 of each of Q (columns [0, 128 H)), K
 *   ([128 H, 256 H)) and V ([256 H, 384 H));
 *   each head v of Q and K: z = v * rsqrt(mean(v^2) + eps) * gamma, gamma the
 *   head weight (norm_q for Q, norm_k for K); then each pair (z[2i], z[2i+1]) ->
 *   (z[2i] cos - z[2i+1] sin, z[2i+1] cos + z[2i] sin), cos = rope_cos[i][m] and
 *   sin = rope_sin[i][m];
 *   V as svdq_w4a4_linear computes it.
 * All of it in float32 from the accumulator, with one rounding at the output.
 *   N        multiple of 384 (three projections of whole 128-column heads)
 *   norm_q, norm_k  device bf16 [128], 2-byte aligned, or NULL (weight 1)
 *   eps      finite, >= 0 (a head whose values are all zero needs eps > 0)
 *   rope_cos, rope_sin  device float32 [64, M], angle-major (angle i of token
 *            row m at i * M + m: the rows an epilogue warp holds read one
 *            contiguous run per angle), 4-byte aligned; both NULL: no rotation
 * Other arguments, layouts and errors as for svdq_w4a4_linear; INVALID_ARG when
 * N is not a multiple of 384, eps is out of range or only one table is given.
 */
svdq_status svdq_w4a4_linear_qkv_norm_rope(int M, int N, int K, int r, const void* a_codes,
                                           const void* a_scales, const float* xl1,
                                           const void* w_codes, const void* w_scales, const void* L2,
                                           const void* bias, const void* norm_q, const void* norm_k,
                                           float eps, const float* rope_cos, const float* rope_sin,
                                           void* Y, int ldy, svdq_out out, svdq_stream_t stream);

/*
 * awq_w4a16_linear -- step a7, the AWQ W4A16 linear (Diffusers blog, "From
 * SVDQuant to Nunchaku Lite": awq_w4a16 for the memory-bound adaptive-norm
 * modulation projections; int4 weights, a bf16 scale and zero point per 64
 * values along K, 16-bit activations).
 *
 *   Y[m,n] = sum_k X[m,k] (q[n,k] - z[n,k/64]) s[n,k/64] + bias[n]
 *
 * Two kernels serve it, by M: up to 64 tokens a GEMV on the warp-level MMA
 * (launches of at most 16 tokens, each streaming the weights once); above 64 a
 * tensor-core GEMM (tcgen05, tokens in tiles of up to 128, each tile streaming
 * the weights once). Both form (q - z) exactly in bf16 and scale each group's
 * float32 sum by s in float32. SVDQ_AWQ_PATH=0 / 1 in the environment forces the
 * GEMV (M <= 64 only) / the GEMM for any M, for measurement.
 *
 * X        device, bf16 [M, K] (row-major, K contiguous), M >= 1
 * qweight  device, awq_qweight_bytes(N, K) bytes, fragment order from svdq_pack(AWQ)
 * sz       device, awq_sz_bytes(N, K) bytes, interleaved (s, z) from svdq_pack(AWQ);
 *          every zero point z is an integer in [0, 15], as the format defines
 * bias     device, bf16 [N] or NULL
 * Y        device, bf16 [M, N]
 * group must be 64; INVALID_ARG / ALIGNMENT otherwise.
 */
svdq_status awq_w4a16_linear(int M, int N, int K, int group, const void* X, const void* qweight,
                             const void* sz, const void* bias, void* Y, svdq_stream_t stream);

/*
 * svdq_pack / svdq_unpack -- convert between plain and tiled storage
 * (unpack(pack(x)) == x bit for bit).
 *
 * ACT / WEIGHT: plain_codes [rows, K/2] bytes -> tiled codes (the same bytes,
 *   NVFP4 and INT4);
 *   plain_scales: NVFP4 uint8 [rows, K/16] E4M3 codes, INT4 fp16 [rows, K/64]
 *   -> tiled scales (layouts above). plain_zeros must be NULL.
 * AWQ: plain_codes = qweight [N, K/2] (element 2j low nibble, values 0..15),
 *   plain_scales = bf16 [N, K/64], plain_zeros = bf16 [N, K/64]
 *   -> tiled_codes (awq_qweight_bytes), tiled_scales (awq_sz_bytes). format ignored.
 *   Fragment order: for 16-row block b and group g, 32 lanes x 16 bytes; lane t
 *   (r0 = t/4, c0 = 2(t%4)) holds words w_j, j = 0..3 (k = 64g + 16j + ...); nibble
 *   slot s of w_j holds W[r0 + {0,8,0,8,0,8,0,8}[s]][c0 + {0,0,8,8,1,1,9,9}[s]].
 *   (s, z) pairs sit at [N/16][K/64][16][2].
 * All pointers device; rows of padding are written as zeros.
 */
svdq_status svdq_pack(svdq_pack_kind kind, svdq_format format, int rows, int K,
                      const void* plain_codes, const void* plain_scales, const void* plain_zeros,
                      void* tiled_codes, void* tiled_scales, svdq_stream_t stream);
svdq_status svdq_unpack(svdq_pack_kind kind, svdq_format format, int rows, int K,
                        const void* tiled_codes, const void* tiled_scales, void* plain_codes,
                        void* plain_scales, void* plain_zeros, svdq_stream_t stream);

/*
 * svdq_pack_lowrank -- the down-projection operand of svdq_quantize_act. The
 * smoothing folds into the factor (x_hat L1 = X diag(smooth_inv) L1), which is
 * split into two bf16 terms so the tensor cores see it at about 16-bit-squared
 * precision:
 *   v = RN32(smooth_inv[k] * L1[k][j]),  hi = RN_bf16(v),  lo = RN_bf16(v - hi)
 *   L1s[0][j][k] = hi, L1s[1][j][k] = lo
 * L1          device, bf16 [K, r] (the SVD factor, K rows)
 * smooth_inv  device, float32 [K] or NULL (then v = L1)
 * L1s         device, bf16 [2][r][K], written
 * K % 64 == 0, r % 16 == 0, 16 <= r <= 256.
 */
svdq_status svdq_pack_lowrank(int K, int r, const void* L1, const float* smooth_inv, void* L1s,
                              svdq_stream_t stream);

/*
 * Offline weight preparation (Nunchaku README, "Method": stage 2 migrates the
 * activation outliers into the weights, X_hat = X diag(lambda)^-1 and
 * W_hat = W diag(lambda); stage 3 splits W_hat into a 16-bit low-rank part L1 L2
 * and a residual R that is quantized to 4 bits). These calls run everything of
 * it except the SVD, which the caller's linear-algebra library computes from
 * W_hat = W diag(1 / smooth_inv) (in float64). Not part of the timed path.
 *
 * svdq_column_absmax -- absmax[k] = max_m |A[m,k]| (exact) of a bf16 matrix.
 *   A       device, bf16 [rows, lda], 16-byte aligned, lda % 8 == 0, lda >= K
 *   absmax  device, float32 [K], written (cleared first on the stream)
 *   K % 8 == 0.
 *
 * svdq_smoothing -- the smoothing vector of one layer from the calibration
 * activations' channel maxima and the weight:
 *   lambda_k = sqrt(x_absmax[k] / max_n |W[n,k]|) in float64 (1 if either is 0),
 *   smooth_inv[k] = RN32(1 / lambda_k) in float64, then rounded once to float32
 *   x_absmax    device, float32 [K] (e.g. svdq_column_absmax of calibration X)
 *   W           device, bf16 [N, K], 16-byte aligned
 *   smooth_inv  device, float32 [K], written
 *
 * svdq_lowrank_factors -- the 16-bit low-rank factors from the SVD
 * W_hat = U diag(S) Vh (float64, singular values in decreasing order), each
 * element rounded once to bf16 (nearest even):
 *   L1[k,j] = RN_bf16(Vh[j,k] sqrt(S[j]))  [K, r],   L2[j,n] = RN_bf16(sqrt(S[j]) U[n,j])  [r, N]
 *   U [N, ldu] (ldu >= r), S [>= r], Vh [>= r rows, ldvh] (ldvh >= K): device, float64
 *   L1, L2      device, bf16, written;  1 <= r <= min(N, K).
 *
 * svdq_residual -- the residual that is quantized:
 *   R[n,k] = RN_bf16( W[n,k] * (1 / smooth_inv[k]) - sum_j L1[k,j] L2[j,n] ),
 *   each step in float64, one rounding to bf16 (nearest even) at the end
 *   W           device, bf16 [N, K];  smooth_inv  device, float32 [K]
 *   L1, L2      device, bf16 [K, r] and [r, N] (the SVD factors); NULL iff r == 0
 *   R           device, bf16 [N, K], written (quantize it with svdq_quantize_act,
 *               no smoothing, rank 0)
 *   0 <= r <= 4096.
 *
 * awq_quantize_weight -- the AWQ W4A16 weight quantizer (Diffusers blog,
 * quantization_config: awq_w4a16, int4, group 64), per row and 64-wide group:
 *   s = RN_bf16((max - min) / 15), or 1 if max == min;  z = clamp(rint(-min / s), 0, 15);
 *   q = clamp(rint(w / s + z), 0, 15)   (float64 arithmetic, rint to even)
 * written straight into the layouts awq_w4a16_linear reads (the output of
 * svdq_pack(AWQ)).
 *   W        device, bf16 [N, K]
 *   qweight  device, awq_qweight_bytes(N, K) bytes, written
 *   sz       device, awq_sz_bytes(N, K) bytes, written
 *   K % 64 == 0.
 * All five: INVALID_ARG / ALIGNMENT on bad arguments, before any launch.
 */
svdq_status svdq_column_absmax(int rows, int K, const void* A, int lda, float* absmax,
                               svdq_stream_t stream);
svdq_status svdq_smoothing(int N, int K, const float* x_absmax, const void* W, float* smooth_inv,
                           svdq_stream_t stream);
svdq_status svdq_lowrank_factors(int N, int K, int r, const double* U, int ldu, const double* S,
                                 const double* Vh, int ldvh, void* L1, void* L2, svdq_stream_t stream);
svdq_status svdq_residual(int N, int K, int r, const void* W, const float* smooth_inv, const void* L1,
                          const void* L2, void* R, svdq_stream_t stream);
svdq_status awq_quantize_weight(int N, int K, const void* W, void* qweight, void* sz,
                                svdq_stream_t stream);

/*
 * svdq_check_device_status -- synchronises `stream`, then reads and clears the
 * device status word of the current device. Returns SVDQ_ERR_TIMEOUT if any
 * kernel's bounded wait ran out since the last check, SVDQ_ERR_CUDA if the
 * stream reported an error, else SVDQ_OK.
 */
svdq_status svdq_check_device_status(svdq_stream_t stream);

/*
 * svdq_debug_wait_timeout -- diagnostics: launches one CTA that waits on a
 * barrier no one arrives at, with a bound of `limit_us` microseconds, no copy in
 * flight. The wait runs out, the kernel records SVDQ_ERR_TIMEOUT in the status
 * word and returns normally. Used to test the failure-detection path without
 * faulting or hanging the GPU. 1 <= limit_us <= 1000000.
 */
svdq_status svdq_debug_wait_timeout(int limit_us, svdq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
