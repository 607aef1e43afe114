/*
 * kronq.h — C ABI of libkronq.so, the per-sublayer quantization engine of
 * KronQ (Kronecker-factored-Hessian post-training quantization) for NVIDIA
 * B200 (sm_100a).
 *
 * Sources (web pages about arXiv 2607.07964, "KronQ: LLM Quantization via
 * Kronecker-Factored Hessian"), cited below by these short names:
 *   [gptget-en]  gptget.net, "KronQ: LLM Quantization via Kronecker-Factored
 *                Hessian" (English summary): Methodology, Technical
 *                Contribution, Novelty, Abstract.
 *   [gptget-zh]  gptget.net, same title, Chinese summary: 方法论, 技术贡献.
 *   [aimodeling] aimodeling.com news, "KronQ：Kronecker Hessian 拆掉 GPTQ 的
 *                2-bit 墙" (English title "KronQ: Kronecker Hessians break
 *                GPTQ's 2-bit wall").
 *   [wmrh]       wmrh.cn long-form article on KronQ, sections 一 … 九 and the
 *                closing Q&A (Q1–Q3).
 *
 * The engine, per linear sublayer W (d_out x d_in, y = W x):
 *   1. covariances  H_X = X^T X / n,  H_G = G^T G / n      [wmrh §二; aimodeling]
 *   2. sensitivity  tr(H_G) * tr(H_X)                      [wmrh §三, §六; aimodeling]
 *   3. BiIP: diagonal rescale from diag(H_X), diag(H_G), then a seeded
 *      orthogonal rotation on both sides of W, H_X and H_G rotated to match
 *                                                          [wmrh §三, §八, Q2; aimodeling]
 *   4. damped Cholesky factor U of H_X'^{-1} (H_G is not needed after 3,
 *      because it cancels from the per-column update)      [wmrh §四, §七]
 *   5. GPTQ-style column-wise OBS quantize-and-compensate with asymmetric
 *      min-max group scales at 2/3/4 bits                  [gptget-en Methodology; wmrh §四, §五]
 *   plus a greedy mixed-precision bit allocator driven by step 2 [wmrh §六].
 *
 * ---------------------------------------------------------------------------
 * Conventions (all entry points except kronq_allocate_bits and
 * kronq_status_string):
 *   - Every pointer is a DEVICE pointer owned by the caller. The library never
 *     allocates device memory; scratch space is passed as (ws, ws_bytes), sized
 *     by kronq_workspace_bytes(). ws must be 256-byte aligned.
 *   - Every matrix is row-major and dense. d_out x d_in means d_out rows.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream). Inputs must stay alive until the stream reaches the
 *     call.
 *   - The return value reports argument, shape and launch errors only.
 *     Numerical outcomes go to the device int32 word *info_dev, which the
 *     call first sets to 0 (stream-ordered). After synchronising, the caller
 *     reads it: 0 = ok; (KRONQ_ERR_NOT_PD | (col << 8)) when the damped
 *     Cholesky meets a pivot <= 0 or non-finite at column `col`;
 *     KRONQ_ERR_NONFINITE when an input holds a NaN/Inf the call checks for.
 *   - There is no CPU fallback: without a usable CUDA device every call
 *     returns KRONQ_ERR_CUDA.
 * ---------------------------------------------------------------------------
 * Rotation and random-number specification (BiIP, step 3).
 *
 * [wmrh §三, §七, Q2] realise the two-sided incoherence rotation as a
 * bidirectional Hadamard transform; [wmrh §八] puts a diagonal scaling from
 * diag(H_X), diag(H_G) before it. The pages give neither the scaling exponent
 * nor the construction for sizes that are not powers of two; the library
 * fixes them as follows (both the GPU path and the test oracle implement this
 * text independently).
 *
 *   splitmix64 (Steele, Lea & Flood 2014; reference C by S. Vigna): for a
 *   64-bit state s, sm64(s) = mix(s + 0x9E3779B97F4A7C15) with
 *     mix(z): z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9;
 *             z = (z ^ (z >> 27)) * 0x94D049BB133111EB;
 *             return z ^ (z >> 31);            (all arithmetic mod 2^64)
 *   so sm64(0) = 0xE220A8397B1DCDAF is the generator's first output for seed 0.
 *
 *   Per side (side = 0 for the input dimension d_in, 1 for the output
 *   dimension d_out): key = sm64(sm64(seed) + side).
 *   Size d = had * m with had a power of two and 1 <= m <= 256.
 *   Index i in [0, d) splits as i = a*m + b, a in [0, had), b in [0, m).
 *     sign_i = +1 if bit 63 of sm64(key + i) is 0, else -1.
 *     Q_m: let kq = key ^ 0xA5A5A5A5A5A5A5A5. For t = r*m + c (r, c in [0,m)):
 *       u1 = ((sm64(kq + 2t) >> 11) + 1) * 2^-53          in (0, 1]
 *       u2 =  (sm64(kq + 2t + 1) >> 11) * 2^-53           in [0, 1)
 *       G[r][c] = sqrt(-2 ln u1) * cos(2 pi u2)            (Box–Muller)
 *     Q_m is the orthogonal factor of the QR factorisation G = Q_m R with
 *     every R[j][j] > 0 (unique; computed in fp64). For m = 1, Q_1 = [1].
 *   Hhat = Sylvester Hadamard of order had (Hhat[a][a'] = (-1)^popcount(a&a'))
 *          divided by sqrt(had).
 *   The side's rotation is U = (Hhat kron Q_m) * diag(sign):
 *     (U v)[a*m + b] = sum_{a',b'} Hhat[a][a'] * Q_m[b][b'] * sign[a'*m+b'] * v[a'*m+b'].
 *   Diagonal scale: s_i = max(h_ii, 1e-8 * mean(diag h))^scale_exp, with h the
 *   side's covariance (H_X for the input side, H_G for the output side).
 *
 *   BiIP then produces
 *     W'   = U_G * S_G * W * S_X * U_X^T
 *     H_X' = U_X * S_X^-1 * H_X * S_X^-1 * U_X^T
 *     H_G' = U_G * S_G^-1 * H_G * S_G^-1 * U_G^T
 *   so that tr(H_G' dW' H_X' dW'^T) = tr(H_G dW H_X dW^T) for every dW.
 * ---------------------------------------------------------------------------
 * Quantizer (step 5), per row and per group of `group` consecutive input
 * columns, evaluated on the row's current (compensated) weights at the
 * group's first column [wmrh §五: W2/W3/W4, g128]:
 *   xmin = min(0, min w), xmax = max(0, max w)
 *   if xmax == xmin: scale = 1, zero = 0
 *   else:            scale = (xmax - xmin) / (2^bits - 1), zero = rint(-xmin / scale)
 *   q = clamp(rint(w / scale) + zero, 0, 2^bits - 1),  w_hat = scale * (q - zero)
 *   (rint = round half to even). Then, with U the upper Cholesky factor of
 *   (H_X' + lambda I)^-1:  err = (w_j - w_hat_j) / U[j][j];
 *   w_k -= err * U[j][k] for every k > j of the row.  H_G does not appear
 *   [wmrh §四].
 * Packed codes: per row a little-endian bitstream of d_in codes, code of
 *   column c in bits [c*bits, c*bits + bits) of the row; the row occupies
 *   bits*d_in/32 uint32 words (d_in % 32 == 0 is required).
 * ---------------------------------------------------------------------------
 */
#ifndef KRONQ_H
#define KRONQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *kronq_stream_t; /* ABI-identical to cudaStream_t */

typedef enum {
  KRONQ_OK = 0,
  KRONQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad dtype     */
  KRONQ_ERR_UNSUPPORTED = 2, /* valid but outside the supported shapes     */
  KRONQ_ERR_NOT_PD = 3,      /* info word only: pivot <= 0 (col in b8..31) */
  KRONQ_ERR_NONFINITE = 4,   /* info word only: NaN/Inf met               */
  KRONQ_ERR_TIMEOUT = 5,     /* a bounded device-side wait gave up         */
  KRONQ_ERR_CUDA = 6         /* a CUDA launch or runtime call failed       */
} kronq_status;

typedef enum { KRONQ_F32 = 0, KRONQ_BF16 = 1 } kronq_dtype;

/* Factorisation of one side's dimension d = had * m (see the spec above). */
typedef struct {
  int64_t had; /* power of two, >= 1 */
  int64_t m;   /* 1 <= m <= 256      */
} kronq_rot;

/* flags for kronq_opts.flags */
#define KRONQ_FLAG_NO_ROT_IN   0x1u /* skip U_X (input-side rotation)  */
#define KRONQ_FLAG_NO_ROT_OUT  0x2u /* skip U_G (output-side rotation) */
#define KRONQ_FLAG_NO_SCALE    0x4u /* S_X = S_G = I                   */

typedef struct {
  int32_t bits;      /* 2, 3 or 4                                          */
  int32_t group;     /* 32, 64 or 128; divides d_in                        */
  int32_t block;     /* OBS block width; must be 128                       */
  float damp_rel;    /* lambda = damp_rel * mean(diag H_X')                */
  float scale_exp;   /* exponent of the diagonal scale (0.25 by default)   */
  uint64_t seed;     /* BiIP seed                                          */
  kronq_rot rot_in;  /* d_in  = rot_in.had  * rot_in.m                     */
  kronq_rot rot_out; /* d_out = rot_out.had * rot_out.m                    */
  uint32_t flags;    /* KRONQ_FLAG_*                                       */
} kronq_opts;

/* Which call a workspace size is asked for. */
typedef enum {
  KRONQ_WS_BIIP = 0,
  KRONQ_WS_CHOL = 1,
  KRONQ_WS_QUANT = 2,
  KRONQ_WS_LOSS = 3,
  KRONQ_WS_QUANT_SPLIT = 4
} kronq_ws_kind;

/*
 * Step 1 — calibration covariance [wmrh §二; aimodeling; gptget-en Methodology:
 * H_G from one backward pass].
 *   H = alpha * A^T A + beta * H
 * A: n x d (row stride lda elements, lda >= d), dtype KRONQ_BF16 (tensor-core
 * path, fp32 accumulation) or KRONQ_F32 (fp32 path). H: d x d fp32, both
 * triangles written. For one pass over all rows use alpha = 1/n, beta = 0
 * (H need not be initialised then). BF16 needs d % 128 == 0 and lda % 8 == 0
 * and a 16-byte aligned A; otherwise KRONQ_ERR_UNSUPPORTED. n == 0 scales H by
 * beta. Symmetric in its result; the two triangles are written from the same
 * accumulator tile, so they are bitwise equal.
 * info_dev: KRONQ_ERR_TIMEOUT when a pipeline wait of the tensor-core path
 * ran out (H is then incomplete and must not be used).
 */
kronq_status kronq_accum_cov(kronq_stream_t stream, const void *A,
                             kronq_dtype dtype, int64_t n, int64_t d,
                             int64_t lda, float alpha, float beta, float *H,
                             int32_t *info_dev);

/*
 * Step 2 — sublayer sensitivity [wmrh §三, §六; aimodeling].
 * out_dev[0] = tr(H_X), out_dev[1] = tr(H_G), out_dev[2] = their product,
 * summed in fp64 from the fp32 diagonals. Call it on the covariances BEFORE
 * kronq_biip (the rotation keeps traces, the diagonal rescale does not).
 */
kronq_status kronq_sensitivity(kronq_stream_t stream, const float *H_X,
                               int64_t d_in, const float *H_G, int64_t d_out,
                               double *out_dev);

/*
 * Step 3 — bidirectional incoherence processing [wmrh §三, §八, Q2;
 * aimodeling; gptget-en Technical Contribution]. See the spec above.
 * W: d_out x d_in (dtype wdtype, read only). W_rot: d_out x d_in fp32 output.
 * H_X (d_in^2) and H_G (d_out^2): full symmetric fp32, rotated in place.
 * s_x[d_in], s_g[d_out]: fp32 outputs, the diagonal scales used (all 1 with
 * KRONQ_FLAG_NO_SCALE). ws: kronq_workspace_bytes(KRONQ_WS_BIIP, ...).
 * Requires d_in % 32 == 0, had*m == d per side, had a power of two,
 * 1 <= m <= 256, d <= 65536. info: NONFINITE when a diagonal is not finite;
 * TIMEOUT when a bounded wait of a pass (a bulk copy landing) ran out (the
 * outputs are then incomplete and must not be used).
 */
kronq_status kronq_biip(kronq_stream_t stream, const kronq_opts *opts,
                        const void *W, kronq_dtype wdtype, int64_t d_out,
                        int64_t d_in, float *W_rot, float *H_X, float *H_G,
                        float *s_x, float *s_g, void *ws, size_t ws_bytes,
                        int32_t *info_dev);

/*
 * Step 3 for callers that cannot allocate device memory. The pages have no
 * counterpart: this is a deployment convenience, not part of the method.
 * Some callers cannot give the library a workspace: frameworks that reserve
 * all of HBM for their own pool allocator, plugin hosts that pass only
 * input and output buffers, or loops where cudaMalloc/cudaFree would
 * synchronise the device. This call behaves exactly like kronq_biip (same
 * arguments without ws/ws_bytes, same results, errors and info word) but
 * keeps its scratch in a fixed 4 MiB device array inside the library. It
 * calls no allocator.
 * - The array lives in the module image: every GPU that loads libkronq.so
 *   holds 4 MiB for it until the process exits.
 * - The first call on a device looks up the array's device address, with
 *   that device current, and caches it. Make that first call before any
 *   stream capture on the device.
 * - All calls share the one array. It keeps the last call's contents, but
 *   nothing in it has to start at zero: every byte a call reads is written
 *   earlier in the same call.
 * - Calls that overlap on the GPU (other streams, other host threads) race
 *   on the array. Serialise them.
 * - The cached address belongs to the device's current CUDA context; do not
 *   keep using the library across cudaDeviceReset in the same process.
 * - Sizes whose scratch would not fit return KRONQ_ERR_UNSUPPORTED. Every
 *   size that kronq_biip accepts (d <= 65536, m <= 256) fits.
 */
kronq_status kronq_biip_noalloc(kronq_stream_t stream, const kronq_opts *opts,
                                const void *W, kronq_dtype wdtype,
                                int64_t d_out, int64_t d_in, float *W_rot,
                                float *H_X, float *H_G, float *s_x, float *s_g,
                                int32_t *info_dev);

/*
 * Step 4 — damped inverse Cholesky factor [wmrh §四; GPTQ-style OBS needs
 * the upper factor of the inverse Hessian].
 * In: H (d x d fp32, full symmetric, e.g. H_X'). Out, in place: U upper
 * triangular with U^T U = (H + lambda I)^-1, lambda = damp_rel * mean(diag H),
 * strict lower triangle set to 0. Computed as H + lambda I = R R^T (R upper,
 * reverse-order Cholesky) and U = R^-1, in fp32 with 3xTF32 tensor-core
 * trailing updates. Requires d % 128 == 0. info: NOT_PD with the column;
 * NONFINITE when the mean of the diagonal is not finite.
 * Shared state: the recursion forks onto CUDA streams and events that the
 * library creates once per device and keeps. Calls on one device from several
 * host threads are therefore serialised: each call holds a per-device lock
 * while it enqueues, and its work queues behind the previous call's work on
 * those internal streams.
 */
kronq_status kronq_chol_inv(kronq_stream_t stream, float *H, int64_t d,
                            float damp_rel, void *ws, size_t ws_bytes,
                            int32_t *info_dev);

/*
 * Step 5 — blocked column-wise OBS quantization [gptget-en Methodology;
 * wmrh §四, §五]. See the quantizer spec above.
 * W_rot: d_out x d_in fp32; in: the weights to quantize (W' after BiIP);
 * out: the dequantized weights w_hat. U: d_in x d_in from kronq_chol_inv.
 * codes: d_out x (bits*d_in/32) uint32. scales: d_out x (d_in/group) fp32.
 * zeros: d_out x (d_in/group) uint8. opts: bits, group, block used.
 * Requires d_in % 128 == 0.
 */
kronq_status kronq_quantize_sublayer(kronq_stream_t stream,
                                     const kronq_opts *opts, float *W_rot,
                                     const float *U, int64_t d_out,
                                     int64_t d_in, uint32_t *codes,
                                     float *scales, uint8_t *zeros, void *ws,
                                     size_t ws_bytes, int32_t *info_dev);

/*
 * Measurement — the Kronecker-factored layer loss [aimodeling: H ≈ H_X ⊗ H_G;
 * wmrh §二]: *loss_dev = tr(H_G dW H_X dW^T) with dW = W_ref - W_hat, summed in
 * fp64 over fp32 products (fp32-accurate tensor-core GEMMs). d_in, d_out % 128
 * == 0. ws: kronq_workspace_bytes(KRONQ_WS_LOSS, ...). info_dev: TIMEOUT when
 * a GEMM pipeline wait ran out (the loss is then not valid).
 */
kronq_status kronq_layer_loss(kronq_stream_t stream, const float *W_ref,
                              const float *W_hat, const float *H_X,
                              const float *H_G, int64_t d_out, int64_t d_in,
                              double *loss_dev, void *ws, size_t ws_bytes,
                              int32_t *info_dev);

/*
 * Diagnostics (no counterpart on the pages): exercises the library's bounded
 * device wait. One kernel waits on a shared-memory barrier that nothing
 * completes, through the same wait routine the tensor-core pipelines use,
 * with a limit of limit_ns (1 .. 1e9 ns) instead of their 4 s. The wait gives
 * up, the kernel writes KRONQ_ERR_TIMEOUT to *info_dev and returns; the CUDA
 * context stays usable. Lets a caller check, without any fault, that a wait
 * which runs out is reported rather than hanging.
 */
kronq_status kronq_selftest_timeout(kronq_stream_t stream, uint64_t limit_ns,
                                    int32_t *info_dev);

/*
 * fp32-accurate dense product, on the tensor cores (the contraction behind the
 * Cholesky recursion, the OBS trailing updates and the layer loss; the pages
 * name no such routine): C = alpha * A * B^T + beta * C with row-major
 * operands on the device,
 *   A: M x K (a_mn = 0, pitch lda) or its transpose stored K x M (a_mn = 1),
 *   B: N x K (b_mn = 0, pitch ldb) or its transpose stored K x N (b_mn = 1),
 *   C: M x N, pitch ldc; beta = 0 ignores the old C.
 * Each fp32 operand is split into a high and a low part and three MMAs
 * (hi*hi, hi*lo, lo*hi) accumulate in fp32: TF32 parts, or, for large
 * products when ws holds kronq_gemm_f32_workspace_bytes(M, N, K) bytes
 * (device, 256-byte aligned, busy until the product completes on the stream),
 * fp16 parts of the operand rows scaled by powers of two. ws may be NULL.
 * Small products (M * N * K <= 2^24) skip the split and run as plain fp32
 * FMA on the CUDA cores, where a tensor-core pipeline costs more to set up
 * than it saves. Pointers 16-byte aligned, pitches multiples of 4 elements; M, N, K >= 0.
 * C must not overlap A or B. INVALID_ARG for negative sizes or null
 * pointers, UNSUPPORTED for misaligned operands, TIMEOUT in *info_dev
 * (nonzero) if a pipeline wait ran out.
 */
kronq_status kronq_gemm_f32(kronq_stream_t stream, int64_t M, int64_t N,
                            int64_t K, float alpha, const float *A, int64_t lda,
                            int a_mn, const float *B, int64_t ldb, int b_mn,
                            float beta, float *C, int64_t ldc, void *ws,
                            size_t ws_bytes, int32_t *info_dev);
/* Workspace bytes that let kronq_gemm_f32 take the fp16 path (0 if M, N or
 * K <= 0). */
size_t kronq_gemm_f32_workspace_bytes(int64_t M, int64_t N, int64_t K);

/*
 * Steps 4 and 5 in split form (no counterpart on the pages: a cheaper route
 * to the same OBS decisions). With H + λI = R Rᵀ (R upper) and U = R^-1,
 * kronq_chol_split leaves
 *     H = [U11, R12; 0, U22],  split at h = kronq_chol_split_point(d)
 *                              = 128 * floor(d / 256),
 * i.e. the root block right of the split keeps the Cholesky factor R12
 * instead of the inverse factor U12, which saves the two products that form
 * U12 (about d^3/4 flop of the 2 d^3/3). Same arguments, workspace
 * (KRONQ_WS_CHOL) and errors as kronq_chol_inv; d >= 256.
 *
 * kronq_quantize_split runs the OBS sweep of kronq_quantize_sublayer on that
 * form: the first h columns with U11, then the second half starting from
 *     W2 + ((W1 - What1) R12) U22
 * (the GPTQ recursion gives E U = W - What for the scaled errors E, so the
 * first half reaches the second through R12 alone), with U22. The decisions
 * are those of the one-pass sweep with the full U; the extra product costs
 * d_out * m^2 flop (m = d_in - h), so the split pays when d_in > d_out.
 * Arguments as kronq_quantize_sublayer with F the output of kronq_chol_split;
 * workspace KRONQ_WS_QUANT_SPLIT; d_in >= 256.
 */
kronq_status kronq_chol_split(kronq_stream_t stream, float *H, int64_t d,
                              float damp_rel, void *ws, size_t ws_bytes,
                              int32_t *info_dev);
int64_t kronq_chol_split_point(int64_t d);
kronq_status kronq_quantize_split(kronq_stream_t stream, const kronq_opts *opts,
                                  float *W_rot, const float *F, int64_t d_out,
                                  int64_t d_in, uint32_t *codes, float *scales,
                                  uint8_t *zeros, void *ws, size_t ws_bytes,
                                  int32_t *info_dev);

/*
 * Using the quantized sublayer [aimodeling: packed low-bit weights applied
 * through a fused dequant + BiIP matvec; wmrh Q2: the two Hadamard transforms
 * per layer at inference]. For n_tokens activations x (rows of an
 * n_tokens x d_in fp32 matrix) the call computes, in the original basis,
 *     y = S_G^-1 U_G^T W_hat' U_X S_X^-1 x      (y: n_tokens x d_out fp32)
 * with W_hat'[i][c] = scales[i][c/group] * (q[i][c] - zeros[i][c/group]) read
 * straight from the packed codes of kronq_quantize_sublayer (never expanded in
 * memory), and the rotations of the spec above (opts: the same bits, group,
 * seed, rot_in, rot_out and flags as the BiIP and OBS calls that produced the
 * codes; s_x, s_g: the scales kronq_biip returned).
 * kronq_matvec_prepare fills a caller-owned descriptor (device, 256-byte
 * aligned, kronq_matvec_desc_bytes bytes) with the per-side factors sign/s
 * and the Q_m factors once; kronq_dequant_matvec then needs a workspace of
 * kronq_matvec_workspace_bytes(d_out, d_in, n_tokens) bytes. x, y and codes
 * 16-byte aligned; n_tokens <= 4096 (the codes are streamed once per
 * token, the decode case is one token). info_dev: 0 (no numerical check is
 * made).
 */
size_t kronq_matvec_desc_bytes(const kronq_opts *opts, int64_t d_out, int64_t d_in);
size_t kronq_matvec_workspace_bytes(int64_t d_out, int64_t d_in, int64_t n_tokens);
kronq_status kronq_matvec_prepare(kronq_stream_t stream, const kronq_opts *opts,
                                  const float *s_x, const float *s_g, int64_t d_out,
                                  int64_t d_in, void *desc, size_t desc_bytes);
kronq_status kronq_dequant_matvec(kronq_stream_t stream, const kronq_opts *opts,
                                  const void *desc, const uint32_t *codes,
                                  const float *scales, const uint8_t *zeros, int64_t d_out,
                                  int64_t d_in, const float *x, int64_t n_tokens, float *y,
                                  void *ws, size_t ws_bytes, int32_t *info_dev);

/* Workspace bytes needed by one call (opts may be NULL except for BIIP and
 * QUANT). Returns 0 for unsupported arguments. */
size_t kronq_workspace_bytes(kronq_ws_kind which, int64_t d_out, int64_t d_in,
                             const kronq_opts *opts);

/*
 * Mixed-precision bit allocation [wmrh §六: upgrade the most sensitive
 * sublayers first]. HOST pointers. All sublayers start at 2 bits; pass 1
 * visits them in descending score (ties: lower index first) and upgrades
 * 2 -> 3 when the parameter-weighted mean bit width stays <= avg_budget;
 * pass 2 does the same for 3 -> 4. bits_out[i] in {2,3,4}.
 * KRONQ_ERR_INVALID_ARG for n <= 0, null pointers, numel <= 0, non-finite
 * scores or avg_budget < 2.
 */
kronq_status kronq_allocate_bits(const double *score, const int64_t *numel,
                                 int n, double avg_budget, int *bits_out);

/* Static, human-readable name of a status code. */
const char *kronq_status_string(kronq_status s);

/* Diagnostics (no counterpart on the pages): the number of CUDA kernels this
 * process has launched through the library since it was loaded. Host call,
 * thread-safe, never fails. */
uint64_t kronq_kernel_launches(void);

/* Diagnostics: the CUDA runtime's description of the last CUDA call that made
 * an entry point return KRONQ_ERR_CUDA in this process ("no error" if none).
 * Static string owned by the CUDA runtime; host call, never fails. */
const char *kronq_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* KRONQ_H */
