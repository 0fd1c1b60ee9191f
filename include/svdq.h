/*
 * svdq.h — C ABI of the B200 (sm_100a) SVDQuant W4A4 NVFP4 linear layer.
 *
 * The layer (blog "Bringing Nunchaku 4-bit Diffusion Inference to Diffusers",
 * sections "Background: SVDQuant and Nunchaku" and "Introducing Nunchaku Lite"):
 *
 *     Y = (X . L1) . L2  +  Q4(X) . Q4(R)^T  +  b,        R = W - (L1 . L2)^T
 *
 * X: M x K activations (bf16), W: N x K weight (bf16), L1: K x r and L2: r x N
 * the 16-bit low-rank factors (bf16), b: N bias (bf16), Y: M x N (bf16).
 * Q4 is NVFP4: one E2M1 code per element, one E4M3 scale per 16 contiguous
 * K-elements ("group_size": 16 in the blog's quantization_config), and one
 * FP32 decode scale per tensor (g_x for X, g_w for R).
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never allocates or frees device memory. Buffers must be 16-byte aligned.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; no call synchronises the host, except
 *    svdq_read_device_error.
 *  - Every function returns an svdq_status. Arguments are validated on the
 *    host before any launch; an invalid call launches nothing and returns
 *    SVDQ_ERR_INVALID_ARG / _UNSUPPORTED_SHAPE / _MISALIGNED. A device that is
 *    not compute capability 10.0 (B200, sm_100a) gives
 *    SVDQ_ERR_UNSUPPORTED_DEVICE (the blog's hardware section: the quantizer
 *    checks the GPU's capability and raises a clear error rather than produce
 *    wrong outputs). A failed launch gives SVDQ_ERR_CUDA.
 *  - Kernels never spin without bound. A wait that exceeds its limit records
 *    SVDQ_ERR_TIMEOUT in a per-device error word and the kernel returns;
 *    svdq_read_device_error reports it after the caller synchronises.
 *  - Shape rules: K % 256 == 0, N % 128 == 0, r in {16, 32, 64, 128},
 *    M >= 0 (M == 0 is a no-op). Leading dimensions are in elements, multiples
 *    of 8 and at least the row length.
 *
 * Data layouts (all row-major)
 * ----------------------------
 *  codes   uint8 [rows][K/2]; byte j holds element 2j in bits 0..3 and element
 *          2j+1 in bits 4..7. E2M1 code: sign bit 3, exponent bits 2..1 (bias
 *          1), mantissa bit 0.
 *  scales  uint8 E4M3 codes (bias 7, max 448), one per 16 K-elements, in a
 *          tiled order the tensor cores read directly: rows are padded to a
 *          multiple of 128; the byte of (row, kb) with kb = k/16 sits at
 *              ((row/128) * (K/64) + kb/4) * 512 + (row%32) * 16
 *                  + ((row%128)/32) * 4 + kb%4
 *          (svdq_scale_offset computes it on the host).
 *  gscale  fp32 [4] (device): {g_x, g_w, alpha = fp32(g_x * g_w), 0}
 *  l1t     bf16 [r][K]   = L1 transposed (packed by svdq_pack_weight)
 *  l2s     bf16 [2][N][r]: the up-projection pre-divided by alpha, split in
 *          two bf16 parts so that hi + lo = L2^T / alpha to ~2^-17:
 *          v = fp32(L2[j][n] / alpha), hi = bf16(v), lo = bf16(v - hi);
 *          plane 0 holds hi, plane 1 holds lo. (The 4-bit product and the
 *          low-rank product then share one fp32 accumulator, which the
 *          epilogue multiplies by alpha once.)
 *  xl1     bf16 [M][r]   = bf16(X . L1), fp32 accumulation
 *  inv_smooth  fp32 [K]  = fp32(1 / lambda), the smoothing factors of a
 *          smoothed layer (written by svdq_pack_weight), or NULL
 *
 * Entry points
 * ------------
 *  load time   svdq_smooth_factors (calibration of the smoothing), svdq_lowrank_init
 *              (truncated SVD on the GPU), svdq_act_global_scale (calibrated g_x),
 *              svdq_pack_weight
 *  per call    svdq_quantize_act + svdq_w4a4_gemm, or svdq_linear_forward (both),
 *              svdq_linear_forward_dynamic (g_x from each call's X),
 *              svdq_linear_forward_noalloc (no workspace argument),
 *              svdq_linear_forward_qkv (fused QKV: per-head RMSNorm + rotary),
 *              svdq_mlp_up_forward (MLP pair: GELU and the down projection's
 *              quantised input in the up projection's epilogue)
 *  AWQ W4A16   svdq_awq_pack, svdq_awq_gemv (weight-only INT4, group 64)
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,        /* null pointer, negative size, bad rank */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2,  /* K % 256, N % 128, leading dimension  */
  SVDQ_ERR_MISALIGNED = 3,         /* a pointer not 16-byte aligned          */
  SVDQ_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 / no GPU  */
  SVDQ_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed   */
  SVDQ_ERR_TIMEOUT = 6,            /* a kernel wait ran out (device error)   */
  SVDQ_ERR_WORKSPACE = 7           /* workspace too small                    */
} svdq_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(int status);

/* Library version, major*10000 + minor*100 + patch. */
int svdq_version(void);

/* Byte offset of the E4M3 scale of (row, kblock) in the tiled scale layout
 * described above, for a tensor with K columns. Host-only, pure function.
 * Errors: INVALID_ARG if row < 0, kblock outside [0, K/16) or out == NULL;
 * UNSUPPORTED_SHAPE if K % 64 != 0. */
svdq_status svdq_scale_offset(int K, int row, int kblock, size_t* out);

/* The device rule every entry point applies (host only, no device needed):
 * SVDQ_OK for compute capability 10.0 (B200; the kernels are built for
 * sm_100a), SVDQ_ERR_UNSUPPORTED_DEVICE for any other capability. The blog's
 * hardware section: the GPU's capability is checked up front and an
 * unsupported GPU gets a clear error instead of wrong outputs. */
svdq_status svdq_device_supported(int major, int minor);

/* ------------------------------------------------------------ sizes (host) */
/* Bytes of each packed-weight buffer for an N x K weight with rank r. */
svdq_status svdq_weight_sizes(int N, int K, int r, size_t* codes_bytes, size_t* scales_bytes,
                              size_t* l1t_bytes, size_t* l2s_bytes);
/* Bytes of the quantised-activation buffers for M rows (scales padded to 128 rows). */
svdq_status svdq_act_sizes(int M, int K, int r, size_t* codes_bytes, size_t* scales_bytes,
                           size_t* xl1_bytes);
/* Workspace bytes svdq_linear_forward needs (activation codes, scales and XL1). */
svdq_status svdq_forward_workspace_size(int M, int K, int r, size_t* bytes);

/* ------------------------------------------------------------ load time */
/* Pack one layer (untimed, load time). Blog section "Background: SVDQuant and
 * Nunchaku": the low-rank branch holds the hardest part of the weight, the
 * remaining residual is quantised to 4 bits.
 *   W   bf16 [N][K], L1 bf16 [K][r], L2 bf16 [r][N]   (L1.L2 is the rank-r
 *       factorisation of W^T)
 *   smooth  device float [K] smoothing factors lambda (positive, finite), or
 *       NULL for none (lambda = 1). With smoothing (same section: outliers
 *       move from the activations into the weights) L1 must be the factor
 *       with 1/lambda folded in (svdq_lowrank_init with the same smooth), and
 *       the per-call functions must be given inv_smooth.
 *   g_x device float: the layer's calibrated (static) activation decode scale,
 *       e.g. from svdq_act_global_scale on calibration activations (with the
 *       same inv_smooth).
 *   Writes: w_codes [N][K/2], w_scales (tiled), gscale[4], l1t [r][K],
 *           l2s [2][N][r] (layouts above), and with smoothing inv_smooth
 *           [K] = fp32(1 / lambda) (16-byte aligned; NULL exactly when smooth
 *           is NULL, SVDQ_ERR_INVALID_ARG otherwise; a lambda that is not a
 *           positive finite number records SVDQ_ERR_INVALID_ARG in the device
 *           error word).
 * R[n,k] = lambda_k (W[n,k] - sum_j L1[k,j] L2[j,n]) is formed in float64
 * (j ascending, products exact; the multiplication by lambda_k is one more
 * float64 rounding) and rounded once to float32; g_w = fp32(amax|R| / 2688)
 * (1 if R == 0); then R is quantised with the NVFP4 rule of svdq_quantize_act.
 * Requires alpha = g_x g_w >= 2^-100 (so L2 / alpha stays finite in bf16).
 * The output buffers must not overlap the inputs. */
svdq_status svdq_pack_weight(int N, int K, int r, const void* W, const void* L1, const void* L2,
                             const float* smooth, const float* g_x, void* w_codes, void* w_scales,
                             float* gscale, void* l1t, void* l2s, float* inv_smooth, void* stream);

/* Smoothing calibration (load time): per input channel k,
 *     lambda_k = amax_m|X[m,k]|^alpha / amax_n|W[n,k]|^(1 - alpha)
 * in float64, clamped to [2^-32, 2^32], rounded once to fp32; lambda_k = 1
 * where either amax is 0. The blog (section "Background: SVDQuant and
 * Nunchaku") says outliers move from the activations into the weights but not
 * how the factors are chosen; this is SmoothQuant's rule (Xiao et al. 2023).
 * alpha = 0.5 is computed as sqrt(ax) / sqrt(aw), each step correctly rounded.
 * X bf16 [M][ldx] (calibration activations), W bf16 [N][K]; alpha in [0, 1];
 * lambda: device float [K]. */
svdq_status svdq_smooth_factors(int M, int N, int K, const void* X, int64_t ldx, const void* W, float alpha,
                                float* lambda, void* stream);

/* The layer followed by FLUX's fused QKV post-processing (blog, section
 * "Quantizing models with structural rewrites": one fused operator takes the
 * grouped QKV projection, the Q/K normalisation and the rotary embedding).
 * W is the grouped [Q; K; V] weight, N = 3 * heads * 128 (head_dim 128), and
 * Y is laid out [Q | K | V]. With q = bf16(layer output) per head row:
 *     n_i = q_i / sqrt(mean_i(q_i^2) + eps) * w_i       (w = norm_q_weight for
 *                                                        Q heads, norm_k_weight
 *                                                        for K heads; bf16[128])
 *     (n_2j, n_2j+1) -> (n_2j c_j - n_2j+1 s_j,  n_2j+1 c_j + n_2j s_j)
 * (each pair rotated by the angle theta_j of its token), with c_j =
 * rope_cos[m][j] = cos(theta_j), s_j = rope_sin[m][j] (float32 [M][ld_rope],
 * 64 used per token), computed in fp32 and rounded to bf16 once; V columns
 * are the plain layer output. Other arguments, the workspace and the shape
 * rules are those of svdq_linear_forward; additionally N == 3 * heads * 128,
 * ld_rope >= 64 and ld_rope % 4 == 0, norm weights and rope tables 16-byte
 * aligned, 0 <= eps. The normalisation and rotation happen in the GEMM's
 * epilogue (no extra pass over Y). */
svdq_status svdq_linear_forward_qkv(int M, int N, int K, int r, const void* X, int64_t ldx,
                                    const void* w_codes, const void* w_scales, const float* gscale,
                                    const void* l1t, const void* l2s, const float* inv_smooth,
                                    const void* bias, int heads,
                                    const void* norm_q_weight, const void* norm_k_weight, float eps,
                                    const float* rope_cos, const float* rope_sin, int64_t ld_rope,
                                    void* Y, int64_t ldy, void* workspace, size_t workspace_bytes,
                                    void* stream);

/* Load time (S0): the rank-r factors of the 16-bit branch from a truncated
 * SVD of W^T (blog, section "Background: SVDQuant and Nunchaku": the branch
 * holds the weight's dominant singular directions). With W^T = U S V^T:
 *     L1 = bf16(U_r S_r)   (K x r, row-major)
 *     L2 = bf16(V_r^T)     (r x N, row-major)
 * computed in float64 by randomized subspace iteration (Halko, Martinsson and
 * Tropp 2011): a Gaussian sketch of r + 32 columns drawn from `seed` by a
 * counter-based generator, `power_iters` power iterations (each re-
 * orthonormalised by shifted Cholesky QR), then the exact SVD of the sketched
 * problem (two-sided Jacobi on its Gram matrix). The result is deterministic
 * for a given seed. It approaches the optimal rank-r factors as power_iters
 * grows: separated singular values converge fast; on a flat spectrum with
 * power_iters = 32 the residual energy ||W^T - L1 L2||_F^2 is within about
 * 2e-4 of the Eckart-Young minimum (rank 128; 1e-6 at rank 32). sigma
 * (device, r doubles, may be NULL) receives S_r in decreasing order.
 * Shapes: r in {16, 32, 64, 128}, r <= min(N, K), K % 8 == 0 (N and K need not
 * satisfy the GEMM's rules). W, L1, L2 16-byte aligned, sigma 8-byte aligned,
 * workspace 256-byte aligned and at least svdq_lowrank_workspace_size bytes
 * (SVDQ_ERR_WORKSPACE otherwise); power_iters in [0, 64].
 * With smoothing (smooth: device float [K] lambda, 16-byte aligned, or NULL)
 * the matrix decomposed is diag(lambda) W^T and L1 = bf16(U_r S_r / lambda_k
 * per row, in float64), so X . L1 = X^ . U_r S_r for X^ = X diag(1/lambda).
 * The blog does not say how the SVD is computed; this is the load-time step
 * that feeds svdq_pack_weight. */
svdq_status svdq_lowrank_workspace_size(int N, int K, int r, size_t* bytes);
svdq_status svdq_lowrank_init(int N, int K, int r, const void* W, const float* smooth, void* L1, void* L2,
                              double* sigma, unsigned long long seed, int power_iters, void* workspace,
                              size_t ws_bytes, void* stream);

/* Activation scale: *g_out = fp32(amax|X^| / 2688), or 1 for an all-zero X,
 * with X^ = fp32(x * inv_smooth[k]) (inv_smooth: device float [K], 16-byte
 * aligned, or NULL for X^ = X). X bf16 [M][ldx]; g_out is a device float.
 * Run once on calibration activations it gives the static g_x. */
svdq_status svdq_act_global_scale(int M, int K, const void* X, int64_t ldx, const float* inv_smooth,
                                  float* g_out, void* stream);

/* ------------------------------------------------------------ per call */
/* Activation quantisation fused with the low-rank down projection (blog
 * figure caption in "Background: SVDQuant and Nunchaku": the down projection
 * is fused with the quantisation kernel). One pass over X [M][ldx] (bf16):
 *   x^ = fp32(x * inv_smooth[k]) with smoothing, else x;
 *   per 16-element block of x^: S = e4m3_rn_sat(amax / fp32(6 g_x)),
 *   sd = fp32(dec(S) g_x), code = e2m1_rn_sat(fp32(x^ * fp32(1/sd))) (0 if sd == 0);
 *   xl1 = bf16(X . L1) of the raw X, with fp32 accumulation (L1 given as
 *   l1t [r][K]; with smoothing it carries 1/lambda).
 * g_x is a device float (gscale[0] of a packed layer); inv_smooth is the
 * packed layer's [K] floats (16-byte aligned) or NULL.
 * Writes codes [M][K/2], scales (tiled, rows padded to 128; padding rows are
 * written as zero scales), xl1 [M][r]. Deterministic. */
svdq_status svdq_quantize_act(int M, int K, int r, const void* X, int64_t ldx, const float* g_x,
                              const void* l1t, const float* inv_smooth, void* codes, void* scales, void* xl1,
                              void* stream);

/* The block-scaled FP4 GEMM with the low-rank up projection and bias fused in
 * its epilogue (blog figure caption: the up projection is fused with the 4-bit
 * compute kernel):
 *   Y[m,n] = bf16( alpha * ( sum_k dec(Xc)dec(SX) dec(Rc)dec(SR)
 *                            + sum_j xl1[m,j] (hi + lo)[n,j] ) + b[n] )
 *          = bf16( g_x g_w * Q4(X).Q4(R)^T + xl1 . L2 + b )   (to fp32 accuracy)
 * a_codes/a_scales/xl1 as written by svdq_quantize_act; w_codes, w_scales,
 * gscale, l2s as written by svdq_pack_weight; bias may be NULL; Y bf16 [M][ldy]. */
svdq_status svdq_w4a4_gemm(int M, int N, int K, int r, const void* a_codes, const void* a_scales,
                           const void* xl1, const void* w_codes, const void* w_scales, const float* gscale,
                           const void* l2s, const void* bias, void* Y, int64_t ldy, void* stream);

/* The whole layer: svdq_quantize_act (with g_x = gscale[0] and inv_smooth)
 * into `workspace`, then svdq_w4a4_gemm.
 * workspace_bytes must be >= svdq_forward_workspace_size(M, K, r). */
svdq_status svdq_linear_forward(int M, int N, int K, int r, const void* X, int64_t ldx,
                                const void* w_codes, const void* w_scales, const float* gscale,
                                const void* l1t, const void* l2s, const float* inv_smooth,
                                const void* bias, void* Y, int64_t ldy, void* workspace,
                                size_t workspace_bytes, void* stream);

/* The whole layer with a dynamic activation scale: g_x is computed from this
 * call's X instead of the calibrated gscale[0]:
 *     g = fp32(amax|X^| / 2688)  (1 for an all-zero X^; X^ = X * inv_smooth),
 *     alpha' = fp32(g g_w),
 * and the packed hi/lo planes of L2^T / alpha are re-expressed for alpha'
 * (v = hi + lo, v' = fp32(v fp32(alpha / alpha')), hi' = bf16(v'),
 * lo' = bf16(v' - hi'); unchanged when alpha' == alpha). Then the layer runs as
 * svdq_linear_forward with these scales. This costs one more read of X (the
 * amax pass) and a pass over the N x r planes. The blog does not say whether
 * the activation scale is calibrated or per call; this entry point is the
 * per-call reading, svdq_linear_forward the calibrated one.
 * Workspace: svdq_dynamic_workspace_size(M, N, K, r) bytes, 256-byte aligned;
 * after the call it holds, at offset svdq_forward_workspace_size(M, K, r),
 * the floats {g, g_w, alpha', amax}. Other arguments as
 * svdq_linear_forward. */
svdq_status svdq_dynamic_workspace_size(int M, int N, int K, int r, size_t* bytes);
svdq_status svdq_linear_forward_dynamic(int M, int N, int K, int r, const void* X, int64_t ldx,
                                        const void* w_codes, const void* w_scales, const float* gscale,
                                        const void* l1t, const void* l2s, const float* inv_smooth,
                                        const void* bias, void* Y, int64_t ldy, void* workspace,
                                        size_t workspace_bytes, void* stream);

/* Same computation as svdq_linear_forward, for callers that cannot supply a
 * workspace: plugin interfaces of inference runtimes that pass only a layer's
 * inputs and outputs, and code running after the process has fixed its device
 * memory budget, where calling an allocator is not allowed. (The blog has no
 * counterpart; this is an interface convenience.)
 *   - Allocates nothing. The intermediates go to one fixed scratch array of
 *     16 MiB (16777216 bytes) inside the library, which every GPU that loads
 *     the library keeps until the process exits.
 *   - Shapes whose svdq_forward_workspace_size exceeds that limit are rejected
 *     with SVDQ_ERR_WORKSPACE (and a message on stderr) before any launch;
 *     e.g. M=4608, K=3072, r=32 (8.3 MB) fits, M=18432, K=3072 does not.
 *   - The first call on a device looks up the scratch array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture on that device.
 *   - All calls on a device share the scratch: calls that may overlap on the
 *     GPU (different streams, or several host threads) race and must be
 *     serialised by the caller. No part of the scratch needs to start at zero.
 * Arguments, layouts and errors otherwise as svdq_linear_forward. */
svdq_status svdq_linear_forward_noalloc(int M, int N, int K, int r, const void* X, int64_t ldx,
                                        const void* w_codes, const void* w_scales, const float* gscale,
                                        const void* l1t, const void* l2s, const float* inv_smooth,
                                        const void* bias, void* Y, int64_t ldy, void* stream);

/* ------------------------------------------------------------ MLP pair */
/* The up projection of a transformer block's feed-forward pair with GELU and
 * the down projection's activation quantisation fused into its GEMM epilogue
 * (blog section "Introducing Nunchaku Lite": part of the full engine's speed
 * comes from fused GELU / MLP kernels). For the layer X [M][K] -> N (arguments as
 * svdq_linear_forward):
 *   y = bf16(layer output), h = bf16(GELU(y)) (GELU = x Phi(x), or with
 *   approximate != 0 its tanh form; fp32, evaluated without cancellation in
 *   the negative tail),
 * and h is written directly as the down projection's quantised activation:
 *   h_codes  [M][N/2], h_scales (tiled, rows padded to 128, padding zero):
 *            the NVFP4 rule of svdq_quantize_act with g = *g_h;
 *   h_xl1    [M][r_down] = bf16(h . L1_down), given l1t_down = L1_down^T,
 *            bf16 [r_down][N] row-major (the l1t that svdq_pack_weight writes
 *            for the down projection); accumulated in fp32 on the tensor cores
 *            over each CTA pair's run of tiles sharing their rows, one partial
 *            per run, the partials summed in tile order (deterministic).
 * These are the buffers svdq_w4a4_gemm takes as a_codes, a_scales and xl1 for
 * the down projection (a QuantAct of M rows, K = N, rank r_down). h itself is
 * stored only when h_out (bf16 [M][ldh]) is given. Requires N % 256 == 0 (the
 * CTA-pair GEMM) and r_down == 32. Workspace: svdq_mlp_workspace_size bytes,
 * 16-byte aligned. */
svdq_status svdq_mlp_workspace_size(int M, int N, int K, int r, int r_down, size_t* bytes);
svdq_status svdq_mlp_up_forward(int M, int N, int K, int r, const void* X, int64_t ldx, const void* w_codes,
                                const void* w_scales, const float* gscale, const void* l1t, const void* l2s,
                                const float* inv_smooth, const void* bias, int r_down, const float* g_h,
                                const void* l1t_down, int approximate, void* h_codes, void* h_scales, void* h_xl1,
                                void* h_out, int64_t ldh, void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------ AWQ W4A16 */
/* The second kernel family of the blog's section "Introducing Nunchaku Lite":
 * awq_w4a16, 4-bit weights with 16-bit activations for the adaptive-
 * normalisation and modulation projections (memory-bound, precision-
 * sensitive); section "Native loading in Diffusers": int4, group size 64,
 * bfloat16. Layout of a packed N x K weight (K % 64 == 0):
 *   codes  u8 [N][K/2], element 2j in the low nibble of byte j
 *   scales bf16 [N][K/64], zeros u8 [N][K/64] (one per row and 64-group)
 * Sizes in bytes: */
svdq_status svdq_awq_sizes(int N, int K, size_t* codes_bytes, size_t* scales_bytes, size_t* zeros_bytes);

/* Quantise W bf16 [N][K] (load time). Per row and 64-group of w = fp32(W *
 * act_scale[k]) (or W), the AWQ reference pseudo-quantiser's rule, every step
 * one correctly rounded fp32 operation:
 *   s = bf16(fp32(max(fp32(max w - min w), 1e-5) / 15)),
 *   z = clamp(rne(fp32(-min w / s)), 0, 15),
 *   q = clamp(rne(fp32(w / s)) + z, 0, 15).
 * act_scale: device float [K] activation-aware factors a_k (positive, finite),
 * or NULL; with it inv_act [K] receives fp32(1 / a_k) (NULL exactly when
 * act_scale is NULL; both 16-byte aligned). W and codes 16-byte aligned,
 * scales 2-byte aligned. Deterministic. */
svdq_status svdq_awq_pack(int N, int K, const void* W, const float* act_scale, void* codes, void* scales,
                          void* zeros, float* inv_act, void* stream);

/* Y[m,n] = bf16( sum_k x^[m,k] (q[n,k] - z[n,g]) s[n,g] + b[n] ), g = k / 64,
 * x^ = fp32(x * inv_act[k]) (or x); the dequantised weight is exact in fp32 and
 * the sum is accumulated in fp32. X bf16 [M][ldx] (ldx % 8 == 0, 16-byte
 * aligned), Y bf16 [M][ldy], bias bf16 [N] or NULL, inv_act float [K]
 * (16-byte aligned) or NULL. Any M >= 0 (rows are processed eight at a time); K * 4 <= 96 KB. The
 * layer is HBM-bound for the few rows a modulation projection has: each warp
 * streams one weight row, the activations sit in shared memory. */
svdq_status svdq_awq_gemv(int M, int N, int K, const void* X, int64_t ldx, const void* codes, const void* scales,
                          const void* zeros, const float* inv_act, const void* bias, void* Y, int64_t ldy,
                          void* stream);

/* ------------------------------------------------------------ errors */
/* Reads (and, if clear != 0, resets) the device error word of the current
 * device: 0 or an svdq_status recorded by a kernel (e.g. SVDQ_ERR_TIMEOUT).
 * Synchronises the device first. */
svdq_status svdq_read_device_error(int* code, int clear);

/* Self-test of the bounded waits (blog section "Hardware support": a failure
 * must surface as a clear error, not as wrong outputs or a hung process).
 * Every kernel of this library waits on mbarriers with a time limit; when a
 * limit runs out the kernel records SVDQ_ERR_TIMEOUT in the per-device error
 * word and returns. This call launches one small kernel, asynchronously on
 * `stream`, whose single wait is on an mbarrier that nothing ever arrives on,
 * with a limit of limit_us microseconds (1 .. 1000000; otherwise
 * SVDQ_ERR_INVALID_ARG and no launch). After the caller synchronises,
 * svdq_read_device_error returns SVDQ_ERR_TIMEOUT, and the CUDA context stays
 * usable: the kernel ends normally, with no trap and no fault. Nothing else
 * is read or written. */
svdq_status svdq_selftest_bounded_wait(int limit_us, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
