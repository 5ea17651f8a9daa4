/*
 * svdq.h -- C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SVDQuant, "Absorbing outliers by low-rank components for 4-bit
 * diffusion models"; abstract as translated on ai-digest.ru, and the
 * "technical principles" section of chattools.cn article 584):
 *
 *     Y = Xh L1 L2 + Q(Xh) Q(R) + bias,      Xh = X diag(lambda)^-1
 *
 * X [M][K] is the activation, lambda [K] the smoothing factors that move
 * activation outliers into the weights, L1 [K][r] and L2 [r][N] the 16-bit
 * low-rank branch from the SVD of diag(lambda) W, R = diag(lambda) W - L1 L2
 * the residual, and Q() the 4-bit NVFP4 quantiser: E2M1 values with one
 * unsigned E4M3 scale per 16 consecutive elements along K, scale = amax / 6.
 * The pages' engine fuses the low-rank branch into the 4-bit kernels to avoid
 * a second pass over the activation (ai-digest.ru abstract, chattools.cn
 * "kernel fusion" bullet); here the down-projection Xh L1 shares the
 * quantiser's read of X and the up-projection (Xh L1) L2 accumulates into
 * the 4-bit GEMM's tensor-memory accumulator.
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensors are dense, row-major, in DEVICE memory, allocated and owned
 *    by the caller.  The library allocates no device memory.  Its host-side
 *    state is a cache of encoded TMA descriptors (a pure function of the
 *    buffers' addresses and shapes, so reuse is always valid) and the
 *    kernels' shared-memory limits set per device; on the device it keeps a
 *    per-device status word (see svdq_sync_status).  All calls are safe to
 *    make from several host threads.
 *  - bf16 tensors are passed as `const void*` / `void*` (IEEE bfloat16).
 *  - Every pointer must be 16-byte aligned.  K must be a multiple of 64,
 *    N a multiple of 16, r one of 0, 16, 32, ..., 128, M >= 1.  Sizes are
 *    bounded by M, N <= 2^22 and K <= 2^20 (SVDQ_ERR_UNSUPPORTED_SHAPE
 *    beyond), which keeps every grid dimension and index in range.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    are asynchronous and stream-ordered; none synchronises.
 *  - Argument errors are detected on the host before anything is launched
 *    and returned as a status; no call aborts or exits.
 *  - Inputs must be finite; NaN or Inf gives unspecified codes.
 *  - LoRA adapters (chattools.cn, item "LoRA集成": no re-quantisation) need
 *    no call of their own: an adapter A [K][ra], B [ra][N] joins the
 *    low-rank branch as L1' = [L1 | bf16(lambda A)], L2' = [L2 ; B] (rank
 *    r + ra <= 128), since Xh diag(lambda) A = X A; R stays as packed.
 *
 * Packed NVFP4 layout (codes and scales)
 * --------------------------------------
 *  - codes: uint8 [rows][K/2]; element k of a row is in byte k/2, in the
 *    low nibble for even k and the high nibble for odd k.  E2M1 code: bit 3
 *    sign, bits 0-2 magnitude index into {0, .5, 1, 1.5, 2, 3, 4, 6}.
 *  - scales: uint8 unsigned-E4M3, one per 16 elements along K, in the
 *    tensor cores' block-scale tile layout: rows are padded to a multiple of
 *    128; tile (row/128, g/4) (g = k/16) is 512 contiguous bytes, tiles of a
 *    128-row band are consecutive along K, and inside a tile (row, g) is at
 *    byte (row % 32) * 16 + ((row % 128) / 32) * 4 + (g % 4).  Scales of the
 *    padding rows are written as 0.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,       /* null pointer, negative size */
  SVDQ_ERR_UNSUPPORTED_SHAPE = 2, /* K % 64, N % 16, r not in {0,16,...,128} */
  SVDQ_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  SVDQ_ERR_CUDA = 4,              /* a CUDA runtime/driver call failed */
  SVDQ_ERR_TIMEOUT = 5            /* a kernel's bounded wait expired */
} svdq_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(int status);

/* Bytes of the packed buffers for `rows` vectors of length K:
 * codes_bytes = rows * K / 2, scales_bytes = ceil(rows / 128) * 128 * K / 16.
 * Host-only; K must be a multiple of 64. */
svdq_status svdq_packed_sizes(int64_t rows, int64_t K, size_t* codes_bytes, size_t* scales_bytes);

/*
 * Residual packer, run once per weight (the 4-bit residual of the SVDQuant
 * principles: the part of diag(lambda) W left after removing the low-rank
 * branch is quantised to 4 bits).
 *   R        fp32 [K][N]   residual diag(lambda) W - L1 L2
 *   r_codes  uint8 [N][K/2]        output: NVFP4 codes, one row per output
 *                                   channel n, groups of 16 along K
 *   r_scales uint8, svdq_packed_sizes(N, K) bytes, tile layout above
 */
svdq_status svdq_pack_residual(const float* R, int64_t K, int64_t N, uint8_t* r_codes,
                               uint8_t* r_scales, void* stream);

/*
 * Workspace of svdq_quantize_act for these sizes on the current device, in
 * bytes (0 when the call needs none: r == 0, or enough rows that no tile is
 * split along K).  Host-only.
 */
svdq_status svdq_quantize_act_workspace(int64_t M, int64_t K, int64_t r, size_t* bytes);

/*
 * Activation step of one forward pass: smoothing, 4-bit quantisation and the
 * low-rank down-projection from one read of X.
 *   X          bf16 [M][K]
 *   inv_lambda fp32 [K]     1 / lambda_j, rounded to fp32 by the caller;
 *                           Xh = RN_f32(X * inv_lambda) element-wise
 *   L1         bf16 [K][r]  low-rank down-projection (NULL iff r == 0)
 *   x_codes    uint8 [M][K/2]               output: NVFP4 codes of Xh
 *   x_scales   uint8, svdq_packed_sizes(M, K) output: scales of Xh
 *   T          bf16 [M][r]  output: bf16(bf16(Xh) L1), fp32 accumulation
 *                           (NULL iff r == 0)
 *   workspace  device scratch of at least svdq_quantize_act_workspace()
 *              bytes, 16-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE
 *              (NULL allowed when that size is 0).  When there are fewer
 *              128-row tiles than SMs, the CTAs sharing a tile sum their
 *              partial T there in a fixed order; the call leaves the
 *              workspace's counters at zero again, so one zero fill serves
 *              all later calls.  Calls that may run concurrently (other
 *              streams) need workspaces of their own.
 * NVFP4 group rule (16 values v along K): s = E4M3_RNE_satfinite(
 * RN_f32(amax / 6)); rcp = RN_f32(1 / decode(s)) (0 if decode(s) == 0);
 * q_i = E2M1_RNE_satfinite(RN_f32(v_i * rcp)).
 */
svdq_status svdq_quantize_act(const void* X, const float* inv_lambda, const void* L1, int64_t M,
                              int64_t K, int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * The activation step on GELU inputs: svdq_quantize_act with
 *     Xh = RN_f32(GELU(x) * inv_lambda),
 * GELU(x) = 0.5 x (1 + erf(x / sqrt 2)) evaluated in fp32 (no bf16 rounding
 * between GELU and the smoothing multiply), erf by the purely rational
 * approximation of Abramowitz and Stegun, Handbook of Mathematical Functions,
 * 7.1.28 (|error| <= 3e-7; in fp32 about 1.5e-6), one rounded operation per
 * step in a fixed order so the codes are reproducible bit for bit.  The
 * MLP's activation then costs no pass of its own over the hidden states
 * (chattools.cn article 584, "Nunchaku": the low-rank and low-bit kernels
 * are fused to avoid redundant memory access; here the fusion reaches the
 * next layer's input).  Arguments, workspace and errors as svdq_quantize_act.
 */
svdq_status svdq_quantize_act_gelu(const void* X, const float* inv_lambda, const void* L1, int64_t M,
                                   int64_t K, int64_t r, uint8_t* x_codes, uint8_t* x_scales, void* T,
                                   void* workspace, size_t workspace_bytes, void* stream);

/*
 * Fused 4-bit linear: Y = deq(x) deq(R)^T + T L2 + bias, written as bf16.
 * The block-scaled FP4 product and the rank-r bf16 product accumulate in
 * the same fp32 tensor-memory accumulator; bias is added in fp32 and the
 * result rounded once to bf16.
 *   x_codes, x_scales   from svdq_quantize_act (M rows)
 *   T                   bf16 [M][r] (NULL iff r == 0)
 *   r_codes, r_scales   from svdq_pack_residual (N rows)
 *   L2                  bf16 [r][N] (NULL iff r == 0)
 *   bias                bf16 [N] or NULL
 *   Y                   bf16 [M][N] output
 */
svdq_status svdq_linear(const uint8_t* x_codes, const uint8_t* x_scales, const void* T,
                        const uint8_t* r_codes, const uint8_t* r_scales, const void* L2,
                        const void* bias, int64_t M, int64_t K, int64_t N, int64_t r, void* Y,
                        void* stream);

/*
 * NVFP4 with per-tensor global scales (the NVFP4 format named by the
 * taicenter.com article on Han Song's team and FLUX carries an fp32 scale per
 * tensor above the per-16 E4M3 scales).  With global scales g_x for Xh and
 * g_w for R, a group encodes as s = E4M3_RNE_satfinite(RN_f32(s_f / g)) and
 * dequantises to q * decode(s) * g, and the layer is
 *     Y = g_x g_w deq(x) deq(R)^T + T L2 + bias.
 * For powers of two g this encoding of Z is exactly the plain encoding of
 * Z / g, so the plain calls serve it on pre-scaled operands:
 *   svdq_quantize_act with inv_lambda / g_x  -> x codes, scales, and T / g_x
 *   svdq_pack_residual of R / g_w            -> r codes, scales
 *   svdq_linear_scaled with L2 / g_w and alpha = g_x g_w
 * (every pre-scale is exact).  svdq_linear_scaled is svdq_linear with the
 * accumulator multiplied by alpha before the bias is added:
 *     Y = bf16(acc * alpha + bias),
 * alpha a power of two in [2^-100, 2^100] (SVDQ_ERR_INVALID_ARG otherwise),
 * so the product is exact; alpha = 1 is svdq_linear.
 */
svdq_status svdq_linear_scaled(const uint8_t* x_codes, const uint8_t* x_scales, const void* T,
                               const uint8_t* r_codes, const uint8_t* r_scales, const void* L2, const void* bias,
                               int64_t M, int64_t K, int64_t N, int64_t r, float alpha, void* Y, void* stream);

/*
 * LoRA adapter joined to the low-rank branch, on the device (chattools.cn
 * article 584, "main functions", item LoRA integration: adapters apply to
 * the quantised model without re-quantising it).  With Xh = X
 * diag(lambda)^-1, the adapter A [K][ra], B [ra][N] (bf16) joins as
 *     L1_out [K][r + ra] = [L1 | bf16(RN_f32(lambda_k * A_kj))]
 *     L2_out [r + ra][N] = [L2 ; B]
 * so that Xh L1_out L2_out = Xh L1 L2 + X A B; the packed residual is
 * unchanged and the layer then runs with rank r + ra through
 * svdq_quantize_act / svdq_linear.  Adapters chain: the outputs may be the
 * inputs of a further call.  Swapping an adapter is a call with the base L1,
 * L2 and another A, B.
 *   L1, L2     bf16 [K][r], [r][N] (both NULL iff r == 0)
 *   lambda     fp32 [K], the smoothing factors (not their reciprocals)
 *   A, B       bf16 [K][ra], [ra][N]
 *   L1_out, L2_out  outputs, caller-allocated; must not overlap the inputs
 * r and ra multiples of 16 with r + ra <= 128, N a multiple of 16.
 */
svdq_status svdq_attach_lora(const void* L1, const void* L2, const float* lambda, const void* A,
                             const void* B, int64_t K, int64_t N, int64_t r, int64_t ra, void* L1_out,
                             void* L2_out, void* stream);

/*
 * Smoothing statistics (chattools.cn article 584, "technical principles":
 * lambda_k = sqrt(max_i |X_ik|) / sqrt(max_n |W_kn|) takes the largest
 * magnitude of each input channel over the calibration activations).
 * Folds one batch into a running per-channel maximum on the device:
 *     amax[k] = max(amax[k], max_i |X[i][k]|),   i < M.
 *   X     bf16 [M][K] row-major, device, 16-byte aligned; not modified
 *   amax  fp32 [K], device, 16-byte aligned, caller-owned; set it to zeros
 *         before the first batch and pass it unchanged to later ones
 * The result is exact (a maximum of bf16 magnitudes) and does not depend on
 * the order of rows or batches; a NaN in X makes its channel's value NaN.
 * Calls on one amax must be stream-ordered.  K a multiple of 8.
 * Errors: SVDQ_ERR_INVALID_ARG (null pointer, M or K <= 0),
 * SVDQ_ERR_UNSUPPORTED_SHAPE, SVDQ_ERR_MISALIGNED, SVDQ_ERR_CUDA.
 */
svdq_status svdq_channel_absmax(const void* X, int64_t M, int64_t K, float* amax, void* stream);

/*
 * Kernel choice of svdq_linear (host-side setting for the whole process):
 *   0  by shape (default): the small-M kernel (128 x 128 tiles with K split
 *      over a cluster and summed in distributed shared memory) for M <= 128
 *      when the large-M kernel's 256 x 256 tiles would cover fewer than a
 *      quarter of the SMs, else the large-M kernel (persistent CTA pairs,
 *      256 x 256 tiles over all of K);
 *   1  always the large-M kernel;   2  always the small-M kernel.
 * Both compute the same Y (the small-M kernel's fp32 sum runs in another
 * order).  Returns SVDQ_ERR_INVALID_ARG for any other value.
 */
svdq_status svdq_set_linear_path(int path);

/*
 * Launch overlap of the layer calls (host-side setting for the whole
 * process; 1 by default).  With 1, svdq_quantize_act(_gelu, _noalloc) and
 * svdq_linear(_scaled) launch their kernels with CUDA's programmatic
 * stream-serialisation attribute: a kernel may be scheduled while the
 * kernel ahead of it in the stream is finishing, sets up (barriers, tensor
 * memory; the linear kernels also prefetch their weight tiles into L2) and
 * waits on the device for that kernel to complete before it reads or writes
 * any buffer.  Stream order is therefore kept for every buffer, whatever
 * kernel precedes the call; only the set-up overlaps.  The layer kernels in
 * turn let the kernel behind them start its set-up early.  Inside a CUDA
 * graph captured from a stream the overlap becomes a programmatic edge.
 * With 0 the kernels launch plainly.  Results are identical either way.
 * Returns SVDQ_ERR_INVALID_ARG for values other than 0 and 1.
 */
svdq_status svdq_set_launch_overlap(int enable);

/*
 * Failure detection.  Every wait inside the kernels is bounded (default
 * 2 s, or SVDQ_WAIT_TIMEOUT_MS from the environment at first use); a wait
 * that expires records SVDQ_ERR_TIMEOUT in the current device's status word
 * and the kernel returns without hanging the GPU.
 *
 * svdq_sync_status synchronises `stream`, returns the recorded status of
 * the current device (SVDQ_OK if none; SVDQ_ERR_CUDA if the stream reports
 * an error) and clears it.  `where`, if not NULL, receives the id of the
 * wait that expired (0 if none).
 */
svdq_status svdq_sync_status(void* stream, int* where);

/* Sets the limit of every bounded wait in kernels launched from now on, in
 * nanoseconds (0 < timeout_ns <= 60 s), for all devices of the process.
 * Host-side setting only; returns SVDQ_ERR_INVALID_ARG outside that range. */
svdq_status svdq_set_wait_timeout(uint64_t timeout_ns);

/* Self test of the bounded wait: launches one CTA that waits on a barrier
 * nothing will complete, with the given limit in nanoseconds; the wait
 * expires and records SVDQ_ERR_TIMEOUT, read back with svdq_sync_status. */
svdq_status svdq_selftest_wait_timeout(uint64_t timeout_ns, void* stream);

/*
 * svdq_quantize_act without a workspace argument, for callers that can
 * neither allocate device memory nor hand the library scratch: for example a
 * plugin inside a host inference engine that owns all device memory and
 * gives its plugins no scratch, or serving code that may not allocate on its
 * request path (an allocation can synchronise the device or fail under
 * memory pressure).  The SVDQuant pages have no counterpart to this call; it
 * only changes where the activation step keeps its scratch.
 *
 * Same arguments and results as svdq_quantize_act, minus the workspace.
 * The scratch is a fixed 8 MiB array inside the library (every GPU that
 * loads the library holds it until the process exits), so:
 *  - shapes whose svdq_quantize_act_workspace() exceeds 8 MiB are refused
 *    with SVDQ_ERR_UNSUPPORTED_SHAPE (e.g. M = 4608 fits up to r = 64);
 *  - the first call on a device that needs scratch sets it up (looks up the
 *    array's device address and zero-fills it, synchronously), so make that
 *    first call before any stream capture;
 *  - all calls share the one array, and each leaves its counters at zero for
 *    the next: calls that may overlap on the GPU (other streams, other host
 *    threads) race with each other and must be serialised by the caller.
 * The call allocates no memory (no cudaMalloc, no cudaFree).
 */
svdq_status svdq_quantize_act_noalloc(const void* X, const float* inv_lambda, const void* L1,
                                      int64_t M, int64_t K, int64_t r, uint8_t* x_codes,
                                      uint8_t* x_scales, void* T, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SVDQ_H_ */
