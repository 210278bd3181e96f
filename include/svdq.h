/*
 * svdq.h -- C ABI of the SVDQuant W4A4 linear layer for NVIDIA B200 (sm_100a).
 *
 * The layer (SVDQuant technical review of arXiv:2411.05007v4, section 4.2,
 * eq. 7; section 6.1):
 *
 *     Y = Q(X~) Q(R) + (X~ L1) L2 + b,   X~ = X diag(lambda)^-1,
 *     R = diag(lambda) W - L1 L2                       (section 5, eq. 10)
 *
 * Math shapes: X is M x K (tokens x input channels), W is K x N.  Arrays
 * cross this ABI in row-major order; the weight is passed in nn.Linear
 * layout [N][K] (its transpose).
 *
 * Number formats (section 2.2, eq. 1; section 8 for group 64):
 *   - INT4 codes: symmetric, per group of 64 consecutive K, scale
 *     s = fl32(max|z| / 7), code = clamp(round_half_even(z / s), -8, 7)
 *     of the exact quotient; s = 0 and codes 0 for an all-zero group.
 *   - Packed codes: two's-complement nibbles, two per byte; byte b of a row
 *     holds k = 2b in the low nibble and k = 2b+1 in the high nibble.
 *   - Scales: fp32, group-major: s_x[g][m] (K/64 x M), s_w[g][n] (K/64 x N).
 *   - 16-bit branch: bf16 (uint16_t bit patterns) with fp32 accumulation.
 *
 * Conventions for every call:
 *   - Calls return svdq_status; nothing is thrown across the ABI.
 *   - Argument checks (null, shape, alignment) are synchronous and happen
 *     before any launch; a failed check launches nothing.
 *   - Device pointers must be 16-byte aligned, leading dimensions must keep
 *     every row 16-byte aligned, else SVDQ_ERR_ALIGNMENT.
 *   - K must be a multiple of 64, else SVDQ_ERR_SHAPE.  Any M >= 0, N >= 1.
 *   - Hot-path calls are asynchronous on `stream`; the caller owns every
 *     device buffer it passes.  A launch failure returns SVDQ_ERR_CUDA.
 *   - A device-side wait that exceeds its bound sets a sticky error word in
 *     the weights handle instead of hanging; read it with
 *     svdq_get_device_error.
 */
#ifndef SVDQ_H_
#define SVDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* cudaStream_t;   /* same type as CUDA's own */

typedef enum {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,     /* null pointer, bad enum, bad rank          */
  SVDQ_ERR_SHAPE = 2,           /* K % 64 != 0, negative sizes, ld too small */
  SVDQ_ERR_ALIGNMENT = 3,       /* device pointer or row not 16-byte aligned */
  SVDQ_ERR_UNSUPPORTED = 4,     /* group != 64, branch rank > 128 or % 8     */
  SVDQ_ERR_NUMERIC = 5,         /* non-finite weights or statistics          */
  SVDQ_ERR_CUDA = 6,            /* a CUDA runtime call or launch failed      */
  SVDQ_ERR_DEVICE_TIMEOUT = 7,  /* a bounded device wait expired             */
  SVDQ_ERR_OOM = 8,             /* device or host allocation failed          */
  SVDQ_ERR_IO = 9               /* file could not be read or written         */
} svdq_status;

enum { SVDQ_EPI_NONE = 0, SVDQ_EPI_GELU = 1 };

/* Number format of a packed handle: the W4A4 group format of every call
 * above, or the W8A8 comparator of svdq_pack_weights_w8a8. */
enum { SVDQ_FORMAT_W4A4 = 0, SVDQ_FORMAT_W8A8 = 1, SVDQ_FORMAT_NVFP4 = 2 };

#define SVDQ_GROUP 64
#define SVDQ_MAX_RANK 128
#define SVDQ_MAX_SPLITS 16      /* K splits per output tile in svdq_linear_splitk */

/* Opaque packed layer, immutable after svdq_pack_weights / svdq_weights_load.
 * Holds device copies of every operand plus host copies for export. */
typedef struct svdq_weights svdq_weights;

const char* svdq_status_string(int status);
int svdq_version(void);

/*
 * Calibration statistic of eq. 4 (section 3.1): absmax[k] = max(absmax[k],
 * max_i |X[i][k]|) over the M rows of a host bf16 matrix X [M][ldx].
 * Call it once per calibration batch on an array that starts at zero.
 * Host only; K need not be a multiple of 64 here.
 */
svdq_status svdq_calib_absmax(int M, int K, const uint16_t* X, int ldx,
                              float* absmax);

/*
 * Offline transform of one layer (review section 5, the offline procedure with a
 * fixed alpha and no refinement).  Host inputs, device result.
 *   lambda_k = act_absmax[k]^alpha / max_n|W[n][k]|^(1-alpha)   (eq. 4);
 *              lambda_k = 1 if either statistic is 0;
 *   W~ = diag(lambda) W (fp64)                                   (eq. 3);
 *   top-`rank` SVD of W~ in fp64: L1 = U S, L2 = V^T             (eq. 10),
 *   stored as bf16;  R = W~ - L1 L2 against the stored factors, quantised
 *   per group of 64 input channels of each output column       (eq. 1);
 *   optional LoRA (eq. 13): L1 <- [L1 | bf16(diag(lambda) A lora_scale)],
 *   L2 <- [L2 ; B]; R is not recomputed.
 * Arguments:
 *   K, N        input / output channels, K % 64 == 0;
 *   rank        SVD rank, 0 <= rank <= min(K, N); the branch rank
 *               rank + lora_rank must be a multiple of 8 and <= 128 (the
 *               low-rank operands move in 16-byte units), else
 *               SVDQ_ERR_UNSUPPORTED;
 *   group       must be 64;
 *   W           host bf16 [N][K];  act_absmax  host fp32 [K], finite, >= 0;
 *   alpha       migration strength in (0, 1) (0.5 in every workload);
 *   bias        host bf16 [N] or NULL (zero bias);
 *   lora_rank   0 or the adapter rank; lora_A host bf16 [K][lora_rank],
 *               lora_B host bf16 [lora_rank][N] (both required if > 0);
 *   stream      stream for the upload (the call synchronises it);
 *   out         receives the handle; *out is NULL on error.
 * The current CUDA device at the time of the call owns the handle.
 */
svdq_status svdq_pack_weights(int K, int N, int rank, int group,
                              const uint16_t* W, const float* act_absmax,
                              double alpha, const uint16_t* bias,
                              int lora_rank, const uint16_t* lora_A,
                              const uint16_t* lora_B, float lora_scale,
                              cudaStream_t stream, svdq_weights** out);

/*
 * Same transform as svdq_pack_weights, without touching a GPU: the handle
 * holds host copies only (export / save work; the hot-path calls reject it
 * with SVDQ_ERR_INVALID_ARG).  Lets a machine without a GPU pack a layer and
 * save it for svdq_weights_load elsewhere.
 */
svdq_status svdq_pack_weights_host(int K, int N, int rank, int group,
                                   const uint16_t* W, const float* act_absmax,
                                   double alpha, const uint16_t* bias,
                                   int lora_rank, const uint16_t* lora_A,
                                   const uint16_t* lora_B, float lora_scale,
                                   svdq_weights** out);

/*
 * Offline pack with the calibration refinement of the review's offline
 * procedure (section 5): for every candidate migration strength alphas[i]
 * (each in (0, 1)) the layer is smoothed, factored and its residual
 * quantised as in svdq_pack_weights; then `refine_iters` alternating steps
 * replace the factors by the rank-r SVD of W~ - deq(Q(R)) and recompute and
 * quantise R against W~.  Each candidate is scored by the calibrated
 * layer-output error on the tokens X_cal (host bf16 [M_cal][ldx]):
 *   err = ||Y_q - X W||_F / ||X W||_F   (fp64, both branches, no bias)
 * where Y_q is the quantised layer (activation statistics from X_cal).  The
 * candidate with the smallest error is packed (the first one on ties); LoRA
 * and bias join as in svdq_pack_weights.  errors (host, n_alpha doubles, may
 * be NULL) receives every candidate's error.  to_device != 0 uploads to the
 * current device (stream ordered); 0 gives a host-only handle.
 * gptq != 0 rounds every residual (the first and each refined one) with
 * GPTQ (review section 8: "residual weights use GPTQ"; the published
 * algorithm of Frantar et al.) instead of to nearest:
 *   H = X~^T X~ on the calibration tokens (x~ = fl32(x * inv_lambda)),
 *   dampened by 1 % of its mean diagonal (an unused channel gets H_kk = 1);
 *   U = upper Cholesky factor of H^-1; input channels in order: on entering
 *   a group of 64 each output column's scale comes from the updated group
 *   (eq. 1), then channel k is rounded (eq. 1 on fl32 of the updated value)
 *   and its error (w - q s) / U_kk is subtracted from every later channel j
 *   times U_kj.  The cost is O(K^3 + N K^2) host work per candidate.
 * Errors: as svdq_pack_weights; SVDQ_ERR_INVALID_ARG for missing or empty
 * calibration tokens, an alpha outside (0, 1) or a negative iteration count;
 * SVDQ_ERR_NUMERIC if the dampened Hessian is not positive definite.
 */
svdq_status svdq_pack_weights_calibrated(int K, int N, int rank, int group,
                                         const uint16_t* W, const uint16_t* X_cal,
                                         int M_cal, int ldx, int n_alpha,
                                         const double* alphas, int refine_iters, int gptq,
                                         const uint16_t* bias, int lora_rank,
                                         const uint16_t* lora_A, const uint16_t* lora_B,
                                         float lora_scale, int to_device,
                                         cudaStream_t stream, double* errors,
                                         svdq_weights** out);

/* Sizes of a handle; any output pointer may be NULL.  `rank` is the total
 * branch rank (svd_rank + lora_rank). */
svdq_status svdq_weights_info(const svdq_weights* w, int* K, int* N, int* rank,
                              int* svd_rank, int* lora_rank);

/*
 * Host copies of the packed operands (for checking against an oracle).  Any
 * output may be NULL.  inv_lambda fp32 [K] (= fl32(1/lambda)); wq uint8
 * [N][K/2] (weight codes, layout as above); s_w fp32 [K/64][N];
 * L1 bf16 [K][rank]; L2 bf16 [rank][N]; bias bf16 [N]; sigma fp64
 * [svd_rank + 1] (leading singular values of W~).
 */
svdq_status svdq_weights_export(const svdq_weights* w, float* inv_lambda,
                                uint8_t* wq, float* s_w, uint16_t* L1,
                                uint16_t* L2, uint16_t* bias, double* sigma);

/* Store / restore a packed layer (review section 5): versioned header and
 * raw host arrays.  load uploads to the current device on `stream`. */
svdq_status svdq_weights_save(const svdq_weights* w, const char* path);
svdq_status svdq_weights_load(const char* path, cudaStream_t stream,
                              svdq_weights** out);
void svdq_weights_free(svdq_weights* w);

/*
 * Fused activation pass (review section 6.1, activation side): one
 * kernel reads X once and writes
 *   xq  [M][K/2]   packed INT4 codes of x~ = fl32(x * inv_lambda_k);
 *   s_x [K/64][M]  fp32 scales, fl32(max|x~| / 7) per token and group;
 *   Z   [M][rank]  bf16 down-projection bf16(bf16(x~) L1), fp32 accumulation
 *                  (ignored, may be NULL, when rank == 0).
 * X is device bf16 [M][ldx], ldx >= K.  All device pointers, 16-byte
 * aligned.  M == 0 is a no-op.
 */
svdq_status svdq_quantize_act(const svdq_weights* w, int M, const uint16_t* X,
                              int ldx, uint8_t* xq, float* s_x, uint16_t* Z,
                              cudaStream_t stream);

/*
 * Fused W4A4 product (review section 6.1, product side): one kernel computes
 *   P_g = sum_{k in g} q_x q_w       (exact integer per group, formed on the
 *                                     tensor cores; |P_g| <= 4096)
 *   acc = sum_g s_x[g][m] s_w[g][n] P_g            (fp32)
 *   Y   = bf16(epi(acc + Z L2 + b))                 written once
 * with epi = identity or GELU (exact-erf form in fp32).  Y is device bf16
 * [M][ldy], ldy >= N.  xq, s_x, Z as produced by svdq_quantize_act.
 */
svdq_status svdq_linear(const svdq_weights* w, int M, const uint8_t* xq,
                        const float* s_x, const uint16_t* Z, uint16_t* Y,
                        int ldy, int epilogue, cudaStream_t stream);

/*
 * The whole layer with its input and output in host memory (review section
 * 6.1: the two fused kernels of the layer, here between a host-to-device
 * copy of X and a device-to-host copy of Y).  Enqueues on `stream`, in
 * order: the copy of X (host bf16 [M][ldx], ldx >= K) to the workspace,
 * svdq_quantize_act, svdq_linear with `epilogue`, and the copy of Y to host
 * bf16 [M][ldy], ldy >= N.  Returns once everything is enqueued; Y is valid
 * after the stream has been synchronised.  Pinned host memory
 * (cudaHostAlloc) lets the copies overlap other streams; pageable memory is
 * accepted, and its copies then block the host.
 * workspace: device memory, 16-byte aligned, at least
 *         svdq_linear_host_workspace(w, M) bytes, owned by the caller; it
 *         holds X, the codes, the scales, Z and Y on the device.  Calls
 *         sharing a workspace must not overlap (same stream, or ordered by
 *         events).
 * Errors: as svdq_quantize_act and svdq_linear (nothing more is enqueued
 * after the first failing step); SVDQ_ERR_INVALID_ARG for a null pointer,
 * SVDQ_ERR_SHAPE for ldx < K, ldy < N or a workspace that is too small,
 * SVDQ_ERR_CUDA if a copy cannot be enqueued.  M == 0 is a no-op.
 */
size_t svdq_linear_host_workspace(const svdq_weights* w, int M);
svdq_status svdq_linear_host(const svdq_weights* w, int M, const uint16_t* X, int ldx,
                             uint16_t* Y, int ldy, int epilogue, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream);

/*
 * Split-K form of svdq_linear for batches too small to fill the GPU with
 * output tiles (review section 9: PixArt-Sigma layers at a few hundred
 * tokens).  The K groups of every 128-row output tile are divided into
 * `splits` consecutive ranges, each handled by its own persistent-CTA work
 * item; a range's fp32 partial sum of s_x s_w P_g (split 0 also adds Z L2)
 * goes to the workspace, and the last range of a tile to finish sums the
 * partials in range order and applies bias, epilogue and the bf16 store.
 * Same operation as svdq_linear; only the fp32 summation order differs.
 *
 * splits: 1 .. min(SVDQ_MAX_SPLITS, K/64), or 0 for the automatic choice
 *         (one split once the output tiles alone cover half the SMs, else
 *         about one work item per SM with at least two groups per range).
 *         One split runs svdq_linear's kernel and gives its exact bits.
 * workspace: device memory, 256-byte aligned, at least
 *         svdq_linear_splitk_workspace(w, M, splits) bytes, owned by the
 *         caller.  Its first part holds arrival counters, which this call
 *         clears (cudaMemsetAsync on `stream`) before the launch; the rest
 *         holds the partial tiles.  Calls sharing a workspace must not
 *         overlap (same stream, or ordered by events).
 * Errors: as svdq_linear; SVDQ_ERR_INVALID_ARG for a bad split count or a
 * null workspace, SVDQ_ERR_ALIGNMENT for a misaligned one, SVDQ_ERR_SHAPE
 * if workspace_bytes is too small.
 */
size_t svdq_linear_splitk_workspace(const svdq_weights* w, int M, int splits);
svdq_status svdq_linear_splitk(const svdq_weights* w, int M, const uint8_t* xq,
                               const float* s_x, const uint16_t* Z, uint16_t* Y,
                               int ldy, int epilogue, int splits, void* workspace,
                               size_t workspace_bytes, cudaStream_t stream);

/*
 * svdq_linear_splitk without a workspace argument: the scratch (arrival
 * counters and fp32 partial tiles) is a fixed 16 MiB device array inside
 * the library, one per device, so the call allocates nothing (no
 * cudaMalloc, no allocating library).  The SVDQuant pages have no
 * counterpart; this exists for allocation-free callers.
 *
 * Same arguments as svdq_linear_splitk.  With an explicit `splits` the
 * result bits equal svdq_linear_splitk's at that split count, and requests
 * whose workspace (svdq_linear_splitk_workspace) exceeds 16 MiB are
 * rejected with SVDQ_ERR_SHAPE.  With splits = 0 the automatic split is
 * lowered, one step at a time, until its workspace fits in 16 MiB (down to
 * a single split, which needs no scratch); the result bits then equal
 * svdq_linear_splitk's at the split actually used.  The call clears the
 * counters before its launch.
 * The scratch is shared by every call on the device: calls that overlap
 * in time (different streams, or handles used concurrently) race and
 * corrupt each other's results, so order them.  The first call on each
 * device looks up the array's address (which can load the library's
 * device code): make it before any stream capture.
 * Errors: as svdq_linear_splitk; SVDQ_ERR_CUDA if the set-up fails.
 */
svdq_status svdq_linear_splitk_noalloc(const svdq_weights* w, int M, const uint8_t* xq,
                                       const float* s_x, const uint16_t* Z, uint16_t* Y,
                                       int ldy, int epilogue, int splits,
                                       cudaStream_t stream);

/*
 * Cross-layer fusion (review section 6.1: the epilogue required by the
 * surrounding model, here the next layer's activation side; Algorithm 2's
 * quantise step run on the producing kernel's output tile).  Computes the
 * layer of `w` exactly as svdq_linear does, but instead of storing Y it
 * applies the next layer's activation pass to the bf16 values Y would
 * hold, so that nothing of Y reaches device memory:
 *   h   = bf16(epi(acc + Z L2 + b))               (svdq_linear's Y, bit for bit)
 *   xq_next, s_x_next: the codes and scales svdq_quantize_act(w_next, h)
 *                      would write (bit-exact: same quantiser);
 *   Z_next [M][rank_next] bf16(bf16(x~) L1_next) with x~ = fl32(h inv_lambda_next),
 *          fp32 accumulation in an order that differs from svdq_quantize_act's
 *          (each output column tile's partial product, then their sum in
 *          column-tile order), so Z_next agrees with it to within fp32
 *          summation error before the bf16 rounding (a one-ulp bf16
 *          difference is possible).  The result is deterministic.
 * A 128 x 128 or 128 x 256 output tile holds whole 64-column groups of the
 * next layer's K, so its codes and scales are complete in the epilogue;
 * only Z_next needs the cross-tile sum.
 *
 * w_next: a W4A4 handle on the same device with K == w's N and rank <= 32.
 * xq_next [M][N/2] uint8, s_x_next [N/64][M] fp32, Z_next [M][rank_next]
 * bf16 (may be NULL when rank_next == 0), device, 16-byte aligned.
 * workspace: device memory owned by the caller, 16-byte aligned, of at
 * least svdq_linear_quantize_next_workspace(w, w_next, M) bytes (fp32
 * [column tiles of w][M][rank_next], the tiles' partial Z_next; 0 bytes and
 * NULL allowed when rank_next == 0).  Every byte the call reads it has
 * written first, so the workspace needs no initialisation; calls sharing
 * one must not overlap.  Launches: the layer kernel and one small kernel
 * that sums the partials and rounds them to bf16.  A device timeout is
 * reported on w's error word.
 * Errors: as svdq_linear; SVDQ_ERR_SHAPE when w_next's K differs from w's
 * N, its rank exceeds 32, or workspace_bytes is too small;
 * SVDQ_ERR_INVALID_ARG for a handle of another format or device, or a
 * missing output.
 */
size_t svdq_linear_quantize_next_workspace(const svdq_weights* w, const svdq_weights* w_next,
                                           int M);
svdq_status svdq_linear_quantize_next(const svdq_weights* w, const svdq_weights* w_next,
                                      int M, const uint8_t* xq, const float* s_x,
                                      const uint16_t* Z, int epilogue, uint8_t* xq_next,
                                      float* s_x_next, uint16_t* Z_next, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, then reads and clears the handle's sticky device
 * error word: SVDQ_OK, or SVDQ_ERR_DEVICE_TIMEOUT if a bounded wait in a
 * kernel of this handle expired since the last read.
 */
svdq_status svdq_get_device_error(const svdq_weights* w, cudaStream_t stream);

/*
 * Test hook, not on the measured path: runs svdq_linear's tensor-core main
 * loop over the output block [row0, row0+nrows) x [col0, col0+ncols) and
 * writes its int32 group partials instead of rescaling them:
 *   P[g][i][j] = sum_{k in group g} q_x[row0+i][k] q_w[col0+j][k]
 * P is device int32 [K/64][nrows][ncols].
 */
svdq_status svdq_debug_partials(const svdq_weights* w, int M, const uint8_t* xq,
                                int row0, int nrows, int col0, int ncols,
                                int32_t* P, cudaStream_t stream);

/*
 * Test hook for the bounded device waits; no counterpart on the pages.
 * Runs svdq_linear (no epilogue) with every device wait bounded by
 * limit_us microseconds (1 .. 2,000,000) instead of the usual 2 s, while the
 * TMA producer of the first CTA withholds its first stage of packed codes:
 * nothing is copied for that stage, so the warps that wait on it give up
 * after the bound, raise the handle's sticky error word and leave the
 * kernel (every wait in it is bounded; the issuing thread waits for its own
 * tensor-core operations before TMEM is freed).  The other CTAs finish
 * normally.  Y is left partly unwritten.  svdq_get_device_error then
 * returns SVDQ_ERR_DEVICE_TIMEOUT (and clears the word); the context and
 * the handle stay usable.  Arguments as svdq_linear; SVDQ_ERR_INVALID_ARG
 * for limit_us out of range.
 */
svdq_status svdq_debug_linear_stall(const svdq_weights* w, int M, const uint8_t* xq,
                                    const float* s_x, const uint16_t* Z, uint16_t* Y,
                                    int ldy, unsigned int limit_us, cudaStream_t stream);

/*
 * ------------------------------------------------------------------------
 * W8A8 comparator (review section 8: the eight-bit setting, rank 16 with
 * dynamic per-token activation and per-channel weight quantisation; its
 * INT8 rows in section 9.3).  The same two-branch layer with 8-bit
 * operands and one scale per token / output channel, so the integer
 * product accumulates over all of K and the scales are applied once:
 *
 *     Y = s_x[m] s_w[n] sum_k q_x[m][k] q_w[n][k] + Z L2 + b
 *
 * Number format: s = fl32(max|z| / 127) over the whole row (a token of x~,
 * or an output column of R over all K), code = clamp(round_half_even(z / s),
 * -128, 127) of the exact quotient (|code| <= 127 for a normal s); s = 0 and
 * codes 0 for an all-zero row.  Smoothing, the bf16 factors, the residual R
 * and the bias are those of svdq_pack_weights.
 * A W8A8 handle is rejected (SVDQ_ERR_INVALID_ARG) by the W4A4 calls, and a
 * W4A4 handle by the calls below; save/load and LoRA are W4A4 only.
 * ------------------------------------------------------------------------
 */

/* Offline pack of the comparator: as svdq_pack_weights (group 64 is not
 * used; K % 64 == 0 is still required), with R quantised per output channel
 * over all K.  to_device != 0 uploads to the current device on `stream`
 * (synchronised); 0 gives a host-only handle for export. */
svdq_status svdq_pack_weights_w8a8(int K, int N, int rank, const uint16_t* W,
                                   const float* act_absmax, double alpha,
                                   const uint16_t* bias, int to_device,
                                   cudaStream_t stream, svdq_weights** out);

/* Host copies of the comparator's residual: wq8 int8 [N][K], s_w8 fp32 [N]
 * (either may be NULL).  The other operands come from svdq_weights_export. */
svdq_status svdq_weights_export_w8a8(const svdq_weights* w, int8_t* wq8, float* s_w8);

/* Format of a handle (SVDQ_FORMAT_*), or -1 for NULL. */
int svdq_weights_format(const svdq_weights* w);

/*
 * Activation pass of the comparator: x~ = fl32(x * inv_lambda_k) as in
 * svdq_quantize_act; then
 *   xq  [M][K]    int8 codes of x~ with one scale per token;
 *   s_x [M]       fp32 scales fl32(max_k |x~| / 127);
 *   Z   [M][rank] bf16 down-projection bf16(bf16(x~) L1), fp32 accumulation.
 * One kernel: each block of tokens is read once from HBM to take its
 * absmax and Z, and a second time (from L2) to quantise.
 */
svdq_status svdq_quantize_act_w8a8(const svdq_weights* w, int M, const uint16_t* X,
                                   int ldx, int8_t* xq, float* s_x, uint16_t* Z,
                                   cudaStream_t stream);

/*
 * Product of the comparator: one tcgen05 kernel, int8 operands copied by
 * TMA straight into the tensor-core layout, the int32 sum over all of K in
 * TMEM, one fp32 scaling s_x[m] s_w[n] per output, then Z L2 (bf16 tensor
 * cores), bias, optional GELU and the bf16 store of Y [M][ldy], as in
 * svdq_linear.
 */
svdq_status svdq_linear_w8a8(const svdq_weights* w, int M, const int8_t* xq,
                             const float* s_x, const uint16_t* Z, uint16_t* Y,
                             int ldy, int epilogue, cudaStream_t stream);

/*
 * ------------------------------------------------------------------------
 * NVFP4 variant (review section 8: NVFP4 uses groups of 16 with FP8
 * scales; section 9.1 on the nonuniform FP4 grid).  The same two-branch
 * layer with FP4 E2M1 operands whose groups of 16 along K carry an FP8 E4M3
 * scale, applied by the tensor cores (block-scaled MMA), and an fp32 scale
 * per row (token of x~, output column of R):
 *
 *   s = fl32(max|row| / 2688)                      (2688 = 6 * 448)
 *   b = e4m3(fl32(max|group| / fl32(6 s)))         nearest-even, <= 448
 *   q = e2m1(z / (b s))                            nearest-even on
 *                                                  {0, .5, 1, 1.5, 2, 3, 4, 6}
 *   Y = s_x[m] s_w[n] sum_k (q_x b_x)(q_w b_w) + Z L2 + b
 *
 * Codes: two per byte, even k in the low nibble, bit 3 = sign.  Group
 * scales cross this ABI in the tensor-core atom layout: for rows
 * [128 a, 128 a + 128) and K block kb of 64, a 512-byte atom at
 * (a * K/64 + kb) * 512 holds row r's four scales at 16 (r % 32) + 4 (r / 32);
 * svdq_nvfp4_sf_bytes(rows, K) gives the size (rows padded to 128).
 * K % 64 == 0; save/load and LoRA are W4A4 only; the W4A4 and W8A8 calls
 * reject an NVFP4 handle and these calls reject the others.
 * ------------------------------------------------------------------------
 */

/* Offline pack (as svdq_pack_weights_w8a8, with R quantised by the NVFP4
 * rule per output column). */
svdq_status svdq_pack_weights_nvfp4(int K, int N, int rank, const uint16_t* W,
                                    const float* act_absmax, double alpha,
                                    const uint16_t* bias, int to_device,
                                    cudaStream_t stream, svdq_weights** out);

/* Host copies of the NVFP4 residual: codes [N][K/2], E4M3 group-scale bits
 * sf [N][K/16] (row-major, not the atom layout), row scales s_w [N]. */
svdq_status svdq_weights_export_nvfp4(const svdq_weights* w, uint8_t* codes, uint8_t* sf,
                                      float* s_w);

/* Bytes of a group-scale array in the atom layout (0 for invalid sizes). */
size_t svdq_nvfp4_sf_bytes(int rows, int K);

/*
 * Activation pass: x~ = fl32(x * inv_lambda_k); then
 *   xq  [M][K/2]  packed E2M1 codes;
 *   sfa           E4M3 group scales, atom layout, svdq_nvfp4_sf_bytes(M, K)
 *                 bytes (the rows past M are written as 0);
 *   s_x [M]       fp32 row scales;
 *   Z   [M][rank] bf16 down-projection bf16(bf16(x~) L1), fp32 accumulation.
 * One kernel, two sweeps of each token block as svdq_quantize_act_w8a8.
 */
svdq_status svdq_quantize_act_nvfp4(const svdq_weights* w, int M, const uint16_t* X,
                                    int ldx, uint8_t* xq, uint8_t* sfa, float* s_x,
                                    uint16_t* Z, cudaStream_t stream);

/*
 * Product: one tcgen05 kernel (kind::mxf4nvf4 block-scaled MMA, scales
 * staged into TMEM by tcgen05.cp) accumulating sum_k (q_x b_x)(q_w b_w)
 * in fp32, and the low-rank product Z L2 (bf16 tensor cores) in a second
 * TMEM buffer; the epilogue forms s_x s_w acc + Z L2 + b (optional GELU)
 * and stores bf16 Y [M][ldy].  Inputs as produced by
 * svdq_quantize_act_nvfp4.
 */
svdq_status svdq_linear_nvfp4(const svdq_weights* w, int M, const uint8_t* xq,
                              const uint8_t* sfa, const float* s_x, const uint16_t* Z,
                              uint16_t* Y, int ldy, int epilogue, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H_ */
