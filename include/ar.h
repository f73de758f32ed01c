/*
 * ar.h -- C ABI of libar, AutoRound per-layer SignSGD tuning on one B200.
 *
 * The method (sources cited by page title and section):
 *   "[llm-compressor] AutoRound: 부호 경사 하강법으로 라운딩 최적화"
 *     - "논문 핵심 내용": RTN w^ = s*round(w/s); offset rounding w^ = s*round(w/s + V)
 *       with V in [-0.5, 0.5]; loss |W^x - Wx|^2; SignSGD V <- V - lr*sign(dL/dV).
 *     - "on_event with SEQUENTIAL_EPOCH_END": the per-layer loop and
 *       _fake_quantize_with_offset, q = clamp(round(W/s + zp + V)), W' = s*(q - zp).
 *     - "AutoRoundModifier 생성자 파라미터": iters 200, lr 0.005, minmax_lr None -> lr,
 *       minmax_shrink 1.0.
 *   "Introducing AutoRound: Intel's Advanced Quantization for LLMs and VLMs",
 *     section 2: rounding and the clipping range are tuned jointly; section 4:
 *     iters = 0 is RTN.
 *   "[SGLang] AutoRound: 자동 라운딩 최적화 양자화", "1. AutoRoundConfig": bits in
 *     {2, 3, 4, 8}; pack_factor = 32 / bits.
 *
 * Conventions for every entry point:
 *   - All tensors are caller-owned DEVICE memory, row-major and contiguous,
 *     unless a parameter says otherwise.  The library allocates nothing; scratch
 *     memory comes from the caller as a workspace.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream).  Results are valid once the stream has
 *     been synchronised.
 *   - The return value reports argument errors (AR_EINVAL, AR_EUNSUPPORTED) and
 *     launch errors (AR_ECUDA).  On any non-AR_OK return nothing has been
 *     enqueued and no output has been written.  Errors detected on the device
 *     (a bounded wait that ran out) are recorded in the workspace and read with
 *     ar_tune_status().  Nothing aborts the process.
 *   - Test hooks, read from the environment on every call (no GPU fault is ever
 *     made; a test can set and clear them between calls):
 *       AR_FAULT=param   every argument check fails: AR_EINVAL, nothing enqueued.
 *       AR_FAULT=alloc   the tuning entry points fail as if their workspace (or,
 *                        for ar_tune_layer_host, its stream and events) could not
 *                        be had: AR_ENOMEM, nothing enqueued.
 *       AR_FAULT=launch  the first contraction launch of a tuning call fails:
 *                        AR_ECUDA; set-up work already enqueued on the workspace
 *                        stays, no output is written, the next call works.
 *       AR_FAULT=bounds  with AR_CHECKS, the step kernels are told that V and D hold
 *                        one element fewer than they do: their last store is
 *                        refused and reported (AR_ECHECK from ar_tune_status).
 *       AR_CHECKS=1      the tuning kernels check every store to V, V_best, D, the
 *                        clip factors, the Gram matrices, the residual and the
 *                        outputs against the buffer sizes; a store outside is
 *                        skipped and recorded in the workspace's status word
 *                        (ar_tune_status returns AR_ECHECK).  Never traps.
 *       AR_TAIL_SPLIT=0  the step contractions run every tile whole; by default
 *                        the tiles of a last partial wave that fills at most half
 *                        of the GPU's SM pairs run as two column halves each.  The
 *                        results are bit-identical either way (a schedule switch).
 *   - Shapes: W is [out, in]; a quantisation group is `group_size` consecutive
 *     elements of one row (-1: the whole row); G = in / group_size groups per row.
 *     Q = 2^bits - 1.  Codes are unsigned in [0, Q].
 *   - Arithmetic of the quantiser is IEEE fp32, one correctly rounded operation
 *     at a time, in this order (asymmetric):
 *       wmin = min(0, min W_grp), wmax = max(0, max W_grp)
 *       s  = (alpha*wmax - beta*wmin) / Q   (s = 1 for an all-zero group)
 *       zp = clamp(rint(-(beta*wmin) / s), 0, Q)
 *       q  = clamp(rint(W/s + V) + zp, 0, Q),  W' = s*(q - zp)
 *     symmetric: amax = max(-wmin, wmax), s = (2*(alpha*amax)) / Q, zp = 2^(bits-1).
 *     rint rounds half to even.  Same inputs give bit-identical codes, scales
 *     and zero-points on every call.
 */
#ifndef AR_H_
#define AR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  AR_OK = 0,
  AR_EINVAL = 1,        /* an argument is out of its documented range */
  AR_EUNSUPPORTED = 2,  /* valid for the method, not implemented by this library */
  AR_ENOMEM = 3,        /* the workspace is smaller than ar_tune_workspace_bytes() */
  AR_ECUDA = 4,         /* a CUDA call failed (no device, launch failure, ...) */
  AR_ETIMEOUT = 5,      /* a device-side bounded wait ran out (see ar_tune_status) */
  AR_ECHECK = 6         /* a device-side bounds check refused a store (AR_CHECKS) */
} ar_status;

typedef enum { AR_F32 = 0, AR_BF16 = 1 } ar_dtype;

/* How ar_tune_layer evaluates the two products of each step (same mathematics):
 *   AR_ALGO_DIRECT: R = X_b D^T (D = W' - W), then G = R^T X_b.  Per step
 *                   4*B*out*in flops (x2 with split operands).
 *   AR_ALGO_GRAM:   G = D H_b with H_b = X_b^T X_b, the calibration block's Gram
 *                   matrix, computed once per call for every block; the loss is
 *                   sum_k D_jk G_jk = sum_b R_bj^2.  Per step 2*out*in^2 flops (x3
 *                   with split operands), plus 2*n_rows*in^2 once, and
 *                   n_rows/B * in^2 * 4 bytes of workspace.
 *   AR_ALGO_AUTO:   the one with fewer flops over the whole call (GRAM only while
 *                   its matrices take at most 64 GiB). */
typedef enum { AR_ALGO_AUTO = 0, AR_ALGO_DIRECT = 1, AR_ALGO_GRAM = 2 } ar_algo;

/* Hyper-parameters of ar_tune_layer ("AutoRoundModifier" fields, plus the
 * readings this library makes where the pages are silent). */
typedef struct {
  int32_t bits;          /* 2, 3, 4 or 8 */
  int32_t group_size;    /* -1 (whole row) or a divisor of in; see ar_tune_layer */
  int32_t sym;           /* 0: asymmetric (alpha, beta); 1: symmetric (alpha only) */
  int32_t iters;         /* SignSGD steps, >= 0; 0 gives RTN */
  float lr;              /* step of V, >= 0 (0.005) */
  float minmax_lr;       /* step of alpha and beta; < 0 means "same as lr" */
  float minmax_shrink;   /* initial alpha = beta (1.0) */
  int32_t keep_best;     /* ar_keep_best: which state is applied (1: per row) */
  int64_t batch_rows;    /* rows of X per step; n_rows must be a multiple */
  uint64_t seed;         /* seeds the calibration-block schedule */
  int64_t start_step;    /* first step index (resume); 0 for a fresh run */
  int32_t algo;          /* ar_algo (0: auto) */
  int32_t split;         /* 1: tensor-core operands as exact bf16 pairs hi + lo
                            (hi = bf16(x), lo = bf16(x - hi): ~16 significant bits);
                            0: single bf16 (faster, the tuning trajectory drifts
                            further from an exact evaluation); 2: pairs, and the
                            Gram step sums K in chunks of 512 (each a fresh
                            tensor-core accumulation, added in fp32 round to
                            nearest): closer to an exact evaluation, slower; Gram
                            form with groups of at most 256 columns that divide
                            256, no full-precision target (else AR_EUNSUPPORTED) */
  int32_t init;          /* ar_init: how alpha and beta start (0: min-max) */
} ar_tune_params;

/* Initial clip factors ("[llm-compressor] AutoRound ...", "on_event with
 * SEQUENTIAL_EPOCH_END": _init_scale_zp is "Min-Max or MSE").
 *   AR_INIT_MINMAX: alpha = beta = minmax_shrink for every group.
 *   AR_INIT_MSE:    per group, the common ratio p = alpha = beta (symmetric: alpha)
 *                   on the grid fp32(100 - i) / fp32(100), i = 0 .. 50 (1.00 down to
 *                   0.50), whose round-to-nearest weights have the smallest squared
 *                   error sum_k (W'_k - W_k)^2.  The elements use ar_fake_quant's fp32
 *                   arithmetic; the sum runs in fp64 over the group's columns in
 *                   order; the first minimum along the grid wins.  minmax_shrink is
 *                   not used.  (The page names the option; this grid search is the
 *                   library's reading of it.) */
typedef enum { AR_INIT_MINMAX = 0, AR_INIT_MSE = 1 } ar_init;

/* Which state ar_tune_layer applies at the end ("[llm-compressor] AutoRound ...",
 * "on_event with SEQUENTIAL_EPOCH_END": the loop computes each step's loss,
 * total_loss, and applies the final V).  A step's batch loss is taken at the state
 * the step starts from; step 0's state (the min-max or MSE start) is a candidate.
 *   AR_KEEP_LAST:       the state after the last step (the page's listing).
 *   AR_KEEP_BEST_ROW:   per output row, the state of the step with that row's
 *                       lowest batch loss mean_b (Y' - Y)_bj^2 (fp32, strictly
 *                       lower; the default).  Rows stay independent.
 *   AR_KEEP_BEST_LAYER: for the whole layer, the state of the step whose layer
 *                       batch loss, the sum over rows of the row losses (taken in
 *                       fp64 in a fixed order), was strictly lowest; every row
 *                       takes that step.  ar_tune_state.best_loss then holds the
 *                       layer's best in every entry. */
typedef enum { AR_KEEP_LAST = 0, AR_KEEP_BEST_ROW = 1, AR_KEEP_BEST_LAYER = 2 } ar_keep_best;

/* Optional caller-owned tuning state (device memory, fp32).  Lets a caller
 * inspect the learned variables, and resume: a run of k steps followed by a run
 * with start_step = k and initialized = 1 equals one run of both. */
typedef struct {
  float* V;            /* [out, in]  rounding offsets, in [-0.5, 0.5] */
  float* alpha;        /* [out, G]   clip factor of the maximum, in [0.5, 1] */
  float* beta;         /* [out, G]   clip factor of the minimum, in [0.5, 1] */
  float* best_loss;    /* [out]      per row, lowest batch loss seen (+inf if none);
                          AR_KEEP_BEST_LAYER: the layer's lowest, in every entry */
  float* V_best;       /* [out, in]  per row, the state at that row's best step */
  float* alpha_best;   /* [out, G] */
  float* beta_best;    /* [out, G] */
  int32_t initialized; /* 0: the call initialises the state (V = 0, alpha = beta =
                          minmax_shrink, best_loss = +inf); 1: the call reads it */
} ar_tune_state;

/* Library version string, e.g. "ar 0.1.0 sm_100a". */
const char* ar_version(void);

/* Human-readable name of a status code. */
const char* ar_status_string(ar_status status);

/* Round-to-nearest quantisation (V = 0, alpha = beta = 1).
 * "[llm-compressor] AutoRound ...", "논문 핵심 내용": w^ = s*round(w/s), with the
 * min-max scale and zero-point above.
 *   W      [out, in], fp32 or bf16 (w_dtype), 16-byte aligned.
 *   codes  [out, in] uint8 out;  scale [out, G] fp32 out;  zp [out, G] int32 out.
 * out == 0 or in == 0 is a no-op.  AR_EINVAL: bits not in {2,3,4,8}, group_size
 * not -1 and not a positive divisor of in, a NULL pointer with out*in > 0. */
ar_status ar_rtn(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, int32_t bits,
                 int32_t group_size, int32_t sym, uint8_t* codes, float* scale,
                 int32_t* zp, void* stream);

/* Offset fake-quantisation with given V, alpha, beta ("_fake_quantize_with_offset").
 *   V [out, in], alpha [out, G], beta [out, G]: fp32 inputs (beta unused when sym).
 *   codes, scale, zp as for ar_rtn;  Wq [out, in] fp32 out = s*(q - zp), may be NULL.
 * Errors as for ar_rtn. */
ar_status ar_fake_quant(const void* W, ar_dtype w_dtype, int64_t out, int64_t in,
                        const float* V, const float* alpha, const float* beta,
                        int32_t bits, int32_t group_size, int32_t sym, uint8_t* codes,
                        float* scale, int32_t* zp, float* Wq, void* stream);

/* Pack b-bit codes into int32 words ("[SGLang] AutoRound ...", "1. AutoRoundConfig":
 * pack_factor = 32/bits, exact for 3 bits).  Each row is one little-endian bit
 * stream: bit j of code i is bit (i*bits + j) % 32 of word (i*bits + j) / 32.
 *   codes  [rows, cols] uint8, every value < 2^bits (higher bits are ignored).
 *   packed [rows, cols*bits/32] int32 out.
 * AR_EINVAL: bits not in {2,3,4,8}, cols*bits not a multiple of 32, NULL pointer.
 * rows == 0 or cols == 0 is a no-op. */
ar_status ar_pack(const uint8_t* codes, int64_t rows, int64_t cols, int32_t bits,
                  int32_t* packed, void* stream);

/* Bytes of workspace ar_tune_layer needs for these sizes and params (0 if they are
 * invalid).  X is read in place (never copied).  Dominated by the per-weight state
 * (about 12 bytes per element of W, 20 in the Gram form), the direct form's residual
 * (out*batch_rows*4 bytes) and, for AR_ALGO_GRAM, the Gram matrices
 * (n_rows/batch_rows * in^2 * 4 bytes). */
size_t ar_tune_workspace_bytes(int64_t out, int64_t in, int64_t n_rows,
                               const ar_tune_params* params);

/* Tune one linear layer with SignSGD and return its codes, scales and zero-points.
 * "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END".  Each step t:
 *   1. fake-quantise W with (V, alpha, beta) (as ar_fake_quant);
 *   2. R = X_b (W' - W)^T on the step's calibration block X_b of batch_rows rows,
 *      and the batch loss mean(R^2) (= mean((Y' - Y)^2), Y = X_b W^T; a bias cancels);
 *   3. G = R^T X_b (dL/dW' up to a positive factor), straight-through through
 *      every rint, masked where a clamp is active;
 *   4. V <- clamp(V - lr*sign(dL/dV), -0.5, 0.5); alpha, beta <- clamp(. - mlr*sign(.),
 *      0.5, 1) with mlr = minmax_lr (lr if < 0); all from gradients at the same point.
 * Step t uses block perm_e[t mod (n_rows/batch_rows)], perm_e a Fisher-Yates shuffle
 * per epoch driven by one SplitMix64 stream seeded with `seed`.  The contractions
 * run on bf16 tensor cores with fp32 accumulation.  With params->split = 1 (the
 * default) every operand that is not exactly bf16 (D = W' - W, R, the Gram
 * matrices) is held as an exact bf16 pair hi + lo (about 16 significant bits) and
 * multiplied as the products hi*hi + lo*hi + hi*lo; with split = 0 it is rounded to
 * one bf16.
 *   W           [out, in], fp32 or bf16, 16-byte aligned.
 *   X           [n_rows, in] bf16 (uint16 bit patterns), 16-byte aligned.
 *   params      host pointer, see ar_tune_params.
 *   state       host pointer to device buffers, or NULL (state kept in the workspace).
 *   workspace   device scratch of at least ar_tune_workspace_bytes(), 256-byte
 *               aligned; its first 4 bytes hold the device status (ar_tune_status).
 *   codes/scale/zp  outputs as for ar_rtn, from the applied state (keep_best).
 *   loss_trace  [iters] fp32 out (batch loss of each step), may be NULL.
 *   final_mse   1 double out: mean((X W'^T - X W^T)^2) over all n_rows rows with
 *               the applied W', may be NULL (skips one pass over X).
 * Supported shapes: in a multiple of 32; batch_rows a multiple of 8; group size
 * (group_size, or in for -1) a multiple of 16 (else AR_EUNSUPPORTED).  Groups that
 * divide 256 (or a whole row of at most 256) are updated inside the step kernel;
 * any other (a whole row of a wider layer, or sizes such as 96 or 384) through
 * per-segment partials and one small kernel per step.  out == 0 or in == 0 is a
 * no-op.
 * AR_EINVAL: bad bits/group_size, iters < 0, lr < 0, batch_rows <= 0 or not a
 * divisor of n_rows, NULL or misaligned pointers.  AR_ENOMEM: ws_bytes too small.
 * Calls sharing a workspace or state must not overlap on the device. */
ar_status ar_tune_layer(const void* W, ar_dtype w_dtype, int64_t out, int64_t in,
                        const uint16_t* X, int64_t n_rows, const ar_tune_params* params,
                        ar_tune_state* state, void* workspace, size_t ws_bytes,
                        uint8_t* codes, float* scale, int32_t* zp, float* loss_trace,
                        double* final_mse, void* stream);

/* Per-call kernel timing of ar_tune_layer_timed (host struct, filled on return). */
typedef struct {
  float residual_ms;         /* DIRECT: summed device time of the R = X_b (W' - W)^T
                                contractions; GRAM: 0 */
  float update_ms;           /* summed device time of the G contractions + updates (with
                                groups wider than 256 or not dividing it, each step's
                                group-finish kernel too) */
  float total_ms;            /* device time of the whole call */
  int32_t gemm_launches;     /* launches of each timed contraction (= iters) */
  int32_t kernel_launches;   /* every kernel this call launched */
  int32_t algo;              /* the ar_algo the call ran (DIRECT or GRAM) */
  float setup_ms;            /* device time before the first step (group statistics, and the
                                first block's Gram matrix; later blocks are
                                prepared just before their first step) */
} ar_tune_timing;

/* ar_tune_layer, with CUDA events recorded on `stream` around each contraction;
 * synchronises `stream` before returning and fills *timing.  Same arguments,
 * results and errors as ar_tune_layer; timing must not be NULL. */
ar_status ar_tune_layer_timed(const void* W, ar_dtype w_dtype, int64_t out, int64_t in,
                              const uint16_t* X, int64_t n_rows, const ar_tune_params* params,
                              ar_tune_state* state, void* workspace, size_t ws_bytes,
                              uint8_t* codes, float* scale, int32_t* zp, float* loss_trace,
                              double* final_mse, void* stream, ar_tune_timing* timing);

/* Workspace of ar_tune_layer_fp_target, in bytes (0 if the arguments are invalid, or if
 * they ask for the Gram form and its workspace would exceed 64 GiB).  On top of
 * ar_tune_workspace_bytes' layout of the same form:
 *   Gram form: two copies of one calibration block as a bf16 pair (4 * batch_rows * in
 *     * 2 bytes), the in x in pair M_b^T, every block's out x in pair C_b
 *     (n_rows/batch_rows * out * in * 4 bytes), their fp32 sum, and W as a pair when
 *     it is fp32;
 *   direct form: one block's dX as a pair (batch_rows * in * 4 bytes), E^T = W dX^T
 *     for every block as an out x n_rows pair (out * n_rows * 4 bytes), and W as a
 *     pair when it is fp32.
 * AR_ALGO_AUTO takes the Gram form while its workspace stays within 64 GiB, the direct
 * form otherwise. */
size_t ar_tune_fp_target_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, ar_dtype w_dtype,
                                         const ar_tune_params* params);

/* ar_tune_layer in the quant-aware mode with a full-precision target
 * ("[llm-compressor] AutoRound ...", "enable_quanted_input 모드" and the
 * "AutoRoundModifier" field enable_quanted_input: each layer is fed the output of
 * the already-quantised layers before it, while the loss compares against the
 * captured full-precision output).
 *   X          [n_rows, in] bf16: the layer's input on the quantised path.
 *   X_target   [n_rows, in] bf16: the input of the full-precision target, Y = X_target W^T.
 * The batch residual is R = X_b W'^T - X_target,b W^T = X_b D^T + dX_b W^T with
 * D = W' - W and dX = X - X_target, so with H_b = X_b^T X_b:
 *   gradient  G = D H_b + W M_b,   M_b = dX_b^T X_b            (in x in)
 *   row loss  L_j = d_j H_b d_j^T + 2 d_j (W M_b)_j^T + |dX_b w_j^T|^2.
 * Gram form: per calibration block (before its first step) the library forms dX_b as
 * a bf16 pair and computes M_b, C_b = W M_b and e_b = |dX_b w_j^T|^2 on the tensor
 * cores; the step kernel adds C_b to G and the two loss terms to the row loss.
 * Direct form: per block it computes E_b^T = W dX_b^T (a bf16 pair), which the
 * residual's epilogue adds to X_b D^T, so R and everything after it are the plain
 * loop's.  final_mse = mean((X W'^T - X_target W^T)^2) over all rows.  Either form
 * (params->algo; see ar_tune_fp_target_workspace_bytes for the automatic choice); an
 * explicit AR_ALGO_GRAM whose workspace would exceed 64 GiB gives AR_EUNSUPPORTED
 * (an 8192 x 29568 layer with 262144 calibration rows in blocks of 16384 would need
 * about 80 GB there, about 14 GB in the direct form).  X_target NULL: AR_EINVAL.  Otherwise arguments, results and
 * errors as ar_tune_layer, with workspace of ar_tune_fp_target_workspace_bytes(). */
ar_status ar_tune_layer_fp_target(const void* W, ar_dtype w_dtype, int64_t out, int64_t in,
                                  const uint16_t* X, const uint16_t* X_target, int64_t n_rows,
                                  const ar_tune_params* params, ar_tune_state* state, void* workspace,
                                  size_t ws_bytes, uint8_t* codes, float* scale, int32_t* zp,
                                  float* loss_trace, double* final_mse, void* stream);

/* Device workspace of ar_tune_layer_host, in bytes (0 if the arguments are invalid):
 * ar_tune_workspace_bytes() plus device copies of W, X and the outputs. */
size_t ar_tune_host_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, ar_dtype w_dtype,
                                    const ar_tune_params* params);

/* ar_tune_layer from host buffers to host buffers: the end-to-end call.
 * Same method, sources, results and errors as ar_tune_layer.  The differences:
 *   W_host, X_host      host pointers (layouts as for ar_tune_layer); page-locked
 *                       memory lets the copies overlap the work, pageable memory
 *                       works but copies synchronously.
 *   codes_host, scale_host, zp_host, loss_trace_host (may be NULL),
 *   final_mse_host (may be NULL)   host outputs, written when the call returns.
 *   workspace           device scratch of at least ar_tune_host_workspace_bytes(),
 *                       256-byte aligned; owned by the caller.
 * X goes to the device one calibration block at a time, on a stream of the call's
 * own, in the order in which the block schedule first needs the blocks.  Each
 * block's first kernel waits only for that block's copy, so the copy overlaps the
 * Gram matrices and the first epoch's steps.  The call starts after the work
 * already queued on `stream` and synchronises `stream` before it returns.  Device
 * errors (AR_ETIMEOUT) are reported directly, as ar_tune_status would.  Tuning
 * state is always fresh (no ar_tune_state).  Creates and destroys one stream and
 * n_rows/batch_rows + 3 events per call; allocates no device memory. */
ar_status ar_tune_layer_host(const void* W_host, ar_dtype w_dtype, int64_t out, int64_t in,
                             const uint16_t* X_host, int64_t n_rows, const ar_tune_params* params,
                             void* workspace, size_t ws_bytes, uint8_t* codes_host, float* scale_host,
                             int32_t* zp_host, float* loss_trace_host, double* final_mse_host,
                             void* stream);

/* The calibration-block schedule ar_tune_layer follows (host only, no GPU):
 * blocks[i] = block index of step first + i, i < count, for n_blocks blocks.
 * Each epoch is a Durstenfeld shuffle of 0..n_blocks-1 (for i = n_blocks-1 down
 * to 1, swap i with x mod (i+1)), x the successive outputs of one SplitMix64
 * stream (Steele, Lea & Flood 2014) seeded with `seed`, continued across
 * epochs; one block draws nothing.  AR_EINVAL if n_blocks < 1, first < 0,
 * count < 0 or blocks is NULL with count > 0. */
ar_status ar_block_schedule(int64_t n_blocks, int64_t first, int64_t count, uint64_t seed,
                            int64_t* blocks);

/* ---------------------------------------------------------------------------
 * Layer chain ("[llm-compressor] AutoRound ...", "enable_quanted_input 모드": with
 * quant-aware calibration each layer is tuned on the output of the already
 * quantised layers before it; the per-layer loop ends by replacing the layer's
 * weight with the fake-quantised W' = s*(q - zp) -- "최종 양자화 적용").
 * ------------------------------------------------------------------------- */

/* W' = s*(q - zp) per element (one fp32 operation after the exact q - zp).
 *   codes [out, in] uint8, scale/zp [out, G] (G = in / group_size; -1: whole row).
 *   Wq_hi [out, in] bf16 bits out: bf16(W'); Wq_lo [out, in] bf16 bits out (may be
 *   NULL): bf16(W' - bf16(W')), so hi + lo carries ~16 significant bits;
 *   Wq [out, in] fp32 out (may be NULL).
 * AR_EINVAL: bad group_size, NULL codes/scale/zp/Wq_hi.  out == 0 or in == 0: no-op. */
ar_status ar_dequant(const uint8_t* codes, const float* scale, const int32_t* zp, int64_t out,
                     int64_t in, int32_t group_size, uint16_t* Wq_hi, uint16_t* Wq_lo,
                     float* Wq, void* stream);

/* Y = bf16(X (Wq_hi + Wq_lo)^T + add): the linear layer with the quantised weight,
 * on the tensor cores (fp32 accumulation), rounded once to bf16.
 *   X [n, in] bf16 bits, Wq_hi/Wq_lo [out, in] bf16 bits (Wq_lo may be NULL),
 *   add [n, out] bf16 bits or NULL (a residual added in fp32 before rounding),
 *   Y [n, out] bf16 bits out.  All 16-byte aligned; in and out multiples of 8.
 *   status: device int32 or NULL; a bounded wait in the kernel that runs out sets
 *   it to AR_ETIMEOUT (Y is then invalid).  The caller zeroes it beforehand.
 * AR_EINVAL: NULL or misaligned pointers, in or out not a multiple of 8.  n == 0: no-op. */
ar_status ar_linear(const uint16_t* X, int64_t n, int64_t in, const uint16_t* Wq_hi,
                    const uint16_t* Wq_lo, int64_t out, const uint16_t* add, uint16_t* Y,
                    int32_t* status, void* stream);

/* y = bf16(silu(a) * b), silu(a) = a / (1 + exp(-a)), in fp32 (the gated MLP input
 * of a LLaMA-style down projection).  a, b, y: count bf16 bits. */
ar_status ar_silu_mul(const uint16_t* a, const uint16_t* b, int64_t count, uint16_t* y, void* stream);

/* Size of the fixed device scratch array used by ar_tune_layer_static (64 MiB). */
#define AR_STATIC_SCRATCH_BYTES (64ull << 20)

/* AR_STATIC_SCRATCH_BYTES as the library was built with it (for bindings that do
 * not read this header).  No GPU needed. */
size_t ar_static_scratch_bytes(void);

/* ar_tune_layer for callers that cannot allocate device memory at call time --
 * code that runs where cudaMalloc is not allowed or not wanted (inside a region
 * whose memory is owned by another allocator, or a path that must not trigger the
 * device synchronisation an allocation can cause).  The pages have no counterpart
 * of this entry point; it is a property of this library.
 * Same arguments, results and errors as ar_tune_layer with state = NULL, minus the
 * workspace: the scratch is one array of AR_STATIC_SCRATCH_BYTES in device memory,
 * created when the library's device code is loaded on a GPU and held by every GPU
 * that loads the library until the process exits.  The call makes no device
 * allocation (no cudaMalloc/cudaFree or other allocator); its host side uses the
 * C++ heap only for the step schedule.
 *   AR_ENOMEM: the layer needs more scratch than AR_STATIC_SCRATCH_BYTES
 *              (ar_tune_workspace_bytes() tells how much it needs); nothing is enqueued.
 * The first call on each device looks up the array's device address (with that
 * device current) and caches it with the id of the current CUDA context; a later
 * call that finds another context current (after cudaDeviceReset, say) looks it
 * up again.  With CUDA's lazy module loading (the default) that first call may
 * also be what loads the library's device code onto the device, and so what
 * creates the array: make the first call on each device before any stream
 * capture and outside any stretch of code that must not allocate.
 * All calls share the one array, and it keeps the last call's contents; every call
 * initialises what it reads.  Calls that overlap on the device (other streams,
 * other threads) race on the array: serialise them.  ar_tune_status() is not
 * available for this entry point (the status word is in the shared array). */
ar_status ar_tune_layer_static(const void* W, ar_dtype w_dtype, int64_t out, int64_t in,
                               const uint16_t* X, int64_t n_rows, const ar_tune_params* params,
                               uint8_t* codes, float* scale, int32_t* zp, float* loss_trace,
                               double* final_mse, void* stream);

/* Device status of the last ar_tune_layer call that used `workspace`: synchronises
 * `stream`, then returns AR_OK, or AR_ETIMEOUT if a kernel's bounded wait ran out
 * (its results are then invalid), AR_ECHECK if a bounds check of the AR_CHECKS
 * mode refused a store (results invalid), or AR_ECUDA if the stream reports an
 * error.  (The tuning library's replacement for a global last-error query: the
 * status lives in the call's own workspace, so concurrent calls on different
 * workspaces never see each other's errors.) */
ar_status ar_tune_status(const void* workspace, void* stream);

/* Per-row batch losses of the last ar_tune_layer (or ar_tune_layer_timed) call that
 * used `workspace`, called with the same out, in, n_rows and params: the loss the
 * keep-best choice compares ("[llm-compressor] AutoRound ...", "on_event with
 * SEQUENTIAL_EPOCH_END": the step loss total_loss, split by output row).
 *   row_loss  [iters, out] fp32 out, device or host memory (copied with unified
 *             addressing): row_loss[t*out + j] = sum over the rows b of step t's
 *             calibration block of R_bj^2, R = X_b (W' - W)^T at the state before
 *             step t's update.  Divide by batch_rows for the row's batch MSE.
 * Asynchronous on `stream`, after the tuning call it reads.  iters == 0, out == 0 or
 * in == 0: nothing to copy.  AR_EINVAL as ar_tune_layer, or a NULL pointer;
 * AR_ENOMEM: ws_bytes smaller than ar_tune_workspace_bytes() for these arguments.
 * The losses sit at the same place in a workspace of ar_tune_layer_fp_target, so
 * this call reads those too when params->algo names the form (AR_ALGO_GRAM or
 * AR_ALGO_DIRECT; with AR_ALGO_AUTO the two entry points may choose differently).
 * (Workspaces of ar_tune_layer_host and ar_tune_layer_static are not read by this
 * call.) */
ar_status ar_tune_row_losses(const void* workspace, size_t ws_bytes, int64_t out, int64_t in, int64_t n_rows,
                             const ar_tune_params* params, float* row_loss, void* stream);

/* Test hook for the bounded-wait path: one CTA waits on a barrier that nothing
 * arrives on, gives up after timeout_ns nanoseconds, writes AR_ETIMEOUT into
 * status[0] (device int) and exits cleanly.  Returns AR_OK once launched. */
ar_status ar_selftest_timeout(int32_t* status, uint64_t timeout_ns, void* stream);

/* Test hook for the quantiser's division.  The fake-quantiser forms u = W/s as the
 * correctly rounded fp32 quotient.  When every weight of a layer is zero or lies
 * in 2^-100 <= |w| <= 2^20, it gets the quotient from the group's correctly
 * rounded reciprocal y = 1/s with one fma residual correction (q = RN(W y),
 * r = s q - W exactly, u = RN(q - r y); P. Markstein, IBM J. Res. Dev. 34(1), 1990),
 * instead of a full IEEE division.  This hook evaluates both forms for every pair
 * (a[i], b[j]), i < na, j < nb (device fp32 arrays).  It skips the pairs outside
 * the fast form's domain: a outside that weight range, b not a positive normal
 * number at most 2^21 (the scales are positive), or a nonzero a/b that is not a
 * normal number below 2^64.  It adds the number of pairs whose results differ in
 * any bit to *mismatches (device uint64), and first_bad[0..1] (device) receive the
 * first such pair.  Returns AR_OK once launched. */
ar_status ar_selftest_division(const float* a, int64_t na, const float* b, int64_t nb, uint64_t* mismatches,
                               float* first_bad, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* AR_H_ */
