// Internal launch interfaces shared by the libar translation units.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace ar {

// One warp per quantisation group: statistics, scale/zero-point, per-element
// fake-quantisation.  Null pointers switch the corresponding input or output off.
struct GroupQuantArgs {
  const void* W = nullptr;  // [out, in] fp32 or bf16
  int w_bf16 = 0;
  int64_t out = 0, in = 0;
  int g = 0, G = 0, bits = 4, sym = 0;
  const float* wmin_in = nullptr;  // [out, G]; null: computed from W
  const float* wmax_in = nullptr;
  float* wmin_out = nullptr;       // [out, G] statistics out
  float* wmax_out = nullptr;
  const float* V = nullptr;        // [out, in]; null: 0
  const float* alpha = nullptr;    // [out, G]; null: 1
  const float* beta = nullptr;
  uint8_t* codes = nullptr;        // [out, in]
  float* scale = nullptr;          // [out, G]
  int32_t* zp = nullptr;           // [out, G]
  float* Wq = nullptr;             // [out, in] fp32 s*(q - zp)
  __nv_bfloat16* D_hi = nullptr;   // [out, in] D = s*(q - zp) - W as hi = bf16(D) ...
  __nv_bfloat16* D_lo = nullptr;   // ... and lo = bf16(D - hi) (may be null)
  int* div_slow = nullptr;         // when set: +1 for every group that has a weight
                                   // that is not div_fast_ok (W/s must use __fdiv_rn)
  // AR_CHECKS: capacities (elements) of the [out, in] and [out, G] outputs; a store
  // outside them is skipped and recorded in *status.  0: no checks.
  int64_t chk_elems = 0, chk_groups = 0;
  int* status = nullptr;
};

cudaError_t launch_group_quant(const GroupQuantArgs& a, cudaStream_t stream);
cudaError_t launch_pack(const uint8_t* codes, int64_t rows, int64_t cols, int bits, int32_t* packed,
                        cudaStream_t stream);
cudaError_t launch_fill_f32(float* p, int64_t n, float value, cudaStream_t stream);
// AR_INIT_MSE: per group, the clip ratio of the grid 1.00 .. 0.50 with the smallest
// round-to-nearest squared error, written to alpha and beta [out, in/g].
cudaError_t launch_mse_init(const void* W, int w_bf16, int64_t out, int64_t in, int g, int bits, bool sym,
                            float* alpha, float* beta, cudaStream_t stream);
// loss_trace[t] = sum_j rowloss[t*out + j] / (batch_rows * out), t < iters (fixed order).
cudaError_t launch_loss_trace(const float* rowloss, int64_t out, int iters, int64_t batch_rows,
                              float* loss_trace, cudaStream_t stream);
// final_mse[0] = sum of parts[0 .. count) / denom in fp64 (fixed order).
cudaError_t launch_sum_to_double(const float* parts, int64_t count, double denom, double* result,
                                 cudaStream_t stream);
cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t stream);
cudaError_t launch_division_selftest(const float* a, int64_t na, const float* b, int64_t nb,
                                     unsigned long long* bad, float* first, cudaStream_t stream);

// Keep-best check of the last step of a Gram-form run (its loss is complete only
// after the step's launch): per row j, L = sum of part[j, 0 .. nparts) in order,
// rowloss[j] = L; if keep_best and L/B < best_in[j], snapshot the state rows.
struct FinalizeBestArgs {
  const float* part = nullptr;
  int nparts = 0;
  int64_t out = 0, in = 0;
  int G = 0;
  float inv_batch = 1.f;
  int keep_best = 1;
  const float* best_in = nullptr;
  float* best_out = nullptr;
  float* rowloss = nullptr;
  const float* V_last = nullptr;
  const float* alpha_last = nullptr;
  const float* beta_last = nullptr;
  float* V_best = nullptr;
  float* alpha_best = nullptr;
  float* beta_best = nullptr;
};
cudaError_t launch_finalize_best(const FinalizeBestArgs& a, cudaStream_t stream);

// Hs = sum over nb blocks of (H_hi[b] + H_lo[b]) in fp32, returned as a bf16 pair,
// and dsum[k] = sum over blocks of diag[b*in + k] (the exact diagonals).
cudaError_t launch_gram_sum(const __nv_bfloat16* H_hi, const __nv_bfloat16* H_lo, int nb, int64_t count,
                            __nv_bfloat16* Hs_hi, __nv_bfloat16* Hs_lo, cudaStream_t stream);
cudaError_t launch_dequant(const uint8_t* codes, const float* scale, const int32_t* zp, int64_t out, int64_t in,
                           int g, __nv_bfloat16* Wq_hi, __nv_bfloat16* Wq_lo, float* Wq, cudaStream_t stream);
cudaError_t launch_silu_mul(const __nv_bfloat16* a, const __nv_bfloat16* b, int64_t count, __nv_bfloat16* y,
                            cudaStream_t stream);
// Full-precision-target mode: dX = X - X_target as a bf16 pair; an fp32 array as
// a bf16 pair; acc += hi + lo; per-row sums of partials (dst) added into total.
cudaError_t launch_diff_pair(const uint16_t* X, const uint16_t* Xt, int64_t n, __nv_bfloat16* hi,
                             __nv_bfloat16* lo, cudaStream_t stream);
cudaError_t launch_split_pair(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                              cudaStream_t stream);
cudaError_t launch_accum_pair(const __nv_bfloat16* hi, const __nv_bfloat16* lo, int64_t n, float* acc,
                              cudaStream_t stream);
cudaError_t launch_row_sum(const float* part, int nparts, int64_t rows, float* dst, float* total,
                           cudaStream_t stream);
cudaError_t launch_diag_sum(const float* diag, int nb, int64_t in, float* dsum, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Persistent tcgen05 GEMM: C[M, N] = sum over K segments of A_s[M, K] B_s[N, K]^T,
// operands bf16 K-major loaded by TMA, fp32 accumulators in tensor memory, fused
// epilogues (see gemm_sm100.cu).
// ---------------------------------------------------------------------------

enum EpiKind : int {
  kEpiStore = 0,   // C as a bf16 (hi, lo) pair; optional per-(row, n-tile) sums of C^2
  kEpiSumSq = 1,   // per-(row, n-tile) sums of C^2
  kEpiUpdate = 2,  // C = G: the SignSGD step (sign updates, keep-best, next D, Gram-form loss)
  kEpiDotD = 3,    // per-(row, n-tile) sums of D * C
  kEpiUpdateFp = 4, // kEpiUpdate with the full-precision-target terms (Cc_hi, e_row)
  // Groups wider than a thread's columns (group_size not dividing 256): the
  // per-element part of the step (G, loss, V, V snapshot) and per-(row, group,
  // 128-column segment) partials of d alpha, d beta into GemmArgs::gpart; the
  // group's update and the next D follow in launch_group_finish.
  kEpiUpdateWide = 5,
  kEpiUpdateFpWide = 6,
  // kEpiUpdate on K summed in chunks of GemmArgs::k_chunk K blocks: each chunk a fresh
  // tensor-core accumulation, added in fp32 (round to nearest) to the tile's running
  // sum by the epilogue before the step runs on the sum (ar_tune_params.split = 2).
  kEpiUpdateExact = 7
};

// Columns per thread in the update epilogue (one column half of a 256-wide tile):
// the segment width of the wide-group partials.
constexpr int kSegCols = 128;

// Operand maps: segment s reads A from a{seg_a[s]} and B from b{seg_b[s]}.
struct GemmMaps {
  CUtensorMap a0, a1, b0, b1;
};

struct GemmArgs {
  int M = 0, N = 0, K = 0;  // K: per segment
  int num_m_blk = 0, num_n_blk = 0, num_k_blk = 0, num_tiles = 0;
  int num_seg = 1;
  int seg_a[3] = {0, 0, 0};
  int seg_b[3] = {0, 0, 0};
  // MN-major operands: the map covers a row-major [K, M] (A) or [K, N] (B) tensor
  // (activations read without a transpose), built with 64-row boxes; loaded in
  // 64 x 64 boxes.  Otherwise the map covers [M or N, K] (K-major).
  int a_mn = 0, b_mn = 0;
  int a_k_off = 0;    // added to A's K coordinate
  int b_row_off = 0;  // added to B's row coordinate
  int b_k_off = 0;    // added to B's K coordinate
  uint64_t timeout_ns = 1000000000ull;
  int* status = nullptr;

  // kEpiStore: C rows j go to row c_row_off + j of [*, ldc]
  __nv_bfloat16* C_hi = nullptr;
  __nv_bfloat16* C_lo = nullptr;  // may be null
  // kEpiStore / kEpiSumSq: when set, hi (+ lo) of [*, ldc_add] (0: ldc) are added to C
  // in fp32 before its row sums and its store (a residual, or the full-precision
  // target's term of the direct form's residual)
  const __nv_bfloat16* C_add = nullptr;
  const __nv_bfloat16* C_add_lo = nullptr;
  int64_t ldc_add = 0;
  int64_t ldc = 0;
  // kEpiStore of a symmetric C (M == N, A == B): only tiles that reach the upper
  // triangle run (num_tiles counts them); each writes its upper elements in place and
  // its strictly upper ones again transposed, so every element is written once.
  int symmetric = 0;
  // 2-SM pair tiles (tcgen05 cta_group::2, clusters of two CTAs): 256 x 256 tiles,
  // num_m_blk counts 256-row blocks, B maps use 128-row boxes.
  int pair = 0;
  // Pair tiles only: one stage per K block holds every operand tile the segments
  // use (each loaded once) and the MMA warp issues all segments from it.
  int fused = 0;
  // Tile order: 0 = m fastest over all rows; g > 0 = groups of g m-blocks, m fastest
  // inside a group, the group's n-blocks in turn (keeps a wave's operands compact).
  int raster_m = 0;
  int64_t c_row_off = 0;
  // Step kinds on pair tiles: tail_split asks that the tiles of a last partial wave
  // of at most half the clusters each run as two column-half units; launch_gemm
  // sets split_tiles (the number of such tiles, the last in tile order).
  int tail_split = 0;
  int split_tiles = 0;
  // kEpiStore / kEpiSumSq / kEpiDotD / kEpiUpdate (Gram loss): per-(row, n-tile) sums
  float* part = nullptr;  // [M, part_ld], part_ld >= num_n_blk * kEpiHalves (kEpiUpdate: part_out)
  int part_ld = 0;
  // kEpiStore: when set, the diagonal (column == row j) is written here in fp32,
  // at [c_row_off + j], and stored as 0 in the bf16 pair
  float* diag_out = nullptr;
  // kEpiStore of a symmetric MN-major product on pair tiles (the Gram matrices):
  // K is summed in chunks of k_chunk K blocks, each a separate accumulation in
  // tensor memory handed to the epilogue, which adds it to the tile's running sums
  // in fp32 (round to nearest) in registers, so no tensor-core accumulation runs
  // over more than one chunk.  0: one accumulation over the whole K.
  int k_chunk = 0;
  // kEpiUpdate / kEpiDotD: when set, C_jk += D_jk * diag_in[k] in fp32 (the exact
  // diagonal of a Gram matrix whose bf16 pair holds only the off-diagonal part)
  const float* diag_in = nullptr;
  // kEpiDotD
  const __nv_bfloat16* Dd_hi = nullptr;  // [M, N]
  const __nv_bfloat16* Dd_lo = nullptr;

  // kEpiUpdate
  const void* W = nullptr;
  int w_bf16 = 0;
  const float* V_in = nullptr;   // state of this step
  float* V_out = nullptr;        // state of the next step (== V_in: in place)
  const float* alpha_in = nullptr;
  float* alpha_out = nullptr;
  const float* beta_in = nullptr;
  float* beta_out = nullptr;
  const float* wmin = nullptr;
  const float* wmax = nullptr;
  __nv_bfloat16* D_hi = nullptr;  // next step's W' - W
  __nv_bfloat16* D_lo = nullptr;  // may be null (single bf16)
  float* V_best = nullptr;
  float* alpha_best = nullptr;
  float* beta_best = nullptr;
  const float* best_in = nullptr;  // [M] best mean loss so far
  float* best_out = nullptr;       // [M]
  float* rowloss = nullptr;        // [M] sum of R^2 of the judged step
  const float* part_in = nullptr;  // [M, nparts] partials of the judged step (null: none)
  int nparts = 0;
  int snap_prev = 0;      // 0: judge this step (snapshot V_in); 1: judge the previous one (snapshot V_out)
  float* part_out = nullptr;  // [M, part_ld] this step's sum_k D G partials (Gram form), or null
  // Full-precision-target mode (Gram form): G += C (this block's W M_b, a bf16 pair
  // [M, N]); the row loss gains 2 sum_k D_jk C_jk, and e_row[j] once per row.
  // kEpiDotD (final MSE): C as fp32 [M, N] (the sum over blocks) via Cs, e via e_row.
  const __nv_bfloat16* Cc_hi = nullptr;
  const __nv_bfloat16* Cc_lo = nullptr;
  const float* Cs = nullptr;
  const float* e_row = nullptr;
  // kEpiUpdate*: *div_slow == 0 (counted by the prepare pass) lets W/s use the
  // fast correctly rounded division; null means always __fdiv_rn.
  const int* div_slow = nullptr;
  float inv_batch = 1.0f;
  int g = 0, G = 0, bits = 4, sym = 0, keep_best = 1;
  float lr = 0.f, mlr = 0.f;
  // kEpiUpdate*Wide: [M * G, gslots, 2] partial (d alpha, d beta); slot k of group
  // gg holds the sum over the group's columns in 128-column segment
  // floor(gg * g / 128) + k.
  float* gpart = nullptr;
  int gslots = 0;
  // AR_CHECKS: capacities (elements) of the buffers the epilogues store to -- C_hi
  // and C_lo (chk_c), the [M, N] state V_out, V_best, D (chk_elems), the [M, G]
  // clip factors (chk_groups).  A store outside them is skipped and recorded in
  // *status (kDevCheck).  0: no checks.
  int64_t chk_c = 0, chk_elems = 0, chk_groups = 0;
};

// After a wide-group step launch: per (row, group), d alpha and d beta as the sum
// of the group's segment partials in slot order, the clip-factor sign updates
// (with the keep-best snapshot of alpha and beta), and the next step's
// D = W' - W from the updated state as a bf16 pair.  One warp per group.
struct GroupFinishArgs {
  const void* W = nullptr;
  int w_bf16 = 0;
  int64_t out = 0, in = 0;
  int g = 0, G = 0, gslots = 0;
  const float* gpart = nullptr;
  const float* V = nullptr;  // the state after the step (the launch's V_out)
  const float* wmin = nullptr;
  const float* wmax = nullptr;
  const float* alpha_in = nullptr;
  const float* beta_in = nullptr;
  float* alpha_out = nullptr;
  float* beta_out = nullptr;
  float* alpha_best = nullptr;
  float* beta_best = nullptr;
  // keep-best: the launch judged a loss (part_in set) and row j improved iff
  // best_out[j] < best_in[j]; snap_prev as in GemmArgs
  int judged = 0, keep_best = 1, snap_prev = 0;
  const float* best_in = nullptr;
  const float* best_out = nullptr;
  __nv_bfloat16* D_hi = nullptr;
  __nv_bfloat16* D_lo = nullptr;
  const int* div_slow = nullptr;
  int bits = 4, sym = 0;
  float mlr = 0.f;
  int64_t chk_elems = 0, chk_groups = 0;  // AR_CHECKS, as in GemmArgs
  int* status = nullptr;
};
cudaError_t launch_group_finish(const GroupFinishArgs& a, cudaStream_t stream);

// Tile sizes: M and K tiles fixed, N tile 128 or 256 per launch.
constexpr int kBM = 128;
constexpr int kBK = 64;
// Two epilogue warps share each accumulator row, one per column half of the tile;
// the per-(row, n-tile) partial sums (GemmArgs::part, part_out) therefore hold
// kEpiHalves entries per n-tile, at n_blk * kEpiHalves + half.
constexpr int kEpiHalves = 2;

cudaError_t launch_gemm(EpiKind kind, int bn, const GemmMaps& maps, const GemmArgs& args, int num_sms,
                        cudaStream_t stream);


// TMA descriptor for a row-major bf16 matrix [rows, cols], box [box_rows, 64]
// with 128-byte swizzle; zero fill outside the matrix.
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);

}  // namespace ar
