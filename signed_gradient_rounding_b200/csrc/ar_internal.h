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
  __nv_bfloat16* D = nullptr;      // [out, in] bf16(s*(q - zp) - W)
};

cudaError_t launch_group_quant(const GroupQuantArgs& a, cudaStream_t stream);
cudaError_t launch_pack(const uint8_t* codes, int64_t rows, int64_t cols, int bits, int32_t* packed,
                        cudaStream_t stream);
cudaError_t launch_fill_f32(float* p, int64_t n, float value, cudaStream_t stream);
cudaError_t launch_transpose_bf16(const uint16_t* X, int64_t rows, int64_t cols, uint16_t* Xt,
                                  cudaStream_t stream);
// loss_trace[t] = sum_j rowloss[t*out + j] / (batch_rows * out), t < iters (fixed order).
cudaError_t launch_loss_trace(const float* rowloss, int64_t out, int iters, int64_t batch_rows,
                              float* loss_trace, cudaStream_t stream);
// final_mse[0] = sum of parts[0 .. count) / denom in fp64 (fixed order).
cudaError_t launch_sum_to_double(const float* parts, int64_t count, double denom, double* result,
                                 cudaStream_t stream);
cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t stream);

// ---------------------------------------------------------------------------
// Persistent tcgen05 GEMM, C[M, N] = A[M, K] * B[N, K]^T, both operands K-major
// bf16 loaded by TMA, fp32 accumulators in tensor memory, fused epilogues.
// ---------------------------------------------------------------------------

enum EpiKind : int {
  kEpiResidual = 0,  // C = R^T tile of one step: store bf16, per-(row, n-tile) sums of R^2
  kEpiUpdate = 1,    // C = G tile: straight-through sign updates of V, alpha, beta; next D
  kEpiLoss = 2       // C = R^T tile: per-(row, n-tile) sums of R^2 only
};

struct GemmArgs {
  int M = 0, N = 0, K = 0;
  int num_m_blk = 0, num_n_blk = 0, num_k_blk = 0, num_tiles = 0;
  int b_row_off = 0;  // added to B's row coordinate (first calibration row of the block)
  int b_k_off = 0;    // added to B's K coordinate
  uint64_t timeout_ns = 1000000000ull;
  int* status = nullptr;

  // kEpiResidual / kEpiLoss
  __nv_bfloat16* Rt = nullptr;  // [M, ldr]
  int64_t ldr = 0;
  float* part = nullptr;        // [M, part_ld] row sums of R^2 per n-tile
  int part_ld = 0;

  // kEpiUpdate
  const void* W = nullptr;
  int w_bf16 = 0;
  float* V = nullptr;
  float* alpha = nullptr;
  float* beta = nullptr;
  const float* wmin = nullptr;
  const float* wmax = nullptr;
  __nv_bfloat16* D = nullptr;
  float* V_best = nullptr;
  float* alpha_best = nullptr;
  float* beta_best = nullptr;
  const float* best_in = nullptr;   // [M] best loss before this step
  float* best_out = nullptr;        // [M] best loss after this step
  float* rowloss = nullptr;         // [M] this step's per-row sum of R^2
  const float* part_in = nullptr;   // [M, nparts] from the residual GEMM
  int nparts = 0;
  float inv_batch = 1.0f;
  int g = 0, G = 0, bits = 4, sym = 0, keep_best = 1;
  float lr = 0.f, mlr = 0.f;
};

// Tile sizes of the GEMM.
constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;

cudaError_t launch_gemm(EpiKind kind, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args,
                        int num_sms, cudaStream_t stream);

// TMA descriptor for a row-major bf16 matrix [rows, cols], box [box_rows, 64]
// with 128-byte swizzle; zero fill outside the matrix.
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                           uint32_t box_rows);

}  // namespace ar
