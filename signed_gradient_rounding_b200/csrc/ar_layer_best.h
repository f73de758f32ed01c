// Layer-wide keep-best (ar_tune_params.keep_best = AR_KEEP_BEST_LAYER), after the
// loop in "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END":
// the step loss total_loss is summed over the layer's outputs, and tracking its
// lowest value picks one step for every row.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace ar {

// After a step's row-loss partials are complete: the layer's batch loss
// Lsum = sum over rows j of fp32(L_j) * inv_batch (L_j the fp32 sum of
// part[j, 0 .. nparts) in index order, as the step epilogues take it), summed in
// fp64 in a fixed order (kLayerBlocks row ranges, each a fixed tree, then the ranges
// in index order).  improved = Lsum < *best; then *best = Lsum and every
// best_rows[j] = Lsum (the state's best_loss in this mode).
//
// The decision reaches the per-row keep-best code unchanged through thresh[j]:
// +inf when the layer improved (every row's loss is below it: every row takes the
// step's state), -inf otherwise (no row does).  The judging launch reads thresh as
// its best_in and writes its best_out to a scratch row array.
//
// init: *best = best_rows[0] (+inf on a fresh state), *ticket = 0; no reduction.
constexpr int kLayerBlocks = 32;
struct LayerBestArgs {
  const float* part = nullptr;
  int nparts = 0;
  int64_t out = 0;
  float inv_batch = 1.f;
  int init = 0;
  double* best = nullptr;          // workspace
  unsigned int* ticket = nullptr;  // workspace, 0 between launches
  double* blocksum = nullptr;      // workspace [kLayerBlocks]
  float* best_rows = nullptr;      // [out]
  float* thresh = nullptr;         // [out]
};
cudaError_t launch_layer_best(const LayerBestArgs& a, cudaStream_t stream);

}  // namespace ar
