// libar C ABI: argument validation, workspace layout, the calibration-block
// schedule and the launch sequence of the tuning loop.
#include <cudaTypedefs.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "../../include/ar.h"
#include "ar_device.cuh"
#include "ar_internal.h"
#include "ar_layer_best.h"

namespace ar {

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime, so the
// library does not link libcuda and loads on machines without a driver).
// ---------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = get_encode_fn();
  if (!encode) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estrides[2] = {1, 1};
  CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                      estrides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

namespace {

// ---------------------------------------------------------------------------
// Calibration-block schedule.  The pages iterate over calibration batches without
// saying how one is picked per step; this library visits the n/B blocks once per
// epoch in the order of a Durstenfeld (Fisher-Yates) shuffle of the identity,
// each swap index being x mod (i + 1) for the next output x of one SplitMix64
// stream (Steele, Lea & Flood, OOPSLA 2014) seeded with `seed` and continued
// across epochs.  A single block draws nothing.
// ---------------------------------------------------------------------------

struct SplitMix64 {
  uint64_t state;
  uint64_t next() {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
};

std::vector<int64_t> block_schedule(int64_t n_blocks, int64_t first, int64_t count, uint64_t seed) {
  std::vector<int64_t> out;
  out.reserve(static_cast<size_t>(count));
  if (n_blocks == 1) {
    out.assign(static_cast<size_t>(count), 0);
    return out;
  }
  SplitMix64 rng{seed};
  std::vector<int64_t> perm(static_cast<size_t>(n_blocks));
  int64_t t = 0;
  while (t < first + count) {
    for (int64_t i = 0; i < n_blocks; ++i) perm[i] = i;
    for (int64_t i = n_blocks - 1; i > 0; --i) {
      const int64_t j = static_cast<int64_t>(rng.next() % static_cast<uint64_t>(i + 1));
      const int64_t tmp = perm[i];
      perm[i] = perm[j];
      perm[j] = tmp;
    }
    for (int64_t i = 0; i < n_blocks && t < first + count; ++i, ++t)
      if (t >= first) out.push_back(perm[i]);
  }
  return out;
}

// ---------------------------------------------------------------------------
// Validation helpers
// ---------------------------------------------------------------------------

bool bits_ok(int bits) { return bits == 2 || bits == 3 || bits == 4 || bits == 8; }

int64_t group_of(int64_t in, int group_size) { return group_size == -1 ? in : group_size; }

bool group_ok(int64_t in, int group_size) {
  const int64_t g = group_of(in, group_size);
  return g > 0 && in % g == 0;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

ar_status from_cuda(cudaError_t e) { return e == cudaSuccess ? AR_OK : AR_ECUDA; }

// Test hooks read from the environment on every call (see ar.h):
//   AR_FAULT=param|alloc|launch|bounds  makes one kind of failure happen on the host;
//   AR_CHECKS=1                          turns on the device-side bounds checks.
enum Fault { kFaultNone = 0, kFaultParam, kFaultAlloc, kFaultLaunch, kFaultBounds };

Fault injected_fault() {
  const char* f = getenv("AR_FAULT");
  if (!f || !*f) return kFaultNone;
  if (!strcmp(f, "param")) return kFaultParam;
  if (!strcmp(f, "alloc")) return kFaultAlloc;
  if (!strcmp(f, "launch")) return kFaultLaunch;
  if (!strcmp(f, "bounds")) return kFaultBounds;
  return kFaultNone;
}

bool checks_on() {
  const char* c = getenv("AR_CHECKS");
  return c && *c && strcmp(c, "0") != 0;
}

// AR_TAIL_SPLIT=0 turns off the column-half split of the step launches' last
// partial wave (GemmArgs::tail_split); it changes the schedule, not the results.
bool tail_split_on() {
  const char* c = getenv("AR_TAIL_SPLIT");
  return !(c && !strcmp(c, "0"));
}

#define AR_CUDA_TRY(expr)                   \
  do {                                      \
    cudaError_t e_ = (expr);                \
    if (e_ != cudaSuccess) return AR_ECUDA; \
  } while (0)

// Groups are whole multiples of 16 columns (the update epilogue walks 16-column
// chunks that never straddle a group).
bool tune_shape_supported(int64_t in, int64_t g, int64_t B) {
  if (in % 32 != 0 || B % 8 != 0) return false;
  return g % 16 == 0;
}

// Groups that fit inside one epilogue thread's columns are updated in the step's
// epilogue; wider or unaligned ones (whole-row groups of a wide layer, or sizes
// that do not divide 256) through per-segment partials and launch_group_finish.
bool wide_groups(int64_t in, int64_t g) { return !((256 % g == 0) || (g == in && in <= 256)); }

ar_status check_tune_args(int64_t out, int64_t in, int64_t n_rows, const ar_tune_params* p) {
  if (injected_fault() == kFaultParam) return AR_EINVAL;
  if (!p || out < 0 || in < 0 || n_rows < 0) return AR_EINVAL;
  if (!bits_ok(p->bits)) return AR_EINVAL;
  if (p->iters < 0 || !(p->lr >= 0.0f) || !isfinite(p->lr) || !isfinite(p->minmax_lr)) return AR_EINVAL;
  if (!(p->minmax_shrink > 0.0f) || !isfinite(p->minmax_shrink)) return AR_EINVAL;
  if (p->start_step < 0) return AR_EINVAL;
  if (p->algo < AR_ALGO_AUTO || p->algo > AR_ALGO_GRAM) return AR_EINVAL;
  if (p->init != AR_INIT_MINMAX && p->init != AR_INIT_MSE) return AR_EINVAL;
  if (p->keep_best < AR_KEEP_LAST || p->keep_best > AR_KEEP_BEST_LAYER) return AR_EINVAL;
  if (p->split < 0 || p->split > 2) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!group_ok(in, p->group_size)) return AR_EINVAL;
  if (p->batch_rows <= 0 || n_rows < p->batch_rows || n_rows % p->batch_rows != 0) return AR_EINVAL;
  if (out >= (1ll << 31) || in >= (1ll << 31) || n_rows >= (1ll << 31)) return AR_EUNSUPPORTED;
  if (!tune_shape_supported(in, group_of(in, p->group_size), p->batch_rows)) return AR_EUNSUPPORTED;
  return AR_OK;
}

// ---------------------------------------------------------------------------
// Plan: which algorithm, tile widths, workspace layout.
// ---------------------------------------------------------------------------

constexpr double kGramMaxBytes = 64.0 * (1ull << 30);
// The full-precision-target mode in the Gram form keeps, on top of the Gram matrices,
// every block's C_b = W M_b as a bf16 pair (n_rows/batch_rows * out * in * 4 bytes).
// It runs in that form while its workspace stays within this, in the direct form
// otherwise (the automatic choice), and an explicit AR_ALGO_GRAM beyond it is
// refused: the 8192 x 29568 down_proj with 16 blocks of 16384 rows would need about
// 80 GB there, and about 14 GB in the direct form.
constexpr size_t kFpTargetMaxBytes = 64ull << 30;

struct Plan {
  int algo = AR_ALGO_DIRECT;
  int split = 1;
  // split = 2: the Gram step sums K in chunks of exact_chunk K blocks (kEpiUpdateExact).
  bool exact = false;
  int exact_chunk = 8;
  int64_t out = 0, in = 0, n = 0, B = 0, g = 0, G = 0, nb = 0, iters = 0;
  int bn_res = 256;   // direct: residual GEMM (N = B)
  int bn_upd = 256;   // update GEMM (N = in)
  int bn_gram = 256;  // Gram matrices (N = in)
  int bn_fin = 256;   // final-MSE GEMM
  int64_t nparts_res = 0, nparts_upd = 0, nparts_fin = 0;
  // Gram-form update GEMM on 2-SM pair tiles (256 x 256, tcgen05 cta_group::2):
  // each SM stages half of the tile's B rows.
  bool pair_upd = true;
  // ... with the three pair products fused per K block (Cfg::kFused): the hi tiles
  // of D and H are staged once per K block rather than twice.
  bool fused_upd = true;
  // Direct form (residual, update, final MSE): X_b (or X_b^T) staged once per K
  // block for both halves of the pair operand instead of once per half.
  bool fused_direct = true;
  // Full-precision-target products (M_b^T, C_b, e_b) on pair tiles with fused stages.
  bool pair_fpt = true;
  // Gram matrices (symmetric, upper tiles only) on pair tiles.
  bool pair_gram = true;
  // Pair tiles in groups of 8 m-blocks (2048 rows): measured ~1.5% faster than
  // one sweep over all rows on the 4096 x 4096 layer.
  int raster_upd = 8;
  // Full-precision-target mode (ar_tune_layer_fp_target; Gram form only), and
  // whether W is fp32 (then held as a bf16 pair for its contractions).
  bool fp_target = false;
  bool w_f32 = false;
  // Wide groups (see wide_groups) and the segment slots of their partials.
  bool wide = false;
  int gslots = 0;
  // Direct-form residual and update GEMMs on pair tiles: measured 3% faster on the
  // 4096-wide layer, 3-10% slower (more energy per step at the power cap) on the
  // 29568-wide one, which is where the automatic choice picks the direct form.
  bool pair_direct = false;
  // Gram matrices summed over chunks of gram_chunk calibration rows (GemmArgs::
  // k_chunk): each chunk is its own tensor-core accumulation, and the epilogue adds
  // the chunks in fp32 (round to nearest).  The tensor cores' fp32 accumulation
  // loses low bits on each of its additions; over a whole 16384-row block that
  // shrank every entry of H_b by about 6e-5 (relative), enough to turn gradient
  // signs that sit within about 1e-5 of their rms.
  int64_t gram_chunk = 2048;
};



Plan make_plan(int64_t out, int64_t in, int64_t n, const ar_tune_params* p, bool fp_target = false,
               bool w_f32 = false) {
  Plan P;
  P.fp_target = fp_target;
  P.w_f32 = w_f32;
  P.split = p->split != 0;
  P.exact = p->split == 2;
  P.out = out;
  P.in = in;
  P.n = n;
  P.B = p->batch_rows;
  P.g = group_of(in, p->group_size);
  P.G = in / P.g;
  P.nb = n / P.B;
  P.iters = p->iters;
  const double pieces_direct = P.split ? 2.0 : 1.0;
  const double pieces_gram = P.split ? 3.0 : 1.0;
  const double direct = P.iters * pieces_direct * 4.0 * P.B * out * in + pieces_direct * 2.0 * n * out * in;
  const double gram =
      P.iters * pieces_gram * 2.0 * out * in * in + 2.0 * n * in * in + pieces_gram * 2.0 * out * in * in;
  const double gram_bytes = (P.nb + 1.0) * in * in * 2.0 * (P.split ? 2.0 : 1.0);
  // Full-precision target: the Gram form also keeps every block's C_b = W M_b (a bf16
  // pair) on top of the Gram matrices; it is chosen while that stays within
  // kFpTargetMaxBytes, the direct form otherwise.
  const double gram_fpt_bytes = gram_bytes + (P.nb * 4.0 + 24.0) * out * in;
  if (p->algo == AR_ALGO_GRAM || (fp_target && p->algo == AR_ALGO_AUTO && gram_fpt_bytes <= kFpTargetMaxBytes))
    P.algo = AR_ALGO_GRAM;
  else if (p->algo == AR_ALGO_DIRECT || fp_target)
    P.algo = AR_ALGO_DIRECT;
  else
    P.algo = (P.iters > 0 && gram < direct && gram_bytes <= kGramMaxBytes) ? AR_ALGO_GRAM : AR_ALGO_DIRECT;
  // N tiles of 256: a 128x128x16 MMA reads as many operand bytes from shared
  // memory per clock as the SM can deliver, 128x256 reads three quarters of that.
  P.bn_upd = 256;
  P.bn_gram = 256;
  P.bn_fin = 256;
  P.wide = wide_groups(in, P.g);
  P.gslots = P.wide ? static_cast<int>(cdiv(P.g, kSegCols) + 1) : 0;
  // Row partial sums: kEpiHalves per n-tile (one per epilogue column half).
  P.nparts_res = cdiv(P.B, P.bn_res) * kEpiHalves;
  P.nparts_upd = cdiv(in, P.bn_upd) * kEpiHalves;
  P.nparts_fin = (P.algo == AR_ALGO_GRAM ? cdiv(in, P.bn_fin) : cdiv(n, P.bn_fin)) * kEpiHalves;
  return P;
}

// Workspace layout (offsets in bytes from the workspace base).
struct Layout {
  size_t status, D_hi, D_lo, D_hi1, D_lo1, V0, V1, a0, a1, b0, b1, V_best, alpha_best, beta_best, best0, best1,
      wmin, wmax, part0, part1, rowloss, gpart, Rt_hi, Rt_lo, H_hi, H_lo, Hs_hi, Hs_lo, Hdiag, Hdsum,
      // full-precision-target mode: this block's dX = X - X_target (pair),
      // M_b^T = X_b^T dX_b (pair), every block's C_b = W M_b (pair), their sum Cs
      // (fp32), e_b[j] = |dX_b w_j^T|^2 and its sum, the partials of e_b, and W as
      // a pair when it is fp32
      dX_hi, dX_lo, Mt_hi, Mt_lo, Cc_hi, Cc_lo, Cs, e, es, epart, Wp_hi, Wp_lo,
      // direct form with a full-precision target: E^T = W dX^T for every block, [out, n]
      // as a bf16 pair (block b in columns b*B ..), added to the residual
      E_hi, E_lo,
      // layer-wide keep-best: the best loss (fp64), the reduction's ticket and its
      // per-range sums; the per-row thresholds and the judging launch's scratch
      layer, layer_rows, total;
};

Layout make_layout(const Plan& P) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 1024);
    return o;
  };
  const size_t elems = static_cast<size_t>(P.out) * P.in;
  const size_t groups = static_cast<size_t>(P.out) * P.G;
  const bool gram = P.algo == AR_ALGO_GRAM;
  const int64_t nparts = std::max(std::max(P.nparts_res, P.nparts_upd), P.nparts_fin);
  L.status = take(256);
  L.layer = take(16 + kLayerBlocks * 8);
  L.layer_rows = take(static_cast<size_t>(P.out) * 2 * 4);
  L.D_hi = take(elems * 2);
  L.D_lo = take(elems * 2);
  // The Gram form reads D_t and writes D_{t+1} in the same launch: two buffers.
  L.D_hi1 = gram ? take(elems * 2) : L.D_hi;
  L.D_lo1 = gram ? take(elems * 2) : L.D_lo;
  L.V0 = take(elems * 4);
  L.V1 = gram ? take(elems * 4) : L.V0;
  L.a0 = take(groups * 4);
  L.b0 = take(groups * 4);
  L.a1 = gram ? take(groups * 4) : L.a0;
  L.b1 = gram ? take(groups * 4) : L.b0;
  L.V_best = take(elems * 4);
  L.alpha_best = take(groups * 4);
  L.beta_best = take(groups * 4);
  L.best0 = take(static_cast<size_t>(P.out) * 4);
  L.best1 = take(static_cast<size_t>(P.out) * 4);
  L.wmin = take(groups * 4);
  L.wmax = take(groups * 4);
  L.part0 = take(static_cast<size_t>(P.out) * nparts * 4);
  L.part1 = gram ? take(static_cast<size_t>(P.out) * nparts * 4) : L.part0;
  L.rowloss = take(static_cast<size_t>(P.out) * std::max<int64_t>(P.iters, 1) * 4);
  L.gpart = P.wide ? take(groups * P.gslots * 2 * 4) : 0;
  if (gram) {
    const size_t h = static_cast<size_t>(P.in) * P.in * 2;
    L.H_hi = take(h * P.nb);
    L.H_lo = P.split ? take(h * P.nb) : L.H_hi;
    L.Hs_hi = take(h);
    L.Hs_lo = P.split ? take(h) : L.Hs_hi;
    L.Hdiag = take(static_cast<size_t>(P.nb) * P.in * 4);
    L.Hdsum = take(static_cast<size_t>(P.in) * 4);
    if (P.fp_target) {
      const size_t blk = static_cast<size_t>(P.B) * P.in * 2;
      L.dX_hi = take(blk);
      L.dX_lo = take(blk);
      L.Mt_hi = take(h);
      L.Mt_lo = take(h);
      L.Cc_hi = take(elems * 2 * P.nb);
      L.Cc_lo = take(elems * 2 * P.nb);
      L.Cs = take(elems * 4);
      L.e = take(static_cast<size_t>(P.nb) * P.out * 4);
      L.es = take(static_cast<size_t>(P.out) * 4);
      L.epart = take(static_cast<size_t>(P.out) * cdiv(P.B, 256) * kEpiHalves * 4);
      if (P.w_f32) {
        L.Wp_hi = take(elems * 2);
        L.Wp_lo = take(elems * 2);
      }
    }
  } else {
    L.Rt_hi = take(static_cast<size_t>(P.out) * P.B * 2);
    L.Rt_lo = P.split ? take(static_cast<size_t>(P.out) * P.B * 2) : L.Rt_hi;
    if (P.fp_target) {
      const size_t blk = static_cast<size_t>(P.B) * P.in * 2;
      L.dX_hi = take(blk);
      L.dX_lo = take(blk);
      L.E_hi = take(static_cast<size_t>(P.out) * P.n * 2);
      L.E_lo = take(static_cast<size_t>(P.out) * P.n * 2);
      if (P.w_f32) {
        L.Wp_hi = take(elems * 2);
        L.Wp_lo = take(elems * 2);
      }
    }
  }
  L.total = off;
  return L;
}

void fill_grid(GemmArgs& a, int64_t M, int64_t N, int64_t K, int bn, int num_seg, bool pair = false) {
  a.M = static_cast<int>(M);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.pair = pair ? 1 : 0;
  a.num_m_blk = static_cast<int>(cdiv(M, pair ? 2 * kBM : kBM));
  a.num_n_blk = static_cast<int>(cdiv(N, bn));
  a.num_k_blk = static_cast<int>(cdiv(K, kBK));
  a.num_tiles = a.num_m_blk * a.num_n_blk;
  a.num_seg = num_seg;
}

// Events around the contractions of a timed call, three per step and none shared
// between steps (work that prepares a block runs between steps): ev[3t] before
// step t's first contraction, ev[3t+1] after it, ev[3t+2] after the update
// (DIRECT; the Gram form has one contraction per step and leaves ev[3t+2] unused).
struct EventTimer {
  std::vector<cudaEvent_t> ev;
  cudaEvent_t start = nullptr, stop = nullptr;
  int launches = 0;
  int algo = 0;
  bool create(int iters) {
    ev.assign(static_cast<size_t>(3 * iters + 1), nullptr);
    for (auto& e : ev)
      if (cudaEventCreate(&e) != cudaSuccess) return false;
    return cudaEventCreate(&start) == cudaSuccess && cudaEventCreate(&stop) == cudaSuccess;
  }
  ~EventTimer() {
    for (auto e : ev)
      if (e) cudaEventDestroy(e);
    if (start) cudaEventDestroy(start);
    if (stop) cudaEventDestroy(stop);
  }
};

// block_ready (optional, one event per calibration block): the stream waits for
// block b's event before the first kernel that reads block b of X.
ar_status tune_impl(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X, int64_t n_rows,
                    const ar_tune_params* p, ar_tune_state* state, void* workspace, size_t ws_bytes,
                    uint8_t* codes, float* scale, int32_t* zp, float* loss_trace, double* final_mse,
                    void* stream, EventTimer* timer, const cudaEvent_t* block_ready = nullptr,
                    const uint16_t* X_target = nullptr) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!W || !X || !workspace || !codes || !scale || !zp) return AR_EINVAL;
  if (!aligned(W, 16) || !aligned(X, 16) || !aligned(workspace, 256)) return AR_EINVAL;
  if (state) {
    const void* ptrs[7] = {state->V,      state->alpha,      state->beta,     state->best_loss,
                           state->V_best, state->alpha_best, state->beta_best};
    for (const void* q : ptrs)
      if (!q || !aligned(q, 16)) return AR_EINVAL;
  }

  if (X_target && !aligned(X_target, 16)) return AR_EINVAL;
  const Plan P = make_plan(out, in, n_rows, p, X_target != nullptr, w_dtype == AR_F32);
  const Layout L = make_layout(P);
  if (P.fp_target && P.algo == AR_ALGO_GRAM && L.total > kFpTargetMaxBytes) return AR_EUNSUPPORTED;
  // The chunked accumulation exists for the plain Gram step with groups inside a thread's
  // columns.
  if (P.exact && (P.algo != AR_ALGO_GRAM || P.wide || P.fp_target)) return AR_EUNSUPPORTED;
  const Fault fault = injected_fault();
  if (ws_bytes < L.total || fault == kFaultAlloc) return AR_ENOMEM;
  const bool gram = P.algo == AR_ALGO_GRAM;
  const int64_t B = P.B;
  const int iters = p->iters;
  const bool checks = checks_on();

  int dev = 0, sms = 0, major = 0;
  AR_CUDA_TRY(cudaGetDevice(&dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  if (major != 10) return AR_EUNSUPPORTED;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  auto H = [&](size_t off) { return reinterpret_cast<__nv_bfloat16*>(ws + off); };
  int* status = reinterpret_cast<int*>(ws + L.status);
  // Second word of the status block: groups whose weights need the IEEE division.
  int* div_slow = status + 1;
  __nv_bfloat16* D_hi = H(L.D_hi);
  __nv_bfloat16* D_lo = H(L.D_lo);
  __nv_bfloat16* Dh[2] = {D_hi, H(L.D_hi1)};
  __nv_bfloat16* Dl[2] = {D_lo, H(L.D_lo1)};
  float* wmin = F(L.wmin);
  float* wmax = F(L.wmax);
  float* part[2] = {F(L.part0), F(L.part1)};
  float* rowloss = F(L.rowloss);
  // Live state: buffer 0 is the caller's state (or the workspace's); the Gram
  // form double-buffers V, alpha, beta because its keep-best check of a step runs
  // one step later.
  float* Vb[2];
  float* ab[2];
  float* bb[2];
  float *best_loss, *V_best, *alpha_best, *beta_best;
  if (state) {
    Vb[0] = state->V;
    ab[0] = state->alpha;
    bb[0] = state->beta;
    best_loss = state->best_loss;
    V_best = state->V_best;
    alpha_best = state->alpha_best;
    beta_best = state->beta_best;
  } else {
    Vb[0] = F(L.V0);
    ab[0] = F(L.a0);
    bb[0] = F(L.b0);
    best_loss = F(L.best0);
    V_best = F(L.V_best);
    alpha_best = F(L.alpha_best);
    beta_best = F(L.beta_best);
  }
  Vb[1] = gram ? F(L.V1) : Vb[0];
  ab[1] = gram ? F(L.a1) : ab[0];
  bb[1] = gram ? F(L.b1) : bb[0];
  float* best_alt = F(L.best1);
  const bool init_state = !state || !state->initialized;
  const size_t elems = static_cast<size_t>(out) * in;
  const size_t groups = static_cast<size_t>(out) * P.G;

  int launches = 0;
  if (timer) {
    timer->algo = P.algo;
    AR_CUDA_TRY(cudaEventRecord(timer->start, st));
  }
  AR_CUDA_TRY(cudaMemsetAsync(status, 0, 2 * sizeof(int), st));
  if (init_state) {
    AR_CUDA_TRY(cudaMemsetAsync(Vb[0], 0, elems * 4, st));
    AR_CUDA_TRY(cudaMemsetAsync(V_best, 0, elems * 4, st));
    if (p->init == AR_INIT_MSE) {
      AR_CUDA_TRY(launch_mse_init(W, w_dtype == AR_BF16, out, in, static_cast<int>(P.g), p->bits, p->sym != 0,
                                  ab[0], bb[0], st));
      AR_CUDA_TRY(cudaMemcpyAsync(alpha_best, ab[0], groups * 4, cudaMemcpyDeviceToDevice, st));
      AR_CUDA_TRY(cudaMemcpyAsync(beta_best, bb[0], groups * 4, cudaMemcpyDeviceToDevice, st));
      launches += 1;
    } else {
      AR_CUDA_TRY(launch_fill_f32(ab[0], groups, p->minmax_shrink, st));
      AR_CUDA_TRY(launch_fill_f32(bb[0], groups, p->minmax_shrink, st));
      AR_CUDA_TRY(launch_fill_f32(alpha_best, groups, p->minmax_shrink, st));
      AR_CUDA_TRY(launch_fill_f32(beta_best, groups, p->minmax_shrink, st));
      launches += 4;
    }
    AR_CUDA_TRY(launch_fill_f32(best_loss, out, INFINITY, st));
    launches += 1;
  }

  // Layer-wide keep-best: after each step's partials are complete, one small
  // reduction takes the layer's decision and hands it to the per-row keep-best code
  // as thresholds (+inf: every row takes the step, -inf: none), which the launch that
  // judges the step (and the wide-group finish, and the last step's finalize) read as
  // best_in; their best_out goes to a scratch array.
  const bool layer_best = p->keep_best == AR_KEEP_BEST_LAYER && iters > 0;
  LayerBestArgs lb;
  lb.out = out;
  lb.inv_batch = 1.0f / static_cast<float>(B);
  lb.best = reinterpret_cast<double*>(ws + L.layer);
  lb.ticket = reinterpret_cast<unsigned int*>(ws + L.layer + 8);
  lb.blocksum = reinterpret_cast<double*>(ws + L.layer + 16);
  lb.best_rows = best_loss;
  lb.thresh = F(L.layer_rows);
  float* layer_scratch = F(L.layer_rows) + out;
  if (layer_best) {
    lb.init = 1;  // the best so far: best_loss[0] (+inf on a fresh state)
    AR_CUDA_TRY(launch_layer_best(lb, st));
    lb.init = 0;
    ++launches;
  }
  auto judge_layer = [&](const float* parts, int64_t nparts) -> cudaError_t {
    if (!layer_best) return cudaSuccess;
    lb.part = parts;
    lb.nparts = static_cast<int>(nparts);
    ++launches;
    return launch_layer_best(lb, st);
  };

  // Full-precision-target mode: the block sums start at zero; an fp32 W is held as
  // a bf16 pair for its contractions.
  const bool fpt = P.fp_target;
  const __nv_bfloat16* Wa_hi = static_cast<const __nv_bfloat16*>(W);
  const __nv_bfloat16* Wa_lo = nullptr;
  if (fpt) {
    if (gram) {
      AR_CUDA_TRY(cudaMemsetAsync(F(L.Cs), 0, elems * 4, st));
      AR_CUDA_TRY(cudaMemsetAsync(F(L.es), 0, static_cast<size_t>(out) * 4, st));
    }
    if (P.w_f32) {
      AR_CUDA_TRY(launch_split_pair(static_cast<const float*>(W), static_cast<int64_t>(elems), H(L.Wp_hi),
                                    H(L.Wp_lo), st));
      ++launches;
      Wa_hi = H(L.Wp_hi);
      Wa_lo = H(L.Wp_lo);
    }
  }

  // Group statistics of W and the first step's D = W' - W.
  GroupQuantArgs prep;
  prep.W = W;
  prep.w_bf16 = w_dtype == AR_BF16;
  prep.out = out;
  prep.in = in;
  prep.g = static_cast<int>(P.g);
  prep.G = static_cast<int>(P.G);
  prep.bits = p->bits;
  prep.sym = p->sym != 0;
  prep.wmin_out = wmin;
  prep.wmax_out = wmax;
  prep.V = Vb[0];
  prep.alpha = ab[0];
  prep.beta = bb[0];
  prep.D_hi = D_hi;
  prep.D_lo = P.split ? D_lo : nullptr;
  prep.div_slow = div_slow;
  if (checks) {
    prep.chk_elems = static_cast<int64_t>(elems);
    prep.chk_groups = static_cast<int64_t>(groups);
    prep.status = status;
  }
  AR_CUDA_TRY(launch_group_quant(prep, st));
  ++launches;

  const uint64_t timeout_ns = 1000000000ull;
  const float mlr = p->minmax_lr < 0.0f ? p->lr : p->minmax_lr;
  const int nseg_d = P.split ? 2 : 1;
  const int nseg_g = P.split ? 3 : 1;
  const std::vector<int64_t> sched = block_schedule(P.nb, p->start_step, iters, p->seed);
  // Gram matrices H_b = X_b^T X_b, as bf16 pairs at rows b*in .. b*in + in.
  GemmMaps gram_maps{};
  GemmArgs h;
  if (gram) {
    // Both operands are X_b^T, read MN-major from the row-major activations through
    // a map of block b alone (made per block), so a K tile that runs past the
    // block's last row reads zeros rather than the next block.
    fill_grid(h, in, in, B, P.bn_gram, 1, P.pair_gram);
    h.a_mn = 1;
    h.b_mn = 1;
    h.symmetric = 1;  // H_b = X_b^T X_b: compute the tiles reaching the upper triangle
    h.num_tiles = 0;
    const int64_t m_height = P.pair_gram ? 2 * kBM : kBM;
    for (int nn = 0; nn < h.num_n_blk; ++nn)
      h.num_tiles += static_cast<int>(std::min<int64_t>(h.num_m_blk, cdiv((nn + 1) * int64_t(P.bn_gram), m_height)));
    h.timeout_ns = timeout_ns;
    h.status = status;
    h.C_hi = H(L.H_hi);
    h.C_lo = P.split ? H(L.H_lo) : nullptr;
    h.ldc = in;
    h.diag_out = F(L.Hdiag);
    h.k_chunk = static_cast<int>(P.gram_chunk / kBK);
    if (checks) h.chk_c = P.nb * in * in;
  }
  // Full-precision-target mode, per block b (dX_b = X_b - X_target,b):
  //   M_b^T = X_b^T dX_b          [in, in]   (pair; A = X_b^T, B = dX_b^T pair)
  //   C_b   = W M_b               [out, in]  (pair; the step adds it to G)
  //   e_b[j] = |dX_b w_j^T|^2     (row sums of squares of W dX_b^T)
  //   Cs += C_b,  es += e_b       (the final MSE over all blocks)
  // Direct form instead: per block only E_b^T = W dX_b^T [out, B], stored into
  // columns b*B .. of the [out, n] pair E; the residual epilogue adds it to
  // X_b D^T, so R = X_b W'^T - X_target,b W^T.
  GemmMaps mt_maps{}, c_maps{}, e_maps{};
  GemmArgs mg, cg, eg;
  if (fpt) {
    const int nseg_w = P.w_f32 ? 3 : 2;  // W pair x operand pair, or W x operand pair
   if (gram) {
    AR_CUDA_TRY(make_tmap_bf16(&mt_maps.b0, H(L.dX_hi), B, in, 64));
    AR_CUDA_TRY(make_tmap_bf16(&mt_maps.b1, H(L.dX_lo), B, in, 64));
    fill_grid(mg, in, in, B, 256, 2, P.pair_fpt);
    mg.fused = P.pair_fpt ? 1 : 0;
    mg.a_mn = 1;  // X_b^T and dX_b^T, read MN-major from the row-major blocks
    mg.b_mn = 1;
    mg.seg_b[1] = 1;
    mg.timeout_ns = timeout_ns;
    mg.status = status;
    mg.C_hi = H(L.Mt_hi);
    mg.C_lo = H(L.Mt_lo);
    mg.ldc = in;
   }
    for (GemmMaps* m : {&c_maps, &e_maps}) {
      AR_CUDA_TRY(make_tmap_bf16(&m->a0, Wa_hi, out, in, kBM));
      if (Wa_lo)
        AR_CUDA_TRY(make_tmap_bf16(&m->a1, Wa_lo, out, in, kBM));
      else
        m->a1 = m->a0;
    }
    const uint32_t fpt_box = P.pair_fpt ? 128 : 256;  // pair tiles: half the B rows per CTA
    if (gram) {
      AR_CUDA_TRY(make_tmap_bf16(&c_maps.b0, H(L.Mt_hi), in, in, fpt_box));
      AR_CUDA_TRY(make_tmap_bf16(&c_maps.b1, H(L.Mt_lo), in, in, fpt_box));
    }
    AR_CUDA_TRY(make_tmap_bf16(&e_maps.b0, H(L.dX_hi), B, in, fpt_box));
    AR_CUDA_TRY(make_tmap_bf16(&e_maps.b1, H(L.dX_lo), B, in, fpt_box));
    for (GemmArgs* g : {&cg, &eg}) {
      fill_grid(*g, out, g == &cg ? in : B, in, 256, nseg_w, P.pair_fpt);
      g->fused = P.pair_fpt ? 1 : 0;
      if (P.w_f32) {  // W_hi X_hi + W_lo X_hi + W_hi X_lo
        g->seg_a[1] = 1;
        g->seg_b[2] = 1;
      } else {        // W X_hi + W X_lo
        g->seg_b[1] = 1;
      }
      g->timeout_ns = timeout_ns;
      g->status = status;
    }
    cg.C_hi = H(L.Cc_hi);
    cg.C_lo = H(L.Cc_lo);
    cg.ldc = in;
    if (gram) {
      eg.part = F(L.epart);
      eg.part_ld = eg.num_n_blk * kEpiHalves;
    } else {
      eg.ldc = n_rows;  // C_hi, C_lo point at block b's columns of E
      if (checks) eg.chk_c = out * n_rows;
    }
  }
  auto fp_target_block = [&](int64_t b) -> cudaError_t {
    const int64_t blk = B * in;
    cudaError_t e = launch_diff_pair(X + b * blk, X_target + b * blk, blk, H(L.dX_hi), H(L.dX_lo), st);
    mt_maps.a0 = gram_maps.a0;  // block b of X (made by ensure_block)
    mt_maps.a1 = gram_maps.a0;
    if (e == cudaSuccess) e = launch_gemm(kEpiStore, 256, mt_maps, mg, sms, st);
    cg.c_row_off = b * out;
    if (e == cudaSuccess) e = launch_gemm(kEpiStore, 256, c_maps, cg, sms, st);
    if (e == cudaSuccess)
      e = launch_accum_pair(H(L.Cc_hi) + b * static_cast<int64_t>(elems), H(L.Cc_lo) + b * static_cast<int64_t>(elems),
                            static_cast<int64_t>(elems), F(L.Cs), st);
    if (e == cudaSuccess) e = launch_gemm(kEpiSumSq, 256, e_maps, eg, sms, st);
    if (e == cudaSuccess) e = launch_row_sum(F(L.epart), eg.part_ld, out, F(L.e) + b * out, F(L.es), st);
    launches += 6;
    return e;
  };

  // In the Gram form each calibration block's Gram matrix is made just before the
  // first step that uses it.  With block_ready events, the block's copy to the
  // device is awaited first (in both forms).
  std::vector<char> have_block(static_cast<size_t>(P.nb), 0), waited_block(static_cast<size_t>(P.nb), 0);
  auto wait_block = [&](int64_t b) -> cudaError_t {
    if (!block_ready || waited_block[b]) return cudaSuccess;
    waited_block[b] = 1;
    return cudaStreamWaitEvent(st, block_ready[b], 0);
  };
  auto fp_target_block_direct = [&](int64_t b) -> cudaError_t {
    const int64_t blk = B * in;
    cudaError_t e = launch_diff_pair(X + b * blk, X_target + b * blk, blk, H(L.dX_hi), H(L.dX_lo), st);
    eg.C_hi = H(L.E_hi) + b * B;
    eg.C_lo = H(L.E_lo) + b * B;
    eg.chk_c = checks ? out * n_rows - b * B : 0;
    if (e == cudaSuccess) e = launch_gemm(kEpiStore, 256, e_maps, eg, sms, st);
    launches += 2;
    return e;
  };
  auto ensure_block = [&](int64_t b) -> cudaError_t {
    if (have_block[b]) return cudaSuccess;
    have_block[b] = 1;
    cudaError_t e = wait_block(b);
    if (e != cudaSuccess) return e;
    if (!gram) return fpt ? fp_target_block_direct(b) : cudaSuccess;
    e = make_tmap_bf16(&gram_maps.a0, X + b * B * in, B, in, 64);
    if (e != cudaSuccess) return e;
    gram_maps.a1 = gram_maps.b0 = gram_maps.b1 = gram_maps.a0;
    h.c_row_off = b * in;
    ++launches;
    e = launch_gemm(kEpiStore, P.bn_gram, gram_maps, h, sms, st);
    if (e != cudaSuccess) return e;
    if (!fpt) return cudaSuccess;
    return fp_target_block(b);
  };

  // The update epilogue's common arguments.
  GemmArgs u;
  u.timeout_ns = timeout_ns;
  u.status = status;
  u.W = W;
  u.w_bf16 = w_dtype == AR_BF16;
  u.wmin = wmin;
  u.wmax = wmax;
  u.D_hi = D_hi;
  u.D_lo = P.split ? D_lo : nullptr;
  u.V_best = V_best;
  u.alpha_best = alpha_best;
  u.beta_best = beta_best;
  u.inv_batch = 1.0f / static_cast<float>(B);
  u.div_slow = div_slow;
  u.g = static_cast<int>(P.g);
  u.G = static_cast<int>(P.G);
  u.bits = p->bits;
  u.sym = p->sym != 0;
  u.keep_best = p->keep_best != 0;
  u.lr = p->lr;
  u.mlr = mlr;
  u.gpart = P.wide ? F(L.gpart) : nullptr;
  u.gslots = P.gslots;
  u.tail_split = tail_split_on() ? 1 : 0;
  if (checks) {
    // AR_FAULT=bounds: the epilogue is told V and D hold one element fewer than
    // they do, so the last chunk's stores are refused (and reported), not made.
    u.chk_elems = static_cast<int64_t>(elems) - (fault == kFaultBounds ? 1 : 0);
    u.chk_groups = static_cast<int64_t>(groups);
  }
  // Wide groups: the group updates and the next D after each step launch.
  auto finish_groups = [&]() -> cudaError_t {
    if (!P.wide) return cudaSuccess;
    GroupFinishArgs f;
    f.W = u.W;
    f.w_bf16 = u.w_bf16;
    f.out = out;
    f.in = in;
    f.g = u.g;
    f.G = u.G;
    f.gslots = u.gslots;
    f.gpart = u.gpart;
    f.V = u.V_out;
    f.wmin = u.wmin;
    f.wmax = u.wmax;
    f.alpha_in = u.alpha_in;
    f.beta_in = u.beta_in;
    f.alpha_out = u.alpha_out;
    f.beta_out = u.beta_out;
    f.alpha_best = u.alpha_best;
    f.beta_best = u.beta_best;
    f.judged = u.part_in != nullptr;
    f.keep_best = u.keep_best;
    f.snap_prev = u.snap_prev;
    f.best_in = u.best_in;
    f.best_out = u.best_out;
    f.D_hi = u.D_hi;
    f.D_lo = u.D_lo;
    f.div_slow = u.div_slow;
    f.bits = u.bits;
    f.sym = u.sym;
    f.mlr = u.mlr;
    f.chk_elems = u.chk_elems;
    f.chk_groups = u.chk_groups;
    f.status = status;
    ++launches;
    return launch_group_finish(f, st);
  };
  // The Gram form's full-precision-target terms enter the step's epilogue; the direct
  // form's are already in R (E_b^T, added by the residual's epilogue).
  const bool fpt_step = fpt && gram;
  const EpiKind upd_kind = P.exact ? kEpiUpdateExact
                           : fpt_step ? (P.wide ? kEpiUpdateFpWide : kEpiUpdateFp)
                                      : (P.wide ? kEpiUpdateWide : kEpiUpdate);
  if (P.exact) u.k_chunk = P.exact_chunk;

  float* best_cur = best_loss;
  float* best_next = best_alt;
  int live = 0;  // buffer holding the live state

  if (gram) {
    // ---------------------------------------------------------- Gram form
    __nv_bfloat16* Hh = H(L.H_hi);
    __nv_bfloat16* Hl = H(L.H_lo);
    GemmMaps m[2]{};  // per parity of t: A = D_t
    // 2-SM pair tiles: each CTA of a pair stages half of the tile's B rows.
    const uint32_t b_box = P.pair_upd ? P.bn_upd / 2 : P.bn_upd;
    for (int q = 0; q < 2; ++q) {
      AR_CUDA_TRY(make_tmap_bf16(&m[q].a0, Dh[q], out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m[q].a1, Dl[q], out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m[q].b0, Hh, P.nb * in, in, b_box));
      AR_CUDA_TRY(make_tmap_bf16(&m[q].b1, Hl, P.nb * in, in, b_box));
    }
    fill_grid(u, out, in, in, P.bn_upd, nseg_g, P.pair_upd);
    u.raster_m = P.raster_upd;
    u.fused = (P.fused_upd && P.pair_upd && nseg_g > 1) ? 1 : 0;
    // (D_hi + D_lo)(H_hi + H_lo) ~ D_hi H_hi + D_lo H_hi + D_hi H_lo
    u.seg_a[0] = 0, u.seg_b[0] = 0;
    u.seg_a[1] = 1, u.seg_b[1] = 0;
    u.seg_a[2] = 0, u.seg_b[2] = 1;
    u.part_ld = static_cast<int>(P.nparts_upd);
    u.nparts = static_cast<int>(P.nparts_upd);
    u.snap_prev = 1;
    for (int t = 0; t < iters; ++t) {
      const int cur = t & 1, nxt = (t + 1) & 1;
      u.b_row_off = static_cast<int>(sched[t] * in);
      u.diag_in = F(L.Hdiag) + sched[t] * in;
      u.V_in = Vb[cur];
      u.V_out = Vb[nxt];
      u.alpha_in = ab[cur];
      u.alpha_out = ab[nxt];
      u.beta_in = bb[cur];
      u.beta_out = bb[nxt];
      u.D_hi = Dh[nxt];
      u.D_lo = P.split ? Dl[nxt] : nullptr;
      u.part_out = part[cur];
      u.part_in = t > 0 ? part[nxt] : nullptr;  // the previous step's partials
      u.rowloss = t > 0 ? rowloss + static_cast<int64_t>(t - 1) * out : nullptr;
      u.best_in = layer_best ? lb.thresh : best_cur;
      u.best_out = layer_best ? layer_scratch : best_next;
      AR_CUDA_TRY(ensure_block(sched[t]));
      if (fpt) {
        u.Cc_hi = H(L.Cc_hi) + sched[t] * static_cast<int64_t>(elems);
        u.Cc_lo = H(L.Cc_lo) + sched[t] * static_cast<int64_t>(elems);
        u.e_row = F(L.e) + sched[t] * out;
      }
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[3 * t], st));
      if (fault == kFaultLaunch) return AR_ECUDA;
      AR_CUDA_TRY(launch_gemm(upd_kind, P.bn_upd, m[cur], u, sms, st));
      AR_CUDA_TRY(finish_groups());
      AR_CUDA_TRY(judge_layer(part[cur], P.nparts_upd));  // this step's loss, judged by the next launch
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[3 * t + 1], st));
      ++launches;
      if (t > 0) std::swap(best_cur, best_next);
    }
    if (iters > 0) {
      const int last = (iters - 1) & 1;
      FinalizeBestArgs f;
      f.part = part[last];
      f.nparts = static_cast<int>(P.nparts_upd);
      f.out = out;
      f.in = in;
      f.G = static_cast<int>(P.G);
      f.inv_batch = 1.0f / static_cast<float>(B);
      f.keep_best = p->keep_best != 0;
      f.best_in = layer_best ? lb.thresh : best_cur;  // the last step's decision, taken after its launch
      f.best_out = layer_best ? layer_scratch : best_next;
      f.rowloss = rowloss + static_cast<int64_t>(iters - 1) * out;
      f.V_last = Vb[last];
      f.alpha_last = ab[last];
      f.beta_last = bb[last];
      f.V_best = V_best;
      f.alpha_best = alpha_best;
      f.beta_best = beta_best;
      AR_CUDA_TRY(launch_finalize_best(f, st));
      ++launches;
      std::swap(best_cur, best_next);
      live = iters & 1;
    }
  } else if (iters > 0) {
    // ---------------------------------------------------------- direct form
    __nv_bfloat16* Rh = H(L.Rt_hi);
    __nv_bfloat16* Rl = H(L.Rt_lo);
    GemmMaps mr{}, mu{};
    // Pair tiles (as for the Gram step): each CTA stages half of a tile's B rows.
    const uint32_t res_box = P.pair_direct ? P.bn_res / 2 : P.bn_res;
    AR_CUDA_TRY(make_tmap_bf16(&mr.a0, D_hi, out, in, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&mr.a1, D_lo, out, in, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&mr.b0, X, n_rows, in, res_box));
    mr.b1 = mr.b0;
    AR_CUDA_TRY(make_tmap_bf16(&mu.a0, Rh, out, B, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&mu.a1, Rl, out, B, kBM));
    // mu.b0 (X_b^T, read MN-major from block b of X) is made per step.

    GemmArgs r;  // residual: R^T = D X_b^T, (D_hi + D_lo) X_b^T
    fill_grid(r, out, B, in, P.bn_res, nseg_d, P.pair_direct);
    r.raster_m = P.raster_upd;
    r.seg_a[1] = 1;
    r.fused = (P.fused_direct && nseg_d > 1) ? 1 : 0;
    r.timeout_ns = timeout_ns;
    r.status = status;
    r.C_hi = Rh;
    r.C_lo = P.split ? Rl : nullptr;
    r.ldc = B;
    r.part = part[0];
    r.part_ld = static_cast<int>(P.nparts_res);
    if (checks) r.chk_c = out * B;
    if (fpt) r.ldc_add = n_rows;  // + E_b^T: block b's columns of E

    fill_grid(u, out, in, B, P.bn_upd, nseg_d, P.pair_direct);  // update: G = (R_hi + R_lo)^T X_b
    u.raster_m = P.raster_upd;
    u.seg_a[1] = 1;
    u.b_mn = 1;
    u.fused = r.fused;
    u.V_in = Vb[0];
    u.V_out = Vb[0];
    u.alpha_in = ab[0];
    u.alpha_out = ab[0];
    u.beta_in = bb[0];
    u.beta_out = bb[0];
    u.part_in = part[0];
    u.nparts = static_cast<int>(P.nparts_res);
    u.snap_prev = 0;
    u.part_out = nullptr;
    for (int t = 0; t < iters; ++t) {
      const int64_t b0 = sched[t] * B;
      r.b_row_off = static_cast<int>(b0);
      AR_CUDA_TRY(ensure_block(sched[t]));
      if (fpt) {
        r.C_add = H(L.E_hi) + b0;
        r.C_add_lo = H(L.E_lo) + b0;
      }
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[3 * t], st));
      if (fault == kFaultLaunch) return AR_ECUDA;
      AR_CUDA_TRY(launch_gemm(kEpiStore, P.bn_res, mr, r, sms, st));
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[3 * t + 1], st));
      AR_CUDA_TRY(judge_layer(part[0], P.nparts_res));  // this step's loss, judged by its update
      AR_CUDA_TRY(make_tmap_bf16(&mu.b0, X + b0 * in, B, in, 64));
      mu.b1 = mu.b0;
      u.best_in = layer_best ? lb.thresh : best_cur;
      u.best_out = layer_best ? layer_scratch : best_next;
      u.rowloss = rowloss + static_cast<int64_t>(t) * out;
      AR_CUDA_TRY(launch_gemm(upd_kind, P.bn_upd, mu, u, sms, st));
      AR_CUDA_TRY(finish_groups());
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[3 * t + 2], st));
      launches += 2;
      std::swap(best_cur, best_next);
    }
  }

  if (iters > 0) {
    if (p->keep_best == AR_KEEP_BEST_ROW && best_cur != best_loss)
      AR_CUDA_TRY(cudaMemcpyAsync(best_loss, best_cur, static_cast<size_t>(out) * 4, cudaMemcpyDeviceToDevice, st));
    if (live != 0) {  // hand the live state back in buffer 0
      AR_CUDA_TRY(cudaMemcpyAsync(Vb[0], Vb[live], elems * 4, cudaMemcpyDeviceToDevice, st));
      AR_CUDA_TRY(cudaMemcpyAsync(ab[0], ab[live], groups * 4, cudaMemcpyDeviceToDevice, st));
      AR_CUDA_TRY(cudaMemcpyAsync(bb[0], bb[live], groups * 4, cudaMemcpyDeviceToDevice, st));
    }
    if (loss_trace) {
      AR_CUDA_TRY(launch_loss_trace(rowloss, out, iters, B, loss_trace, st));
      ++launches;
    }
  }

  // Codes, scales and zero-points of the applied state, and its D for the MSE.
  GroupQuantArgs fin;
  fin.W = W;
  fin.w_bf16 = w_dtype == AR_BF16;
  fin.out = out;
  fin.in = in;
  fin.g = static_cast<int>(P.g);
  fin.G = static_cast<int>(P.G);
  fin.bits = p->bits;
  fin.sym = p->sym != 0;
  fin.wmin_in = wmin;
  fin.wmax_in = wmax;
  fin.V = p->keep_best ? V_best : Vb[0];
  fin.alpha = p->keep_best ? alpha_best : ab[0];
  fin.beta = p->keep_best ? beta_best : bb[0];
  fin.codes = codes;
  fin.scale = scale;
  fin.zp = zp;
  fin.D_hi = final_mse ? D_hi : nullptr;
  fin.D_lo = final_mse && P.split ? D_lo : nullptr;
  if (checks) {
    fin.chk_elems = static_cast<int64_t>(elems);
    fin.chk_groups = static_cast<int64_t>(groups);
    fin.status = status;
  }
  AR_CUDA_TRY(launch_group_quant(fin, st));
  ++launches;

  if (final_mse) {
    GemmMaps m{};
    GemmArgs f;
    f.timeout_ns = timeout_ns;
    f.status = status;
    f.part = part[0];
    if (gram) {
      // sum_j D_j (sum_b H_b) D_j^T over all calibration rows
      for (int64_t b = 0; b < P.nb; ++b) AR_CUDA_TRY(ensure_block(b));
      AR_CUDA_TRY(launch_gram_sum(H(L.H_hi), P.split ? H(L.H_lo) : nullptr, static_cast<int>(P.nb),
                                  in * in, H(L.Hs_hi), P.split ? H(L.Hs_lo) : nullptr, st));
      AR_CUDA_TRY(launch_diag_sum(F(L.Hdiag), static_cast<int>(P.nb), in, F(L.Hdsum), st));
      launches += 1;
      AR_CUDA_TRY(make_tmap_bf16(&m.a0, D_hi, out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m.a1, D_lo, out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m.b0, H(L.Hs_hi), in, in, P.bn_fin));
      AR_CUDA_TRY(make_tmap_bf16(&m.b1, H(L.Hs_lo), in, in, P.bn_fin));
      fill_grid(f, out, in, in, P.bn_fin, nseg_g);
      f.seg_a[1] = 1;
      f.seg_b[2] = 1;
      f.Dd_hi = D_hi;
      f.Dd_lo = P.split ? D_lo : nullptr;
      f.diag_in = F(L.Hdsum);
      if (fpt) {
        f.Cs = F(L.Cs);
        f.e_row = F(L.es);
      }
      f.part_ld = f.num_n_blk * kEpiHalves;
      AR_CUDA_TRY(launch_gemm(kEpiDotD, P.bn_fin, m, f, sms, st));
      launches += 2;
    } else {
      for (int64_t b = 0; b < P.nb; ++b) AR_CUDA_TRY(fpt ? ensure_block(b) : wait_block(b));
      if (fpt) {  // mean((X D^T + E)^2) = mean((X W'^T - X_target W^T)^2)
        f.C_add = H(L.E_hi);
        f.C_add_lo = H(L.E_lo);
        f.ldc_add = n_rows;
      }
      AR_CUDA_TRY(make_tmap_bf16(&m.a0, D_hi, out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m.a1, D_lo, out, in, kBM));
      AR_CUDA_TRY(make_tmap_bf16(&m.b0, X, n_rows, in, P.bn_fin));
      m.b1 = m.b0;
      fill_grid(f, out, n_rows, in, P.bn_fin, nseg_d);
      f.seg_a[1] = 1;
      f.fused = (P.fused_direct && nseg_d > 1) ? 1 : 0;
      f.part_ld = f.num_n_blk * kEpiHalves;
      AR_CUDA_TRY(launch_gemm(kEpiSumSq, P.bn_fin, m, f, sms, st));
      ++launches;
    }
    AR_CUDA_TRY(launch_sum_to_double(part[0], out * f.part_ld, static_cast<double>(n_rows) * out, final_mse, st));
    ++launches;
  }
  if (timer) {
    AR_CUDA_TRY(cudaEventRecord(timer->stop, st));
    timer->launches = launches;
  }
  return AR_OK;
}

}  // namespace
}  // namespace ar

using namespace ar;

extern "C" {

const char* ar_version(void) { return "ar 0.4.0 sm_100a"; }

const char* ar_status_string(ar_status s) {
  switch (s) {
    case AR_OK:
      return "AR_OK";
    case AR_EINVAL:
      return "AR_EINVAL: invalid argument";
    case AR_EUNSUPPORTED:
      return "AR_EUNSUPPORTED: shape or option not supported";
    case AR_ENOMEM:
      return "AR_ENOMEM: workspace too small";
    case AR_ECUDA:
      return "AR_ECUDA: CUDA error";
    case AR_ETIMEOUT:
      return "AR_ETIMEOUT: device wait timed out";
    case AR_ECHECK:
      return "AR_ECHECK: a device-side bounds check refused a store (AR_CHECKS)";
  }
  return "unknown ar_status";
}

ar_status ar_rtn(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, int32_t bits, int32_t group_size,
                 int32_t sym, uint8_t* codes, float* scale, int32_t* zp, void* stream) {
  return ar_fake_quant(W, w_dtype, out, in, nullptr, nullptr, nullptr, bits, group_size, sym, codes, scale, zp,
                       nullptr, stream);
}

ar_status ar_fake_quant(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const float* V,
                        const float* alpha, const float* beta, int32_t bits, int32_t group_size, int32_t sym,
                        uint8_t* codes, float* scale, int32_t* zp, float* Wq, void* stream) {
  if (injected_fault() == kFaultParam) return AR_EINVAL;
  if (!bits_ok(bits) || out < 0 || in < 0) return AR_EINVAL;
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!group_ok(in, group_size)) return AR_EINVAL;
  if (!W || !codes || !scale || !zp) return AR_EINVAL;
  GroupQuantArgs a;
  a.W = W;
  a.w_bf16 = w_dtype == AR_BF16;
  a.out = out;
  a.in = in;
  a.g = static_cast<int>(group_of(in, group_size));
  a.G = static_cast<int>(in / a.g);
  a.bits = bits;
  a.sym = sym != 0;
  a.V = V;
  a.alpha = alpha;
  a.beta = beta;
  a.codes = codes;
  a.scale = scale;
  a.zp = zp;
  a.Wq = Wq;
  return from_cuda(launch_group_quant(a, static_cast<cudaStream_t>(stream)));
}

ar_status ar_pack(const uint8_t* codes, int64_t rows, int64_t cols, int32_t bits, int32_t* packed, void* stream) {
  if (injected_fault() == kFaultParam) return AR_EINVAL;
  if (!bits_ok(bits) || rows < 0 || cols < 0) return AR_EINVAL;
  if ((cols * bits) % 32 != 0) return AR_EINVAL;
  if (rows == 0 || cols == 0) return AR_OK;
  if (!codes || !packed) return AR_EINVAL;
  return from_cuda(launch_pack(codes, rows, cols, bits, packed, static_cast<cudaStream_t>(stream)));
}

size_t ar_tune_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, const ar_tune_params* p) {
  if (check_tune_args(out, in, n_rows, p) != AR_OK) return 0;
  if (out == 0 || in == 0) return 256;
  return make_layout(make_plan(out, in, n_rows, p)).total;
}

ar_status ar_tune_layer(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X,
                        int64_t n_rows, const ar_tune_params* p, ar_tune_state* state, void* workspace,
                        size_t ws_bytes, uint8_t* codes, float* scale, int32_t* zp, float* loss_trace,
                        double* final_mse, void* stream) {
  return tune_impl(W, w_dtype, out, in, X, n_rows, p, state, workspace, ws_bytes, codes, scale, zp, loss_trace,
                   final_mse, stream, nullptr);
}

ar_status ar_tune_layer_timed(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X,
                              int64_t n_rows, const ar_tune_params* p, ar_tune_state* state, void* workspace,
                              size_t ws_bytes, uint8_t* codes, float* scale, int32_t* zp, float* loss_trace,
                              double* final_mse, void* stream, ar_tune_timing* timing) {
  if (!timing || !p) return AR_EINVAL;
  memset(timing, 0, sizeof(*timing));
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  EventTimer timer;
  if (!timer.create(p->iters)) return AR_ECUDA;
  const ar_status s = tune_impl(W, w_dtype, out, in, X, n_rows, p, state, workspace, ws_bytes, codes, scale, zp,
                                loss_trace, final_mse, stream, &timer);
  if (s != AR_OK) return s;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AR_ECUDA;
  if (out == 0 || in == 0) return AR_OK;
  float ms = 0.f;
  for (int t = 0; t < p->iters; ++t) {
    if (cudaEventElapsedTime(&ms, timer.ev[3 * t], timer.ev[3 * t + 1]) != cudaSuccess) return AR_ECUDA;
    if (timer.algo == AR_ALGO_DIRECT) {
      timing->residual_ms += ms;
      if (cudaEventElapsedTime(&ms, timer.ev[3 * t + 1], timer.ev[3 * t + 2]) != cudaSuccess) return AR_ECUDA;
    }
    timing->update_ms += ms;
  }
  if (p->iters > 0) {
    if (cudaEventElapsedTime(&ms, timer.start, timer.ev[0]) != cudaSuccess) return AR_ECUDA;
    timing->setup_ms = ms;
  }
  if (cudaEventElapsedTime(&ms, timer.start, timer.stop) != cudaSuccess) return AR_ECUDA;
  timing->total_ms = ms;
  timing->gemm_launches = p->iters;
  timing->kernel_launches = timer.launches;
  timing->algo = timer.algo;
  return AR_OK;
}

ar_status ar_block_schedule(int64_t n_blocks, int64_t first, int64_t count, uint64_t seed, int64_t* blocks) {
  if (n_blocks < 1 || first < 0 || count < 0 || (count > 0 && !blocks)) return AR_EINVAL;
  const std::vector<int64_t> s = block_schedule(n_blocks, first, count, seed);
  for (int64_t i = 0; i < count; ++i) blocks[i] = s[static_cast<size_t>(i)];
  return AR_OK;
}

// ---------------------------------------------------------------------------
// ar_tune_layer_host: host buffers in and out, copies overlapped with the work.
// ---------------------------------------------------------------------------

namespace {

// Device workspace of the host entry point: the tuning workspace, then device
// copies of W, X and the outputs.
struct HostLayout {
  size_t tune, W, X, codes, scale, zp, trace, mse, total;
};

HostLayout make_host_layout(int64_t out, int64_t in, int64_t n_rows, ar_dtype w_dtype, const ar_tune_params* p) {
  HostLayout H{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 256);
    return o;
  };
  const int64_t G = in / group_of(in, p->group_size);
  H.tune = take(ar_tune_workspace_bytes(out, in, n_rows, p));
  H.W = take(static_cast<size_t>(out) * in * (w_dtype == AR_BF16 ? 2 : 4));
  H.X = take(static_cast<size_t>(n_rows) * in * 2);
  H.codes = take(static_cast<size_t>(out) * in);
  H.scale = take(static_cast<size_t>(out) * G * 4);
  H.zp = take(static_cast<size_t>(out) * G * 4);
  H.trace = take(static_cast<size_t>(std::max(p->iters, 1)) * 4);
  H.mse = take(8);
  H.total = off;
  return H;
}

// The copy stream and per-block events of one call; on every exit path the copies
// still in flight finish before the host buffers are handed back.
struct CopyPipeline {
  cudaStream_t copy = nullptr;
  cudaEvent_t start = nullptr, w_done = nullptr, all_done = nullptr;
  std::vector<cudaEvent_t> block;
  bool create(size_t nblocks) {
    if (cudaStreamCreateWithFlags(&copy, cudaStreamNonBlocking) != cudaSuccess) return false;
    for (cudaEvent_t* e : {&start, &w_done, &all_done})
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
    block.assign(nblocks, nullptr);
    for (auto& e : block)
      if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return false;
    return true;
  }
  ~CopyPipeline() {
    if (copy) {
      cudaStreamSynchronize(copy);
      cudaStreamDestroy(copy);
    }
    for (cudaEvent_t e : {start, w_done, all_done})
      if (e) cudaEventDestroy(e);
    for (cudaEvent_t e : block)
      if (e) cudaEventDestroy(e);
  }
};

}  // namespace

size_t ar_tune_host_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, ar_dtype w_dtype,
                                    const ar_tune_params* p) {
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return 0;
  if (ar_tune_workspace_bytes(out, in, n_rows, p) == 0) return 0;
  return make_host_layout(out, in, n_rows, w_dtype, p).total;
}

ar_status ar_tune_layer_host(const void* W_host, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X_host,
                             int64_t n_rows, const ar_tune_params* p, void* workspace, size_t ws_bytes,
                             uint8_t* codes_host, float* scale_host, int32_t* zp_host, float* loss_trace_host,
                             double* final_mse_host, void* stream) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!W_host || !X_host || !workspace || !codes_host || !scale_host || !zp_host) return AR_EINVAL;
  if (!aligned(workspace, 256)) return AR_EINVAL;
  const HostLayout HL = make_host_layout(out, in, n_rows, w_dtype, p);
  if (ws_bytes < HL.total) return AR_ENOMEM;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int64_t B = p->batch_rows;
  const int64_t nb = n_rows / B;
  const int64_t G = in / group_of(in, p->group_size);
  const size_t w_bytes = static_cast<size_t>(out) * in * (w_dtype == AR_BF16 ? 2 : 4);
  const size_t block_bytes = static_cast<size_t>(B) * in * 2;
  uint16_t* Xd = reinterpret_cast<uint16_t*>(ws + HL.X);

  if (injected_fault() == kFaultAlloc) return AR_ENOMEM;
  CopyPipeline cp;
  if (!cp.create(static_cast<size_t>(nb))) return AR_ECUDA;
  // Copies start after the work already queued on the caller's stream; blocks go
  // in the order the schedule first needs them.
  AR_CUDA_TRY(cudaEventRecord(cp.start, st));
  AR_CUDA_TRY(cudaStreamWaitEvent(cp.copy, cp.start, 0));
  AR_CUDA_TRY(cudaMemcpyAsync(ws + HL.W, W_host, w_bytes, cudaMemcpyHostToDevice, cp.copy));
  AR_CUDA_TRY(cudaEventRecord(cp.w_done, cp.copy));
  std::vector<char> queued(static_cast<size_t>(nb), 0);
  std::vector<int64_t> order;
  order.reserve(static_cast<size_t>(nb));
  for (int64_t b : block_schedule(nb, p->start_step, std::min<int64_t>(p->iters, nb), p->seed))
    if (!queued[b]) {
      queued[b] = 1;
      order.push_back(b);
    }
  for (int64_t b = 0; b < nb; ++b)
    if (!queued[b]) order.push_back(b);
  for (int64_t b : order) {
    AR_CUDA_TRY(cudaMemcpyAsync(Xd + b * B * in, X_host + b * B * in, block_bytes, cudaMemcpyHostToDevice,
                                cp.copy));
    AR_CUDA_TRY(cudaEventRecord(cp.block[b], cp.copy));
  }
  AR_CUDA_TRY(cudaEventRecord(cp.all_done, cp.copy));

  AR_CUDA_TRY(cudaStreamWaitEvent(st, cp.w_done, 0));
  uint8_t* codes = ws + HL.codes;
  float* scale = reinterpret_cast<float*>(ws + HL.scale);
  int32_t* zp = reinterpret_cast<int32_t*>(ws + HL.zp);
  float* trace = loss_trace_host ? reinterpret_cast<float*>(ws + HL.trace) : nullptr;
  double* mse = final_mse_host ? reinterpret_cast<double*>(ws + HL.mse) : nullptr;
  const ar_status s = tune_impl(ws + HL.W, w_dtype, out, in, Xd, n_rows, p, nullptr, ws + HL.tune,
                                HL.W - HL.tune, codes, scale, zp, trace, mse, stream, nullptr, cp.block.data());
  if (s != AR_OK) return s;
  AR_CUDA_TRY(cudaStreamWaitEvent(st, cp.all_done, 0));
  AR_CUDA_TRY(cudaMemcpyAsync(codes_host, codes, static_cast<size_t>(out) * in, cudaMemcpyDeviceToHost, st));
  AR_CUDA_TRY(cudaMemcpyAsync(scale_host, scale, static_cast<size_t>(out) * G * 4, cudaMemcpyDeviceToHost, st));
  AR_CUDA_TRY(cudaMemcpyAsync(zp_host, zp, static_cast<size_t>(out) * G * 4, cudaMemcpyDeviceToHost, st));
  if (trace && p->iters > 0)
    AR_CUDA_TRY(cudaMemcpyAsync(loss_trace_host, trace, static_cast<size_t>(p->iters) * 4, cudaMemcpyDeviceToHost,
                                st));
  if (mse) AR_CUDA_TRY(cudaMemcpyAsync(final_mse_host, mse, 8, cudaMemcpyDeviceToHost, st));
  return ar_tune_status(ws + HL.tune, stream);
}

size_t ar_tune_fp_target_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, ar_dtype w_dtype,
                                         const ar_tune_params* p) {
  if (check_tune_args(out, in, n_rows, p) != AR_OK) return 0;
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return 0;
  if (out == 0 || in == 0) return 256;
  const Plan P = make_plan(out, in, n_rows, p, true, w_dtype == AR_F32);
  const size_t total = make_layout(P).total;
  return (P.algo == AR_ALGO_GRAM && total > kFpTargetMaxBytes) ? 0 : total;
}

ar_status ar_tune_layer_fp_target(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X,
                                  const uint16_t* X_target, int64_t n_rows, const ar_tune_params* p,
                                  ar_tune_state* state, void* workspace, size_t ws_bytes, uint8_t* codes,
                                  float* scale, int32_t* zp, float* loss_trace, double* final_mse, void* stream) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (out == 0 || in == 0) return AR_OK;
  if (!X_target) return AR_EINVAL;
  return tune_impl(W, w_dtype, out, in, X, n_rows, p, state, workspace, ws_bytes, codes, scale, zp, loss_trace,
                   final_mse, stream, nullptr, nullptr, X_target);
}

ar_status ar_tune_status(const void* workspace, void* stream) {
  if (!workspace) return AR_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AR_ECUDA;
  int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return AR_ECUDA;
  if (word == kDevOk) return AR_OK;
  if (word == kDevTimeout) return AR_ETIMEOUT;
  if (word == kDevCheck) return AR_ECHECK;
  return AR_ECUDA;
}

ar_status ar_tune_row_losses(const void* workspace, size_t ws_bytes, int64_t out, int64_t in, int64_t n_rows,
                             const ar_tune_params* p, float* row_loss, void* stream) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (out == 0 || in == 0 || p->iters == 0) return AR_OK;
  if (!workspace || !row_loss) return AR_EINVAL;
  const Layout L = make_layout(make_plan(out, in, n_rows, p));
  if (ws_bytes < L.total) return AR_ENOMEM;
  const size_t bytes = static_cast<size_t>(out) * static_cast<size_t>(p->iters) * sizeof(float);
  return from_cuda(cudaMemcpyAsync(row_loss, static_cast<const uint8_t*>(workspace) + L.rowloss, bytes,
                                   cudaMemcpyDefault, static_cast<cudaStream_t>(stream)));
}

ar_status ar_selftest_division(const float* a, int64_t na, const float* b, int64_t nb, uint64_t* mismatches,
                               float* first_bad, void* stream) {
  if ((na > 0 && !a) || (nb > 0 && !b) || !mismatches || !first_bad || na < 0 || nb < 0) return AR_EINVAL;
  return from_cuda(launch_division_selftest(a, na, b, nb, reinterpret_cast<unsigned long long*>(mismatches),
                                            first_bad, static_cast<cudaStream_t>(stream)));
}

ar_status ar_selftest_timeout(int32_t* status, uint64_t timeout_ns, void* stream) {
  if (!status) return AR_EINVAL;
  return from_cuda(launch_timeout_selftest(status, timeout_ns, static_cast<cudaStream_t>(stream)));
}

ar_status ar_dequant(const uint8_t* codes, const float* scale, const int32_t* zp, int64_t out, int64_t in,
                     int32_t group_size, uint16_t* Wq_hi, uint16_t* Wq_lo, float* Wq, void* stream) {
  if (out < 0 || in < 0) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!group_ok(in, group_size) || !codes || !scale || !zp || !Wq_hi) return AR_EINVAL;
  return from_cuda(launch_dequant(codes, scale, zp, out, in, static_cast<int>(group_of(in, group_size)),
                                  reinterpret_cast<__nv_bfloat16*>(Wq_hi), reinterpret_cast<__nv_bfloat16*>(Wq_lo),
                                  Wq, static_cast<cudaStream_t>(stream)));
}

// Where ar_linear's bounded waits report when the caller passes no status word.
static __device__ int g_linear_status;

ar_status ar_linear(const uint16_t* X, int64_t n, int64_t in, const uint16_t* Wq_hi, const uint16_t* Wq_lo,
                    int64_t out, const uint16_t* add, uint16_t* Y, int32_t* status, void* stream) {
  if (n < 0 || in <= 0 || out <= 0 || in % 8 != 0 || out % 8 != 0) return AR_EINVAL;
  if (n >= (1ll << 31) || in >= (1ll << 31) || out >= (1ll << 31)) return AR_EUNSUPPORTED;
  if (n == 0) return AR_OK;
  if (!X || !Wq_hi || !Y || !aligned(X, 16) || !aligned(Wq_hi, 16) || !aligned(Y, 16)) return AR_EINVAL;
  if ((Wq_lo && !aligned(Wq_lo, 16)) || (add && !aligned(add, 16))) return AR_EINVAL;
  int dev = 0, sms = 0, major = 0;
  AR_CUDA_TRY(cudaGetDevice(&dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  if (major != 10) return AR_EUNSUPPORTED;
  const int bn = 256;
  GemmMaps m{};
  AR_CUDA_TRY(make_tmap_bf16(&m.a0, X, n, in, kBM));
  AR_CUDA_TRY(make_tmap_bf16(&m.b0, Wq_hi, out, in, bn));
  m.a1 = m.a0;
  if (Wq_lo)
    AR_CUDA_TRY(make_tmap_bf16(&m.b1, Wq_lo, out, in, bn));
  else
    m.b1 = m.b0;
  GemmArgs a;
  fill_grid(a, n, out, in, bn, Wq_lo ? 2 : 1);
  a.seg_b[1] = 1;  // X Wq_hi^T + X Wq_lo^T
  a.C_hi = reinterpret_cast<__nv_bfloat16*>(Y);
  a.C_add = reinterpret_cast<const __nv_bfloat16*>(add);
  a.ldc = out;
  if (!status) AR_CUDA_TRY(cudaGetSymbolAddress(reinterpret_cast<void**>(&status), g_linear_status));
  a.status = status;
  return from_cuda(launch_gemm(kEpiStore, bn, m, a, sms, static_cast<cudaStream_t>(stream)));
}

ar_status ar_silu_mul(const uint16_t* a, const uint16_t* b, int64_t count, uint16_t* y, void* stream) {
  if (count < 0) return AR_EINVAL;
  if (count == 0) return AR_OK;
  if (!a || !b || !y) return AR_EINVAL;
  return from_cuda(launch_silu_mul(reinterpret_cast<const __nv_bfloat16*>(a), reinterpret_cast<const __nv_bfloat16*>(b),
                                   count, reinterpret_cast<__nv_bfloat16*>(y), static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------------------
// ar_tune_layer_static: tuning without any device-memory allocation.
//
// The scratch lives in one fixed array in device memory, created when the
// library's device code is loaded on a GPU and held until the process exits.  In
// host code `g_static_scratch` names a host-side stand-in, not the device array,
// so its device address is looked up (cudaGetSymbolAddress) once per device, with
// that device current, on the first call there, and cached together with the id
// of the CUDA context it belongs to.  A call that finds another context current
// (after cudaDeviceReset, or a context the caller pushed) looks it up again.
// ---------------------------------------------------------------------------

static __device__ __align__(256) uint8_t g_static_scratch[AR_STATIC_SCRATCH_BYTES];

namespace {

struct StaticScratch {
  void* ptr = nullptr;
  unsigned long long ctx_id = 0;
};

std::mutex g_static_mu;
StaticScratch g_static[256];

// Id of the current CUDA context (driver entry points fetched through the runtime,
// as for the tensor maps).  False if there is none or the driver lacks the call.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

}  // namespace

size_t ar_static_scratch_bytes(void) { return AR_STATIC_SCRATCH_BYTES; }

ar_status ar_tune_layer_static(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X,
                               int64_t n_rows, const ar_tune_params* p, uint8_t* codes, float* scale, int32_t* zp,
                               float* loss_trace, double* final_mse, void* stream) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (out == 0 || in == 0) return AR_OK;
  if (make_layout(make_plan(out, in, n_rows, p)).total > AR_STATIC_SCRATCH_BYTES) return AR_ENOMEM;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return AR_ECUDA;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_static_mu);
    unsigned long long ctx = 0;
    const bool have_ctx = current_context_id(&ctx);
    StaticScratch& e = g_static[dev];
    if (!e.ptr || !have_ctx || e.ctx_id != ctx) {
      void* ptr = nullptr;
      if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return AR_ECUDA;
      // The lookup makes the device's context current if none was; without a
      // context id the address is looked up on every call.
      unsigned long long now = 0;
      const bool have_now = current_context_id(&now);
      e.ptr = have_now ? ptr : nullptr;
      e.ctx_id = now;
      scratch = ptr;
    } else {
      scratch = e.ptr;
    }
  }
  return tune_impl(W, w_dtype, out, in, X, n_rows, p, nullptr, scratch, AR_STATIC_SCRATCH_BYTES, codes, scale, zp,
                   loss_trace, final_mse, stream, nullptr);
}

}  // extern "C"
