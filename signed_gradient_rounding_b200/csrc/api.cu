// libar C ABI: argument validation, workspace layout, the calibration-block
// schedule and the launch sequence of the tuning loop.
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "../../include/ar.h"
#include "ar_device.cuh"
#include "ar_internal.h"

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

// ---------------------------------------------------------------------------
// Calibration-block schedule.  The pages iterate over calibration batches without
// saying how one is picked per step; this library visits the n/B blocks once per
// epoch in the order of a Durstenfeld (Fisher-Yates) shuffle of the identity,
// each swap index being x mod (i + 1) for the next output x of one SplitMix64
// stream (Steele, Lea & Flood, OOPSLA 2014) seeded with `seed` and continued
// across epochs.  A single block draws nothing.
// ---------------------------------------------------------------------------

namespace {

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

// Workspace layout of ar_tune_layer (offsets in bytes from the workspace base).
struct Layout {
  size_t status, Xt, Rt, D, V, alpha, beta, V_best, alpha_best, beta_best, best_loss, best_alt, wmin, wmax, part,
      rowloss, total;
};

Layout make_layout(int64_t out, int64_t in, int64_t n, int64_t B, int64_t G, int64_t iters) {
  Layout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = round_up(off + bytes, 1024);
    return o;
  };
  const int64_t nparts = std::max(cdiv(B, kBN), cdiv(n, kBN));
  L.status = take(256);
  L.Xt = take(static_cast<size_t>(in) * n * 2);
  L.Rt = take(static_cast<size_t>(out) * B * 2);
  L.D = take(static_cast<size_t>(out) * in * 2);
  L.V = take(static_cast<size_t>(out) * in * 4);
  L.alpha = take(static_cast<size_t>(out) * G * 4);
  L.beta = take(static_cast<size_t>(out) * G * 4);
  L.V_best = take(static_cast<size_t>(out) * in * 4);
  L.alpha_best = take(static_cast<size_t>(out) * G * 4);
  L.beta_best = take(static_cast<size_t>(out) * G * 4);
  L.best_loss = take(static_cast<size_t>(out) * 4);
  L.best_alt = take(static_cast<size_t>(out) * 4);
  L.wmin = take(static_cast<size_t>(out) * G * 4);
  L.wmax = take(static_cast<size_t>(out) * G * 4);
  L.part = take(static_cast<size_t>(out) * nparts * 4);
  L.rowloss = take(static_cast<size_t>(out) * std::max<int64_t>(iters, 1) * 4);
  L.total = off;
  return L;
}

ar_status from_cuda(cudaError_t e) { return e == cudaSuccess ? AR_OK : AR_ECUDA; }

#define AR_CUDA_TRY(expr)                          \
  do {                                             \
    cudaError_t e_ = (expr);                       \
    if (e_ != cudaSuccess) return AR_ECUDA;        \
  } while (0)

bool tune_shape_supported(int64_t in, int64_t g, int64_t B) {
  if (in % 32 != 0 || B % 8 != 0) return false;
  if (g % 32 != 0) return false;
  return (kBN % g == 0) || (g == in && in <= kBN);
}

ar_status check_tune_args(int64_t out, int64_t in, int64_t n_rows, const ar_tune_params* p) {
  if (!p || out < 0 || in < 0 || n_rows < 0) return AR_EINVAL;
  if (!bits_ok(p->bits)) return AR_EINVAL;
  if (p->iters < 0 || !(p->lr >= 0.0f) || !isfinite(p->lr) || !isfinite(p->minmax_lr)) return AR_EINVAL;
  if (!(p->minmax_shrink > 0.0f) || !isfinite(p->minmax_shrink)) return AR_EINVAL;
  if (p->start_step < 0) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!group_ok(in, p->group_size)) return AR_EINVAL;
  if (p->batch_rows <= 0 || n_rows < p->batch_rows || n_rows % p->batch_rows != 0) return AR_EINVAL;
  if (out >= (1ll << 31) || in >= (1ll << 31) || n_rows >= (1ll << 31)) return AR_EUNSUPPORTED;
  if (!tune_shape_supported(in, group_of(in, p->group_size), p->batch_rows)) return AR_EUNSUPPORTED;
  return AR_OK;
}

}  // namespace
}  // namespace ar

using namespace ar;

extern "C" {

const char* ar_version(void) { return "ar 0.1.0 sm_100a"; }

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
  if (!bits_ok(bits) || rows < 0 || cols < 0) return AR_EINVAL;
  if ((cols * bits) % 32 != 0) return AR_EINVAL;
  if (rows == 0 || cols == 0) return AR_OK;
  if (!codes || !packed) return AR_EINVAL;
  return from_cuda(launch_pack(codes, rows, cols, bits, packed, static_cast<cudaStream_t>(stream)));
}

size_t ar_tune_workspace_bytes(int64_t out, int64_t in, int64_t n_rows, const ar_tune_params* p) {
  if (check_tune_args(out, in, n_rows, p) != AR_OK) return 0;
  if (out == 0 || in == 0) return 256;
  const int64_t g = group_of(in, p->group_size);
  return make_layout(out, in, n_rows, p->batch_rows, in / g, p->iters).total;
}

}  // extern "C"

namespace ar {
namespace {

// Events around the contractions of a timed call: ev[2t] before the residual
// GEMM of step t, ev[2t+1] between the two GEMMs, ev[2t+2] after the update GEMM.
struct EventTimer {
  std::vector<cudaEvent_t> ev;
  cudaEvent_t start = nullptr, stop = nullptr;
  int launches = 0;
  bool create(int iters) {
    ev.assign(static_cast<size_t>(2 * iters + 1), nullptr);
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

ar_status tune_impl(const void* W, ar_dtype w_dtype, int64_t out, int64_t in, const uint16_t* X, int64_t n_rows,
                    const ar_tune_params* p, ar_tune_state* state, void* workspace, size_t ws_bytes,
                    uint8_t* codes, float* scale, int32_t* zp, float* loss_trace, double* final_mse,
                    void* stream, EventTimer* timer) {
  const ar_status chk = check_tune_args(out, in, n_rows, p);
  if (chk != AR_OK) return chk;
  if (w_dtype != AR_F32 && w_dtype != AR_BF16) return AR_EINVAL;
  if (out == 0 || in == 0) return AR_OK;
  if (!W || !X || !workspace || !codes || !scale || !zp) return AR_EINVAL;
  if (!aligned(W, 16) || !aligned(X, 16) || !aligned(workspace, 256)) return AR_EINVAL;
  if (state) {
    const void* ptrs[7] = {state->V, state->alpha, state->beta, state->best_loss,
                           state->V_best, state->alpha_best, state->beta_best};
    for (const void* q : ptrs)
      if (!q || !aligned(q, 16)) return AR_EINVAL;
  }

  const int64_t B = p->batch_rows;
  const int64_t g = group_of(in, p->group_size);
  const int64_t G = in / g;
  const int iters = p->iters;
  const Layout L = make_layout(out, in, n_rows, B, G, iters);
  if (ws_bytes < L.total) return AR_ENOMEM;

  int dev = 0, sms = 0, major = 0;
  AR_CUDA_TRY(cudaGetDevice(&dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  AR_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  if (major != 10) return AR_EUNSUPPORTED;

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + L.status);
  uint16_t* Xt = reinterpret_cast<uint16_t*>(ws + L.Xt);
  __nv_bfloat16* Rt = reinterpret_cast<__nv_bfloat16*>(ws + L.Rt);
  __nv_bfloat16* D = reinterpret_cast<__nv_bfloat16*>(ws + L.D);
  float* wmin = reinterpret_cast<float*>(ws + L.wmin);
  float* wmax = reinterpret_cast<float*>(ws + L.wmax);
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* rowloss = reinterpret_cast<float*>(ws + L.rowloss);
  float* best_alt = reinterpret_cast<float*>(ws + L.best_alt);
  float *V, *alpha, *beta, *best_loss, *V_best, *alpha_best, *beta_best;
  if (state) {
    V = state->V;
    alpha = state->alpha;
    beta = state->beta;
    best_loss = state->best_loss;
    V_best = state->V_best;
    alpha_best = state->alpha_best;
    beta_best = state->beta_best;
  } else {
    V = reinterpret_cast<float*>(ws + L.V);
    alpha = reinterpret_cast<float*>(ws + L.alpha);
    beta = reinterpret_cast<float*>(ws + L.beta);
    best_loss = reinterpret_cast<float*>(ws + L.best_loss);
    V_best = reinterpret_cast<float*>(ws + L.V_best);
    alpha_best = reinterpret_cast<float*>(ws + L.alpha_best);
    beta_best = reinterpret_cast<float*>(ws + L.beta_best);
  }
  const bool init_state = !state || !state->initialized;
  const size_t elems = static_cast<size_t>(out) * in;
  const size_t groups = static_cast<size_t>(out) * G;

  int launches = 0;
  if (timer) AR_CUDA_TRY(cudaEventRecord(timer->start, st));
  AR_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  if (init_state) {
    AR_CUDA_TRY(cudaMemsetAsync(V, 0, elems * 4, st));
    AR_CUDA_TRY(cudaMemsetAsync(V_best, 0, elems * 4, st));
    AR_CUDA_TRY(launch_fill_f32(alpha, groups, p->minmax_shrink, st));
    AR_CUDA_TRY(launch_fill_f32(beta, groups, p->minmax_shrink, st));
    AR_CUDA_TRY(launch_fill_f32(alpha_best, groups, p->minmax_shrink, st));
    AR_CUDA_TRY(launch_fill_f32(beta_best, groups, p->minmax_shrink, st));
    AR_CUDA_TRY(launch_fill_f32(best_loss, out, INFINITY, st));
    launches += 5;
  }

  // Group statistics of W and the first step's D = bf16(W' - W).
  GroupQuantArgs prep;
  prep.W = W;
  prep.w_bf16 = w_dtype == AR_BF16;
  prep.out = out;
  prep.in = in;
  prep.g = static_cast<int>(g);
  prep.G = static_cast<int>(G);
  prep.bits = p->bits;
  prep.sym = p->sym != 0;
  prep.wmin_out = wmin;
  prep.wmax_out = wmax;
  prep.V = V;
  prep.alpha = alpha;
  prep.beta = beta;
  prep.D = D;
  AR_CUDA_TRY(launch_group_quant(prep, st));
  ++launches;

  const uint64_t timeout_ns = 1000000000ull;
  const float mlr = p->minmax_lr < 0.0f ? p->lr : p->minmax_lr;
  const int64_t nparts = cdiv(B, kBN);

  if (iters > 0) {
    AR_CUDA_TRY(launch_transpose_bf16(X, n_rows, in, Xt, st));
    ++launches;
    CUtensorMap tmD, tmX, tmRt, tmXt;
    AR_CUDA_TRY(make_tmap_bf16(&tmD, D, out, in, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&tmX, X, n_rows, in, kBN));
    AR_CUDA_TRY(make_tmap_bf16(&tmRt, Rt, out, B, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&tmXt, Xt, in, n_rows, kBN));

    GemmArgs r;  // residual: R^T = D X_b^T
    r.M = static_cast<int>(out);
    r.N = static_cast<int>(B);
    r.K = static_cast<int>(in);
    r.num_m_blk = static_cast<int>(cdiv(out, kBM));
    r.num_n_blk = static_cast<int>(cdiv(B, kBN));
    r.num_k_blk = static_cast<int>(cdiv(in, kBK));
    r.num_tiles = r.num_m_blk * r.num_n_blk;
    r.timeout_ns = timeout_ns;
    r.status = status;
    r.Rt = Rt;
    r.ldr = B;
    r.part = part;
    r.part_ld = static_cast<int>(nparts);

    GemmArgs u;  // update: G = R^T X_b
    u.M = static_cast<int>(out);
    u.N = static_cast<int>(in);
    u.K = static_cast<int>(B);
    u.num_m_blk = static_cast<int>(cdiv(out, kBM));
    u.num_n_blk = static_cast<int>(cdiv(in, kBN));
    u.num_k_blk = static_cast<int>(cdiv(B, kBK));
    u.num_tiles = u.num_m_blk * u.num_n_blk;
    u.timeout_ns = timeout_ns;
    u.status = status;
    u.W = W;
    u.w_bf16 = w_dtype == AR_BF16;
    u.V = V;
    u.alpha = alpha;
    u.beta = beta;
    u.wmin = wmin;
    u.wmax = wmax;
    u.D = D;
    u.V_best = V_best;
    u.alpha_best = alpha_best;
    u.beta_best = beta_best;
    u.part_in = part;
    u.nparts = static_cast<int>(nparts);
    u.inv_batch = 1.0f / static_cast<float>(B);
    u.g = static_cast<int>(g);
    u.G = static_cast<int>(G);
    u.bits = p->bits;
    u.sym = p->sym != 0;
    u.keep_best = p->keep_best != 0;
    u.lr = p->lr;
    u.mlr = mlr;

    const std::vector<int64_t> sched = block_schedule(n_rows / B, p->start_step, iters, p->seed);
    float* best_cur = best_loss;
    float* best_next = best_alt;
    for (int t = 0; t < iters; ++t) {
      const int64_t b0 = sched[t] * B;
      r.b_row_off = static_cast<int>(b0);
      if (timer && t == 0) AR_CUDA_TRY(cudaEventRecord(timer->ev[0], st));
      AR_CUDA_TRY(launch_gemm(kEpiResidual, tmD, tmX, r, sms, st));
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[2 * t + 1], st));
      u.b_k_off = static_cast<int>(b0);
      u.best_in = best_cur;
      u.best_out = best_next;
      u.rowloss = rowloss + static_cast<int64_t>(t) * out;
      AR_CUDA_TRY(launch_gemm(kEpiUpdate, tmRt, tmXt, u, sms, st));
      if (timer) AR_CUDA_TRY(cudaEventRecord(timer->ev[2 * t + 2], st));
      launches += 2;
      std::swap(best_cur, best_next);
    }
    if (p->keep_best && best_cur != best_loss)
      AR_CUDA_TRY(cudaMemcpyAsync(best_loss, best_cur, static_cast<size_t>(out) * 4, cudaMemcpyDeviceToDevice, st));
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
  fin.g = static_cast<int>(g);
  fin.G = static_cast<int>(G);
  fin.bits = p->bits;
  fin.sym = p->sym != 0;
  fin.wmin_in = wmin;
  fin.wmax_in = wmax;
  fin.V = p->keep_best ? V_best : V;
  fin.alpha = p->keep_best ? alpha_best : alpha;
  fin.beta = p->keep_best ? beta_best : beta;
  fin.codes = codes;
  fin.scale = scale;
  fin.zp = zp;
  fin.D = final_mse ? D : nullptr;
  AR_CUDA_TRY(launch_group_quant(fin, st));
  ++launches;

  if (final_mse) {
    CUtensorMap tmD, tmX;
    AR_CUDA_TRY(make_tmap_bf16(&tmD, D, out, in, kBM));
    AR_CUDA_TRY(make_tmap_bf16(&tmX, X, n_rows, in, kBN));
    GemmArgs f;
    f.M = static_cast<int>(out);
    f.N = static_cast<int>(n_rows);
    f.K = static_cast<int>(in);
    f.num_m_blk = static_cast<int>(cdiv(out, kBM));
    f.num_n_blk = static_cast<int>(cdiv(n_rows, kBN));
    f.num_k_blk = static_cast<int>(cdiv(in, kBK));
    f.num_tiles = f.num_m_blk * f.num_n_blk;
    f.timeout_ns = timeout_ns;
    f.status = status;
    f.part = part;
    f.part_ld = f.num_n_blk;
    AR_CUDA_TRY(launch_gemm(kEpiLoss, tmD, tmX, f, sms, st));
    AR_CUDA_TRY(launch_sum_to_double(part, out * f.num_n_blk, static_cast<double>(n_rows) * out, final_mse, st));
    launches += 2;
  }
  if (timer) {
    AR_CUDA_TRY(cudaEventRecord(timer->stop, st));
    timer->launches = launches;
  }
  return AR_OK;
}

}  // namespace
}  // namespace ar

extern "C" {

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
    if (cudaEventElapsedTime(&ms, timer.ev[2 * t], timer.ev[2 * t + 1]) != cudaSuccess) return AR_ECUDA;
    timing->residual_ms += ms;
    if (cudaEventElapsedTime(&ms, timer.ev[2 * t + 1], timer.ev[2 * t + 2]) != cudaSuccess) return AR_ECUDA;
    timing->update_ms += ms;
  }
  if (cudaEventElapsedTime(&ms, timer.start, timer.stop) != cudaSuccess) return AR_ECUDA;
  timing->total_ms = ms;
  timing->gemm_launches = p->iters;
  timing->kernel_launches = timer.launches;
  return AR_OK;
}

ar_status ar_block_schedule(int64_t n_blocks, int64_t first, int64_t count, uint64_t seed, int64_t* blocks) {
  if (n_blocks < 1 || first < 0 || count < 0 || (count > 0 && !blocks)) return AR_EINVAL;
  const std::vector<int64_t> s = block_schedule(n_blocks, first, count, seed);
  for (int64_t i = 0; i < count; ++i) blocks[i] = s[static_cast<size_t>(i)];
  return AR_OK;
}

ar_status ar_tune_status(const void* workspace, void* stream) {
  if (!workspace) return AR_EINVAL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return AR_ECUDA;
  int word = 0;
  if (cudaMemcpy(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return AR_ECUDA;
  if (word == kDevOk) return AR_OK;
  if (word == kDevTimeout) return AR_ETIMEOUT;
  return AR_ECUDA;
}

ar_status ar_selftest_timeout(int32_t* status, uint64_t timeout_ns, void* stream) {
  if (!status) return AR_EINVAL;
  return from_cuda(launch_timeout_selftest(status, timeout_ns, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
