// Elementwise and reduction kernels of libar: group min-max statistics, scale and
// zero-point, offset fake-quantisation (RTN when V = 0, alpha = beta = 1), int32
// bit packing, and the fixed-order loss reductions.
#include <math.h>

#include "ar_device.cuh"
#include "ar_internal.h"
#include "ar_layer_best.h"

namespace ar {

namespace {

__device__ __forceinline__ float load_w(const void* W, int w_bf16, int64_t idx) {
  if (w_bf16) return bf16_bits_to_f32(static_cast<const uint16_t*>(W)[idx]);
  return static_cast<const float*>(W)[idx];
}

// Two fp32 values that are already bf16 values (exactly representable), as a bf16x2 word.
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// kVec consecutive weights as fp32 (kVec = 4: 8- or 16-byte aligned vector load).
template <int kVec>
__device__ __forceinline__ void load_wv(const void* W, int w_bf16, int64_t idx, float (&w)[kVec]) {
  if (kVec == 4) {
    if (w_bf16) {
      const uint2 x = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(W) + idx);
      w[0] = __uint_as_float(x.x << 16);
      w[1] = __uint_as_float(x.x & 0xFFFF0000u);
      w[2] = __uint_as_float(x.y << 16);
      w[3] = __uint_as_float(x.y & 0xFFFF0000u);
    } else {
      const float4 x = *reinterpret_cast<const float4*>(static_cast<const float*>(W) + idx);
      w[0] = x.x;
      w[1] = x.y;
      w[2] = x.z;
      w[3] = x.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < kVec; ++i) w[i] = load_w(W, w_bf16, idx + i);
  }
}

// One warp per group ("[llm-compressor] AutoRound ...", _fake_quantize_with_offset,
// min-max init).  Group j*G + gi covers W[j, gi*g : (gi+1)*g].  Each lane takes kVec
// consecutive weights at a time (kVec = 4 when every pointer is 16-byte aligned and
// in and g are multiples of 4, so the loads and stores are vectors; else 1).  The
// per-element arithmetic is the same either way.
template <int kVec>
__global__ void group_quant_kernel(GroupQuantArgs a) {
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= a.out * a.G) return;
  const int64_t row = warp / a.G;
  const int64_t col0 = (warp - row * a.G) * a.g;
  const int64_t base = row * a.in + col0;

  // Group statistics, and whether every weight of the group admits the fast
  // correctly rounded division by the group's scale (div_fast_ok).
  float mn = 0.0f, mx = 0.0f;  // min(0, min W), max(0, max W)
  bool ok = true;
  for (int k = lane * kVec; k < a.g; k += 32 * kVec) {
    float w[kVec];
    load_wv<kVec>(a.W, a.w_bf16, base + k, w);
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      mn = fminf(mn, w[i]);
      mx = fmaxf(mx, w[i]);
      ok = ok && div_fast_ok(w[i]);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const bool fast = __all_sync(0xffffffffu, ok);
  if (!fast && lane == 0 && a.div_slow) atomicAdd(a.div_slow, 1);
  float wmin = mn, wmax = mx;
  if (a.wmin_in) {
    wmin = a.wmin_in[warp];
    wmax = a.wmax_in[warp];
  }
  const float alpha = a.alpha ? a.alpha[warp] : 1.0f;
  const float beta = a.beta ? a.beta[warp] : 1.0f;
  const GroupScale gs = group_scale(wmin, wmax, alpha, beta, a.bits, a.sym != 0);
  if (lane == 0 && in_bounds(warp, 1, a.chk_groups, a.status)) {
    if (a.wmin_out) {
      a.wmin_out[warp] = wmin;
      a.wmax_out[warp] = wmax;
    }
    if (a.scale) a.scale[warp] = gs.s;
    if (a.zp) a.zp[warp] = static_cast<int32_t>(gs.zp);
  }
  if (!a.codes && !a.Wq && !a.D_hi) return;
  const float Q = qmaxf(a.bits);
  for (int k = lane * kVec; k < a.g; k += 32 * kVec) {
    const int64_t e0 = base + k;
    float w[kVec], v[kVec];
    load_wv<kVec>(a.W, a.w_bf16, e0, w);
    if (!a.V) {
#pragma unroll
      for (int i = 0; i < kVec; ++i) v[i] = 0.0f;
    } else if (kVec == 4) {
      const float4 x = *reinterpret_cast<const float4*>(a.V + e0);
      v[0] = x.x;
      v[1] = x.y;
      v[2] = x.z;
      v[3] = x.w;
    } else {
#pragma unroll
      for (int i = 0; i < kVec; ++i) v[i] = a.V[e0 + i];
    }
    float q[kVec], wq[kVec], dh[kVec], dl[kVec];
#pragma unroll
    for (int i = 0; i < kVec; ++i) {
      const ElemQuant e = quant_elem(w[i], v[i], gs, Q, fast);
      q[i] = e.q;
      wq[i] = e.wq;
      const float d = __fsub_rn(e.wq, w[i]);
      const __nv_bfloat16 hi = __float2bfloat16_rn(d);
      dh[i] = __bfloat162float(hi);
      dl[i] = __fsub_rn(d, dh[i]);
    }
    if (!in_bounds(e0, kVec, a.chk_elems, a.status)) continue;
    if (kVec == 4) {
      if (a.codes)
        *reinterpret_cast<uint32_t*>(a.codes + e0) =
            static_cast<uint32_t>(q[0]) | (static_cast<uint32_t>(q[1]) << 8) |
            (static_cast<uint32_t>(q[2]) << 16) | (static_cast<uint32_t>(q[3]) << 24);
      if (a.Wq) *reinterpret_cast<float4*>(a.Wq + e0) = make_float4(wq[0], wq[1], wq[2], wq[3]);
      if (a.D_hi) {
        *reinterpret_cast<uint2*>(a.D_hi + e0) = make_uint2(pack_bf16x2_rn(dh[0], dh[1]), pack_bf16x2_rn(dh[2], dh[3]));
        if (a.D_lo)
          *reinterpret_cast<uint2*>(a.D_lo + e0) =
              make_uint2(pack_bf16x2_rn(dl[0], dl[1]), pack_bf16x2_rn(dl[2], dl[3]));
      }
    } else {
#pragma unroll
      for (int i = 0; i < kVec; ++i) {
        if (a.codes) a.codes[e0 + i] = static_cast<uint8_t>(q[i]);
        if (a.Wq) a.Wq[e0 + i] = wq[i];
        if (a.D_hi) {
          a.D_hi[e0 + i] = __float2bfloat16_rn(dh[i]);
          if (a.D_lo) a.D_lo[e0 + i] = __float2bfloat16_rn(dl[i]);
        }
      }
    }
  }
}

// One thread per output word; word w of a row holds stream bits [32w, 32w + 32).
__global__ void pack_kernel(const uint8_t* __restrict__ codes, int64_t rows, int64_t cols, int bits,
                            int64_t words_per_row, uint32_t* __restrict__ packed) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= rows * words_per_row) return;
  const int64_t row = idx / words_per_row;
  const int64_t w = idx - row * words_per_row;
  const int64_t bit0 = w * 32;
  const int64_t first = bit0 / bits;
  const int64_t last = (bit0 + 31) / bits;
  const uint32_t mask = (1u << bits) - 1u;
  const uint8_t* src = codes + row * cols;
  uint32_t word = 0;
  for (int64_t i = first; i <= last && i < cols; ++i) {
    const uint32_t c = static_cast<uint32_t>(src[i]) & mask;
    const int64_t shift = i * bits - bit0;
    if (shift >= 0) {
      if (shift < 32) word |= c << shift;
    } else {
      word |= c >> (-shift);
    }
  }
  packed[idx] = word;
}

// The same for bits 2, 4 and 8 (32 / bits codes per word, whole words per row):
// one vector load of the word's codes (4, 8 or 16 bytes, aligned when the codes
// are) instead of one byte load per code.
template <int kBits>
__global__ void pack_pow2_kernel(const uint8_t* __restrict__ codes, int64_t total_words,
                                 uint32_t* __restrict__ packed) {
  constexpr int kPer = 32 / kBits;  // codes per word; rows hold whole words
  constexpr uint32_t kMask = (1u << kBits) - 1u;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total_words) return;
  const uint8_t* src = codes + idx * kPer;
  uint32_t b[kPer / 4];
  if constexpr (kPer == 4) {
    b[0] = *reinterpret_cast<const uint32_t*>(src);
  } else if constexpr (kPer == 8) {
    const uint2 x = *reinterpret_cast<const uint2*>(src);
    b[0] = x.x;
    b[1] = x.y;
  } else {
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    b[0] = x.x;
    b[1] = x.y;
    b[2] = x.z;
    b[3] = x.w;
  }
  uint32_t word = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) word |= ((b[i / 4] >> (8 * (i % 4))) & kMask) << (kBits * i);
  packed[idx] = word;
}

__global__ void fill_f32_kernel(float* p, int64_t n, float v) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    p[i] = v;
}

// AR_INIT_MSE: one warp per group, one lane per grid ratio (two rounds for the 51
// ratios).  Each lane walks the group's columns in order and sums the squared
// round-to-nearest error in fp64 (fma(d, d, acc) rounds once, and d*d is exact
// in fp64, so this is the plain ordered sum of exact squares); the warp then takes
// the smallest (error, grid index) pair, i.e. the first minimum along the grid.
constexpr int kMseGrid = 51;

__global__ void mse_init_kernel(const void* __restrict__ W, int w_bf16, int64_t out, int64_t in, int g, int bits,
                                int sym, float* __restrict__ alpha, float* __restrict__ beta) {
  const int lane = threadIdx.x & 31;
  const int64_t G = in / g;
  const int64_t grp = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (grp >= out * G) return;  // warp-uniform
  const int64_t e0 = (grp / G) * in + (grp % G) * g;
  const uint16_t* wb = static_cast<const uint16_t*>(W) + e0;
  const float* wf = static_cast<const float*>(W) + e0;
  auto wat = [&](int k) { return w_bf16 ? bf16_bits_to_f32(wb[k]) : wf[k]; };

  float mn = 0.0f, mx = 0.0f;  // min(0, min W), max(0, max W) of the group
  bool ok = true;
  for (int k = lane; k < g; k += 32) {
    const float w = wat(k);
    mn = fminf(mn, w);
    mx = fmaxf(mx, w);
    ok = ok && div_fast_ok(w);
  }
  const bool fast = __all_sync(0xffffffffu, ok);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const float Q = qmaxf(bits);
  double best_e = INFINITY;
  int best_i = kMseGrid;
  for (int i = lane; i < kMseGrid + 31; i += 32) {  // both rounds run all 32 lanes
    const bool live = i < kMseGrid;
    const float p = __fdiv_rn(static_cast<float>(100 - (live ? i : 0)), 100.0f);
    const GroupScale gs = group_scale(mn, mx, p, p, bits, sym != 0);
    double acc = 0.0;
    for (int k = 0; k < g; ++k) {
      const float w = wat(k);
      const double d = static_cast<double>(__fsub_rn(quant_elem(w, 0.0f, gs, Q, fast).wq, w));
      acc = fma(d, d, acc);
    }
    if (live && (acc < best_e || (acc == best_e && i < best_i))) {
      best_e = acc;
      best_i = i;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const double oe = __shfl_xor_sync(0xffffffffu, best_e, o);
    const int oi = __shfl_xor_sync(0xffffffffu, best_i, o);
    if (oe < best_e || (oe == best_e && oi < best_i)) {
      best_e = oe;
      best_i = oi;
    }
  }
  if (lane == 0) {
    const float p = __fdiv_rn(static_cast<float>(100 - best_i), 100.0f);
    alpha[grp] = p;
    beta[grp] = p;
  }
}

// ---------------------------------------------------------------------------
// Helpers of the full-precision-target mode (ar_tune_layer_fp_target).
// ---------------------------------------------------------------------------

// x = hi + lo as an exact bf16 pair: hi = bf16(x), lo = bf16(x - hi) (x - hi is exact).
__device__ __forceinline__ void split_pair(float x, __nv_bfloat16& hi, __nv_bfloat16& lo) {
  hi = __float2bfloat16_rn(x);
  lo = __float2bfloat16_rn(__fsub_rn(x, __bfloat162float(hi)));
}

// dX = X - X_target (bf16 inputs; the fp32 difference) as a bf16 pair.
__global__ void diff_pair_kernel(const uint16_t* __restrict__ X, const uint16_t* __restrict__ Xt, int64_t n,
                                 __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float d = __fsub_rn(bf16_bits_to_f32(X[i]), bf16_bits_to_f32(Xt[i]));
    split_pair(d, hi[i], lo[i]);
  }
}

__global__ void split_pair_kernel(const float* __restrict__ x, int64_t n, __nv_bfloat16* __restrict__ hi,
                                  __nv_bfloat16* __restrict__ lo) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    split_pair(x[i], hi[i], lo[i]);
}

// acc += hi + lo (fp32).
__global__ void accum_pair_kernel(const __nv_bfloat16* __restrict__ hi, const __nv_bfloat16* __restrict__ lo,
                                  int64_t n, float* __restrict__ acc) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    acc[i] = __fadd_rn(acc[i], __fadd_rn(__bfloat162float(hi[i]), __bfloat162float(lo[i])));
}

// dst[j] = sum of part[j, 0 .. nparts) in order; total[j] += dst[j].
__global__ void row_sum_kernel(const float* __restrict__ part, int nparts, int64_t rows, float* __restrict__ dst,
                               float* __restrict__ total) {
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= rows) return;
  float L = 0.0f;
  for (int q = 0; q < nparts; ++q) L += part[j * nparts + q];
  dst[j] = L;
  total[j] = __fadd_rn(total[j], L);
}

// One block per step; fixed-order fp64 sums.
__global__ void loss_trace_kernel(const float* __restrict__ rowloss, int64_t out, int64_t batch_rows,
                                  float* __restrict__ loss_trace) {
  __shared__ double red[256];
  const int t = blockIdx.x;
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < out; j += blockDim.x) acc += rowloss[t * out + j];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) loss_trace[t] = static_cast<float>(red[0] / (static_cast<double>(batch_rows) * out));
}

__global__ void sum_to_double_kernel(const float* __restrict__ parts, int64_t count, double denom,
                                     double* __restrict__ result) {
  __shared__ double red[1024];
  double acc = 0.0;
  for (int64_t i = threadIdx.x; i < count; i += blockDim.x) acc += parts[i];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) result[0] = red[0] / denom;
}

// A barrier that nothing arrives on: the bounded wait must give up, record the
// timeout and let the kernel exit.
__global__ void timeout_selftest_kernel(int32_t* status, uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, status, timeout_ns);
    if (ok) atomicExch(status, -1);  // cannot happen: nothing arrives
  }
  __syncthreads();
}

// One warp per row.
__global__ void finalize_best_kernel(FinalizeBestArgs a) {
  const int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (j >= a.out) return;
  float L = 0.0f;
  const float* p = a.part + j * a.nparts;
  for (int q = 0; q < a.nparts; ++q) L += p[q];  // same order as the update epilogue
  bool better = false;
  if (a.keep_best) {
    const float mean = L * a.inv_batch;
    better = mean < a.best_in[j];
    if (lane == 0) a.best_out[j] = better ? mean : a.best_in[j];
  }
  if (lane == 0) a.rowloss[j] = L;
  if (!better) return;
  for (int64_t k = lane; k < a.in; k += 32) a.V_best[j * a.in + k] = a.V_last[j * a.in + k];
  for (int64_t k = lane; k < a.G; k += 32) {
    a.alpha_best[j * a.G + k] = a.alpha_last[j * a.G + k];
    a.beta_best[j * a.G + k] = a.beta_last[j * a.G + k];
  }
}

// One warp per (row, group) of a wide-group step: the group's d alpha and d beta
// from its segment partials (summed in slot order), the clip-factor sign updates
// with their keep-best snapshot (as the update epilogue takes it for narrow
// groups), then the next step's D = W' - W over the group's columns.
__global__ void group_finish_kernel(GroupFinishArgs a) {
  const int64_t grp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (grp >= a.out * a.G) return;  // warp-uniform
  const int64_t j = grp / a.G;
  const int64_t gg = grp - j * a.G;
  const int first = static_cast<int>((gg * a.g) / kSegCols);
  const int last = static_cast<int>(((gg + 1) * a.g - 1) / kSegCols);
  float dal = 0.f, dbe = 0.f;
  const float* p = a.gpart + grp * a.gslots * 2;
  for (int k = 0; k <= last - first; ++k) {
    dal += p[2 * k];
    dbe += p[2 * k + 1];
  }
  const bool sym = a.sym != 0;
  const float al = a.alpha_in[grp], be = a.beta_in[grp];
  const float al_n = clip_step(al, a.mlr, dal);
  const float be_n = sym ? be : clip_step(be, a.mlr, dbe);
  const bool better = a.judged && a.keep_best && a.best_out[j] < a.best_in[j];
  __syncwarp();  // every lane has read alpha_in, beta_in (they may alias the outputs)
  if (lane == 0 && in_bounds(grp, 1, a.chk_groups, a.status)) {
    if (better && !a.snap_prev) {
      a.alpha_best[grp] = al;
      a.beta_best[grp] = be;
    }
    if (better && a.snap_prev) {
      a.alpha_best[grp] = a.alpha_out[grp];
      a.beta_best[grp] = a.beta_out[grp];
    }
    a.alpha_out[grp] = al_n;
    a.beta_out[grp] = be_n;
  }
  const GroupScale gn = group_scale(a.wmin[grp], a.wmax[grp], al_n, be_n, a.bits, sym);
  const float Q = qmaxf(a.bits);
  const bool fast = a.div_slow && *a.div_slow == 0;
  // Eight consecutive elements per lane and iteration (g is a multiple of 16 and
  // in of 32, so the vectors are aligned and never straddle a group).
  const int64_t base = j * a.in + gg * a.g;
  for (int k = lane * 8; k < a.g; k += 32 * 8) {
    const int64_t e = base + k;
    float w[8], v[8];
    if (a.w_bf16) {
      const uint4 x = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.W) + e);
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        w[2 * h] = __uint_as_float(xs[h] << 16);
        w[2 * h + 1] = __uint_as_float(xs[h] & 0xFFFF0000u);
      }
    } else {
      const float4 x0 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.W) + e);
      const float4 x1 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.W) + e + 4);
      w[0] = x0.x, w[1] = x0.y, w[2] = x0.z, w[3] = x0.w, w[4] = x1.x, w[5] = x1.y, w[6] = x1.z, w[7] = x1.w;
    }
    const float4 v0 = *reinterpret_cast<const float4*>(a.V + e);
    const float4 v1 = *reinterpret_cast<const float4*>(a.V + e + 4);
    v[0] = v0.x, v[1] = v0.y, v[2] = v0.z, v[3] = v0.w, v[4] = v1.x, v[5] = v1.y, v[6] = v1.z, v[7] = v1.w;
    uint32_t hi2[4], lo2[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float hv[2], lv[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = 2 * h + q;
        const float d = __fsub_rn(quant_elem(w[i], v[i], gn, Q, fast).wq, w[i]);
        hv[q] = __bfloat162float(__float2bfloat16_rn(d));
        lv[q] = __fsub_rn(d, hv[q]);
      }
      const __nv_bfloat162 hp = __floats2bfloat162_rn(hv[0], hv[1]);
      const __nv_bfloat162 lp = __floats2bfloat162_rn(lv[0], lv[1]);
      hi2[h] = *reinterpret_cast<const uint32_t*>(&hp);
      lo2[h] = *reinterpret_cast<const uint32_t*>(&lp);
    }
    if (!in_bounds(e, 8, a.chk_elems, a.status)) continue;
    *reinterpret_cast<uint4*>(a.D_hi + e) = make_uint4(hi2[0], hi2[1], hi2[2], hi2[3]);
    if (a.D_lo) *reinterpret_cast<uint4*>(a.D_lo + e) = make_uint4(lo2[0], lo2[1], lo2[2], lo2[3]);
  }
}

__global__ void gram_sum_kernel(const __nv_bfloat16* __restrict__ H_hi, const __nv_bfloat16* __restrict__ H_lo,
                                int nb, int64_t count, __nv_bfloat16* __restrict__ Hs_hi,
                                __nv_bfloat16* __restrict__ Hs_lo) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int b = 0; b < nb; ++b) {
      s += __bfloat162float(H_hi[b * count + i]);
      if (H_lo) s += __bfloat162float(H_lo[b * count + i]);
    }
    const __nv_bfloat16 hi = __float2bfloat16_rn(s);
    Hs_hi[i] = hi;
    if (Hs_lo) Hs_lo[i] = __float2bfloat16_rn(s - __bfloat162float(hi));
  }
}

__global__ void diag_sum_kernel(const float* __restrict__ diag, int nb, int64_t in, float* __restrict__ dsum) {
  for (int64_t k = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; k < in;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.0f;
    for (int b = 0; b < nb; ++b) s += diag[b * in + k];
    dsum[k] = s;
  }
}

// W' = s * (q - zp), one element per thread.
__global__ void dequant_kernel(const uint8_t* __restrict__ codes, const float* __restrict__ scale,
                               const int32_t* __restrict__ zp, int64_t out, int64_t in, int g,
                               __nv_bfloat16* __restrict__ Wq_hi, __nv_bfloat16* __restrict__ Wq_lo,
                               float* __restrict__ Wq) {
  const int64_t total = out * in;
  const int64_t G = in / g;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t row = i / in;
    const int64_t gi = row * G + (i - row * in) / g;
    const float w = __fmul_rn(scale[gi], __fsub_rn(static_cast<float>(codes[i]), static_cast<float>(zp[gi])));
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    Wq_hi[i] = hi;
    if (Wq_lo) Wq_lo[i] = __float2bfloat16_rn(__fsub_rn(w, __bfloat162float(hi)));
    if (Wq) Wq[i] = w;
  }
}

__global__ void silu_mul_kernel(const __nv_bfloat16* __restrict__ a, const __nv_bfloat16* __restrict__ b,
                                int64_t count, __nv_bfloat16* __restrict__ y) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < count;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = __bfloat162float(a[i]);
    const float s = x / (1.0f + expf(-x));
    y[i] = __float2bfloat16_rn(s * __bfloat162float(b[i]));
  }
}

}  // namespace

cudaError_t launch_dequant(const uint8_t* codes, const float* scale, const int32_t* zp, int64_t out, int64_t in,
                           int g, __nv_bfloat16* Wq_hi, __nv_bfloat16* Wq_lo, float* Wq, cudaStream_t stream) {
  const int64_t total = out * in;
  if (total == 0) return cudaSuccess;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  dequant_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(codes, scale, zp, out, in, g, Wq_hi, Wq_lo, Wq);
  return cudaGetLastError();
}

cudaError_t launch_silu_mul(const __nv_bfloat16* a, const __nv_bfloat16* b, int64_t count, __nv_bfloat16* y,
                            cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 32) blocks = 148 * 32;
  silu_mul_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a, b, count, y);
  return cudaGetLastError();
}

cudaError_t launch_diag_sum(const float* diag, int nb, int64_t in, float* dsum, cudaStream_t stream) {
  if (in == 0) return cudaSuccess;
  diag_sum_kernel<<<static_cast<unsigned>((in + 255) / 256), 256, 0, stream>>>(diag, nb, in, dsum);
  return cudaGetLastError();
}

// kLayerBlocks blocks of 256 threads; block b sums rows [b * rpb, (b + 1) * rpb).
__global__ void layer_best_kernel(LayerBestArgs a) {
  __shared__ double red[256];
  __shared__ int last_block;
  __shared__ int improved;
  const int tid = threadIdx.x;
  if (a.init) {
    if (blockIdx.x == 0 && tid == 0) {
      *a.best = a.out > 0 ? static_cast<double>(a.best_rows[0]) : static_cast<double>(INFINITY);
      *a.ticket = 0u;
    }
    return;
  }
  const int64_t rpb = (a.out + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rpb;
  const int64_t r1 = min(a.out, r0 + rpb);
  double acc = 0.0;
  for (int64_t j = r0 + tid; j < r1; j += blockDim.x) {
    float L = 0.0f;
    const float* p = a.part + j * a.nparts;
    for (int q = 0; q < a.nparts; ++q) L += p[q];  // as the epilogues sum a row
    acc += static_cast<double>(L * a.inv_batch);
  }
  red[tid] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (tid < w) red[tid] += red[tid + w];
    __syncthreads();
  }
  if (tid == 0) {
    a.blocksum[blockIdx.x] = red[0];
    __threadfence();
    last_block = atomicAdd(a.ticket, 1u) == gridDim.x - 1;
  }
  __syncthreads();
  if (!last_block) return;
  if (tid == 0) {
    __threadfence();
    double total = 0.0;
    for (unsigned int b = 0; b < gridDim.x; ++b) total += __ldcg(a.blocksum + b);
    improved = total < *a.best;
    if (improved) *a.best = total;
    red[0] = total;
    *a.ticket = 0u;
  }
  __syncthreads();
  const float th = improved ? INFINITY : -INFINITY;
  const float v = static_cast<float>(red[0]);
  for (int64_t j = tid; j < a.out; j += blockDim.x) {
    a.thresh[j] = th;
    if (improved) a.best_rows[j] = v;
  }
}

cudaError_t launch_layer_best(const LayerBestArgs& a, cudaStream_t stream) {
  layer_best_kernel<<<a.init ? 1 : kLayerBlocks, 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_finalize_best(const FinalizeBestArgs& a, cudaStream_t stream) {
  if (a.out == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (a.out * 32 + threads - 1) / threads;
  finalize_best_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_gram_sum(const __nv_bfloat16* H_hi, const __nv_bfloat16* H_lo, int nb, int64_t count,
                            __nv_bfloat16* Hs_hi, __nv_bfloat16* Hs_lo, cudaStream_t stream) {
  if (count == 0) return cudaSuccess;
  int64_t blocks = (count + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  gram_sum_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(H_hi, H_lo, nb, count, Hs_hi, Hs_lo);
  return cudaGetLastError();
}

cudaError_t launch_group_quant(const GroupQuantArgs& a, cudaStream_t stream) {
  const int64_t groups = a.out * a.G;
  if (groups == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (groups * 32 + threads - 1) / threads;
  auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const bool vec = a.in % 4 == 0 && a.g % 4 == 0 && al16(a.W) && al16(a.V) && al16(a.codes) && al16(a.Wq) &&
                   al16(a.D_hi) && al16(a.D_lo);
  if (vec)
    group_quant_kernel<4><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  else
    group_quant_kernel<1><<<static_cast<unsigned>(blocks), threads, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_pack(const uint8_t* codes, int64_t rows, int64_t cols, int bits, int32_t* packed,
                        cudaStream_t stream) {
  const int64_t wpr = cols * bits / 32;
  const int64_t total = rows * wpr;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const unsigned blocks = static_cast<unsigned>((total + threads - 1) / threads);
  uint32_t* out = reinterpret_cast<uint32_t*>(packed);
  // Rows hold whole words, so word idx covers codes [idx * 32/bits, ...) of the flat array.
  const bool aligned = (reinterpret_cast<uintptr_t>(codes) & 15u) == 0;
  if (aligned && bits == 8)
    pack_pow2_kernel<8><<<blocks, threads, 0, stream>>>(codes, total, out);
  else if (aligned && bits == 4)
    pack_pow2_kernel<4><<<blocks, threads, 0, stream>>>(codes, total, out);
  else if (aligned && bits == 2)
    pack_pow2_kernel<2><<<blocks, threads, 0, stream>>>(codes, total, out);
  else
    pack_kernel<<<blocks, threads, 0, stream>>>(codes, rows, cols, bits, wpr, out);
  return cudaGetLastError();
}

cudaError_t launch_fill_f32(float* p, int64_t n, float value, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  fill_f32_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(p, n, value);
  return cudaGetLastError();
}

cudaError_t launch_group_finish(const GroupFinishArgs& a, cudaStream_t stream) {
  const int64_t warps = a.out * a.G;
  if (warps == 0) return cudaSuccess;
  const int64_t blocks = (warps * 32 + 255) / 256;
  group_finish_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_mse_init(const void* W, int w_bf16, int64_t out, int64_t in, int g, int bits, bool sym,
                            float* alpha, float* beta, cudaStream_t stream) {
  const int64_t groups = out * (in / g);
  if (groups <= 0) return cudaSuccess;
  const int64_t blocks = (groups + 7) / 8;  // 8 warps, one group each
  mse_init_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(W, w_bf16, out, in, g, bits, sym ? 1 : 0,
                                                                    alpha, beta);
  return cudaGetLastError();
}

static unsigned grid_for(int64_t n) {
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  return static_cast<unsigned>(blocks < 1 ? 1 : blocks);
}

cudaError_t launch_diff_pair(const uint16_t* X, const uint16_t* Xt, int64_t n, __nv_bfloat16* hi,
                             __nv_bfloat16* lo, cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  diff_pair_kernel<<<grid_for(n), 256, 0, stream>>>(X, Xt, n, hi, lo);
  return cudaGetLastError();
}

cudaError_t launch_split_pair(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* lo,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  split_pair_kernel<<<grid_for(n), 256, 0, stream>>>(x, n, hi, lo);
  return cudaGetLastError();
}

cudaError_t launch_accum_pair(const __nv_bfloat16* hi, const __nv_bfloat16* lo, int64_t n, float* acc,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  accum_pair_kernel<<<grid_for(n), 256, 0, stream>>>(hi, lo, n, acc);
  return cudaGetLastError();
}

cudaError_t launch_row_sum(const float* part, int nparts, int64_t rows, float* dst, float* total,
                           cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  row_sum_kernel<<<static_cast<unsigned>((rows + 255) / 256), 256, 0, stream>>>(part, nparts, rows, dst, total);
  return cudaGetLastError();
}

cudaError_t launch_loss_trace(const float* rowloss, int64_t out, int iters, int64_t batch_rows,
                              float* loss_trace, cudaStream_t stream) {
  if (iters == 0) return cudaSuccess;
  loss_trace_kernel<<<iters, 256, 0, stream>>>(rowloss, out, batch_rows, loss_trace);
  return cudaGetLastError();
}

cudaError_t launch_sum_to_double(const float* parts, int64_t count, double denom, double* result,
                                 cudaStream_t stream) {
  sum_to_double_kernel<<<1, 1024, 0, stream>>>(parts, count, denom, result);
  return cudaGetLastError();
}

// Every pair (a[i], b[j]) in the fast division's domain -- div_fast_ok(a[i]), b[j]
// a positive normal number at most 2^21 (a scale), and a/b zero or a normal number
// below 2^64 in magnitude -- counts the pairs where the quantiser's fast quotient
// differs in any bit from __fdiv_rn, and records the first such pair found.
__global__ void division_selftest_kernel(const float* __restrict__ a, int64_t na, const float* __restrict__ b,
                                         int64_t nb, unsigned long long* __restrict__ bad, float* __restrict__ first) {
  for (int64_t t = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; t < na * nb;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = a[t % na], y = b[t / na];
    if (!div_fast_ok(x) || !(y >= 0x1p-126f) || !(y <= 0x1p21f)) continue;
    const float exact = __fdiv_rn(x, y);
    if (!(fabsf(exact) < 0x1p64f) || (x != 0.0f && !(fabsf(exact) >= 0x1p-126f))) continue;
    const float fast = div_rn_by(x, y, __frcp_rn(y));
    if (__float_as_uint(fast) != __float_as_uint(exact)) {
      if (atomicAdd(bad, 1ull) == 0ull) {
        first[0] = x;
        first[1] = y;
      }
    }
  }
}

cudaError_t launch_division_selftest(const float* a, int64_t na, const float* b, int64_t nb,
                                     unsigned long long* bad, float* first, cudaStream_t stream) {
  if (na <= 0 || nb <= 0) return cudaSuccess;
  division_selftest_kernel<<<148 * 8, 256, 0, stream>>>(a, na, b, nb, bad, first);
  return cudaGetLastError();
}

cudaError_t launch_timeout_selftest(int32_t* status, uint64_t timeout_ns, cudaStream_t stream) {
  timeout_selftest_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

}  // namespace ar
