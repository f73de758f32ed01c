// Persistent warp-specialised bf16 GEMM for sm_100a with fused epilogues.
//
//   C[M, N] = sum over segments s of  A_s[M, K] * B_s[N, K]^T
//
// A and B are bf16, loaded by TMA in the 128-byte swizzle, K-major ([rows, K]) or
// MN-major ([K, rows]: activations read in place); C is fp32 in tensor memory.  A
// "segment" is one product with its own pair of operand maps, so an operand kept
// as an exact bf16 pair x = hi + lo (hi = bf16(x), lo = bf16(x - hi), about 16
// significant bits) is multiplied as extra segments of the same accumulation:
// (hi_a + lo_a)(hi_b + lo_b) ~ hi_a hi_b + lo_a hi_b + hi_a lo_b.
//
// Roles (320 threads, one CTA per SM; or clusters of two CTAs on 256-row pair
// tiles with tcgen05 cta_group::2):
//   warp 0      TMA producer.  Per stage either one 64-wide K block of one
//               segment's A and B tiles, or (fused stages) one K block of every
//               map the segments use, each staged once; completion counted on the
//               stage's mbarrier.
//   warp 1      MMA issuer: tcgen05.mma (M=128 or 256, N=BN, K=16), four per
//               segment in the stage (the Gram step's three pair products go per
//               K16 step, the two that share D_hi through the A collector buffer),
//               into one of two BN-column fp32 accumulators in tensor memory;
//               tcgen05.commit frees the stage and, after the last K block, hands
//               the accumulator to the epilogue.
//   warps 2..9  epilogue: two warps per 32-lane slice of tensor memory (a warp may
//               only read the slice warp % 4), one per column half of the tile.
//               Each thread owns one accumulator row and walks its half's columns
//               with tcgen05.ld while the MMA warp fills the other accumulator.
//               The halves never wait for each other: each writes its own row
//               partial sums (kEpiHalves entries per n-tile).
//
// Epilogues (the contractions of the AutoRound SignSGD loop,
// "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END"):
//   kEpiStore   C as a bf16 pair (hi, lo) into [rows, ldc], optionally with the row
//               sums of C^2 per n-tile: the residual R^T = D X_b^T of one step, or a
//               calibration block's Gram matrix H_b = X_b^T X_b.
//   kEpiSumSq   row sums of C^2 per n-tile only (final MSE over all rows).
//   kEpiUpdate  C = G = dL/dW' up to a positive factor: straight-through sign
//               updates of V (per element) and of alpha, beta (per group: a group
//               lies inside one thread's columns), the per-row keep-best snapshot,
//               the next step's D = W' - W as a bf16 pair, and (Gram form) the row
//               loss sum_k D_jk G_jk -- the gradient never reaches memory.
//   kEpiDotD    row sums of D * C per n-tile (the Gram form of the final MSE).
//
// Every mbarrier wait is bounded (GemmArgs::timeout_ns); a role that gives up
// records the timeout in *status and the CTA drains its in-flight copies and MMAs
// before it frees tensor memory and exits.
#include <atomic>

#include "ar_device.cuh"
#include "ar_internal.h"

namespace ar {

namespace {

constexpr int kEpiWarps = 4 * kEpiHalves;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kTileABytes = kBM * kBK * 2;  // 16 KB

// Per-CTA operand staging: 128 A rows and kBN (pair: kBN / 2) B rows per stage.
// Fused stages (kNA > 0): a stage holds one K block of each of the kNA A maps and
// kNB B maps the segments use, and the MMA warp issues every segment's product
// from it, so an operand that several segments share (the hi half of a pair, or a
// plain operand multiplied by both halves of the other) is staged once per K block
// instead of once per segment.  kNA = kNB = 0: one stage per (segment, K block).
template <int kBN, bool kPair, int kNA = 0, int kNB = 0>
struct Cfg {
  static constexpr bool kFused = kNA > 0;
  static constexpr int kTileBBytes = (kPair ? kBN / 2 : kBN) * kBK * 2;
  static constexpr int kStageBytes = kFused ? kNA * kTileABytes + kNB * kTileBBytes : kTileABytes + kTileBBytes;
  static constexpr int kStages = (kStageBytes <= 32 * 1024) ? 6 : (kStageBytes <= 48 * 1024 ? 4 : 3);
  static constexpr int kOffA1 = kTileABytes;  // fused: A0, (A1,) B0, (B1)
  static constexpr int kOffB0 = kFused ? kNA * kTileABytes : kTileABytes;
  static constexpr int kOffB1 = kOffB0 + kTileBBytes;
  static constexpr int kTmemCols = 2 * kBN;
  static constexpr int kBarOffset = kStages * kStageBytes;
  static constexpr int kSmemBytes = kBarOffset + 1024 + 1024;
  static constexpr uint32_t kIdesc = umma_idesc_bf16(kPair ? 2 * kBM : kBM, kBN);
};

__device__ __forceinline__ uint64_t operand_desc(uint32_t addr, bool mn) {
  return mn ? umma_desc_sw128_mn(addr) : umma_desc_sw128(addr);
}

// One operand tile of `rows` M (or N) indices x kBK K values into shared memory.
// K-major maps: one box.  MN-major maps: rows / 64 boxes of 64 x 64, 8 KB apart
// (the canonical MN-major layout of umma_desc_sw128_mn).
constexpr int kMnBoxBytes = 64 * kBK * 2;

template <bool kPair>
__device__ __forceinline__ void load_tile(uint8_t* dst, const CUtensorMap* map, bool mn, int k, int row, int rows,
                                          uint64_t* full, uint32_t leader_full) {
  if (!mn) {
    if (kPair)
      tma_load_2d_pair(dst, map, k, row, leader_full);
    else
      tma_load_2d(dst, map, k, row, full);
    return;
  }
  for (int j = 0; j < rows / 64; ++j) {
    if (kPair)
      tma_load_2d_pair(dst + j * kMnBoxBytes, map, row + 64 * j, k, leader_full);
    else
      tma_load_2d(dst + j * kMnBoxBytes, map, row + 64 * j, k, full);
  }
}

struct Smem {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(Smem) <= 1024, "barrier block");

// 32 consecutive W values (16-byte aligned) as fp32.
__device__ __forceinline__ void load_w32(const void* W, int w_bf16, int64_t idx, float (&w)[32]) {
  if (w_bf16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(W) + idx);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint4 x = p[q];
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        w[q * 8 + 2 * h] = __uint_as_float(xs[h] << 16);
        w[q * 8 + 2 * h + 1] = __uint_as_float(xs[h] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(W) + idx);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 x = p[q];
      w[q * 4 + 0] = x.x;
      w[q * 4 + 1] = x.y;
      w[q * 4 + 2] = x.z;
      w[q * 4 + 3] = x.w;
    }
  }
}

// 8 consecutive bf16 values (16 bytes, aligned) as fp32.
__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 x = *reinterpret_cast<const uint4*>(p);
  const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    v[2 * h] = __uint_as_float(xs[h] << 16);
    v[2 * h + 1] = __uint_as_float(xs[h] & 0xFFFF0000u);
  }
}

// 32 consecutive bf16 values as fp32.
__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* p, float (&v)[32]) {
  load_w32(p, 1, 0, v);
}

__device__ __forceinline__ void load_f32x32(const float* p, float (&v)[32]) {
  const float4* q4 = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 x = q4[q];
    v[q * 4 + 0] = x.x;
    v[q * 4 + 1] = x.y;
    v[q * 4 + 2] = x.z;
    v[q * 4 + 3] = x.w;
  }
}

// 16-column variants for the update epilogue, which keeps two chunks in registers.
constexpr int kUC = 16;

__device__ __forceinline__ void load_w16(const void* W, int w_bf16, int64_t idx, float (&w)[kUC]) {
  if (w_bf16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(W) + idx);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 x = p[q];
      const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        w[q * 8 + 2 * h] = __uint_as_float(xs[h] << 16);
        w[q * 8 + 2 * h + 1] = __uint_as_float(xs[h] & 0xFFFF0000u);
      }
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(W) + idx);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 x = p[q];
      w[q * 4 + 0] = x.x;
      w[q * 4 + 1] = x.y;
      w[q * 4 + 2] = x.z;
      w[q * 4 + 3] = x.w;
    }
  }
}

__device__ __forceinline__ void load_f32x16(const float* p, float (&v)[kUC]) {
  const float4* q4 = reinterpret_cast<const float4*>(p);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float4 x = q4[q];
    v[q * 4 + 0] = x.x;
    v[q * 4 + 1] = x.y;
    v[q * 4 + 2] = x.z;
    v[q * 4 + 3] = x.w;
  }
}

__device__ __forceinline__ void store_f32x16(float* p, const float (&v)[kUC]) {
  float4* q4 = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int q = 0; q < 4; ++q) q4[q] = make_float4(v[q * 4 + 0], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi) (x - hi is exact in fp32).
__device__ __forceinline__ void split_bf16(float x, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(x));
  lo = __fsub_rn(x, hi);
}

// Store 8 values (a multiple-of-8 column chunk) as hi and, if wanted, lo bf16.
__device__ __forceinline__ void store_pair8(const float* x, __nv_bfloat16* hi_dst, __nv_bfloat16* lo_dst) {
  float h[8], l[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) split_bf16(x[i], h[i], l[i]);
  *reinterpret_cast<uint4*>(hi_dst) =
      make_uint4(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]), pack_bf16x2(h[4], h[5]), pack_bf16x2(h[6], h[7]));
  if (lo_dst)
    *reinterpret_cast<uint4*>(lo_dst) = make_uint4(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]),
                                                   pack_bf16x2(l[4], l[5]), pack_bf16x2(l[6], l[7]));
}

// Tile t of the launch -> (m_blk, n_blk).  Plain: m fastest.  Symmetric: only the
// tiles with some column >= row, n-major, ceil((n + 1) * BN / BM) of them per n
// (BM: the m-block height, 256 rows for pair tiles).
template <int kBN, bool kPair>
__device__ __forceinline__ void tile_pos(const GemmArgs& a, int t, int& m_blk, int& n_blk) {
  if (!a.symmetric) {
    if (a.raster_m <= 0 || a.raster_m >= a.num_m_blk) {
      m_blk = t % a.num_m_blk;
      n_blk = t / a.num_m_blk;
      return;
    }
    const int per_group = a.raster_m * a.num_n_blk;
    const int grp = t / per_group;
    const int gm = min(a.raster_m, a.num_m_blk - grp * a.raster_m);  // m-blocks in this group
    const int ti = t - grp * per_group;
    m_blk = grp * a.raster_m + ti % gm;
    n_blk = ti / gm;
    return;
  }
  for (n_blk = 0; n_blk < a.num_n_blk; ++n_blk) {
    constexpr int kMH = kPair ? 2 * kBM : kBM;
    const int cnt = min(a.num_m_blk, ((n_blk + 1) * kBN + kMH - 1) / kMH);
    if (t < cnt) break;
    t -= cnt;
  }
  m_blk = t;
}

// Work unit u -> tile, and the column half it covers: the last split_tiles tiles in
// tile order are two units each, one per column half (nh = 0, 1); every other tile
// is one unit (nh = -1).  A launch whose tile count leaves a last partial wave of at
// most half the clusters splits those tiles, so that wave takes half as long.
__device__ __forceinline__ int unit_tile(int num_tiles, int split_tiles, int u, int& nh) {
  const int whole = num_tiles - split_tiles;
  if (u < whole) {
    nh = -1;
    return u;
  }
  nh = (u - whole) & 1;
  return whole + ((u - whole) >> 1);
}

// ---------------------------------------------------------------------------
// epilogues
// ---------------------------------------------------------------------------

// kEpiStore: 32 consecutive columns col0.. of row j (nvalid of them in range): the
// diagonal element into diag_out (stored as 0 in the pair), and the bf16 pair store (a symmetric C writes its upper elements in place and the strictly upper ones
// again transposed, so every element is written once).
__device__ __forceinline__ void store_cols32(const GemmArgs& a, int j, int col0, int nvalid, float (&x)[32]) {
  if (a.diag_out && j >= col0 && j < col0 + 32) {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (col0 + i == j) {
        a.diag_out[a.c_row_off + j] = x[i];
        x[i] = 0.0f;
      }
  }
  const int64_t off = (a.c_row_off + j) * a.ldc + col0;
  if (!in_bounds(off, nvalid, a.chk_c, a.status)) return;
  if (!a.symmetric) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q * 8 < nvalid) store_pair8(x + q * 8, a.C_hi + off + q * 8, a.C_lo ? a.C_lo + off + q * 8 : nullptr);
    return;
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int c8 = col0 + q * 8;
    if (q * 8 >= nvalid || c8 + 7 < j) continue;
    if (c8 >= j) {
      store_pair8(x + q * 8, a.C_hi + off + q * 8, a.C_lo ? a.C_lo + off + q * 8 : nullptr);
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (c8 + i >= j) {
          float h, l;
          split_bf16(x[q * 8 + i], h, l);
          a.C_hi[off + q * 8 + i] = __float2bfloat16_rn(h);
          if (a.C_lo) a.C_lo[off + q * 8 + i] = __float2bfloat16_rn(l);
        }
    }
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const int col = col0 + i;
    if (i < nvalid && col > j) {
      float h, l;
      split_bf16(x[i], h, l);
      const int64_t mo = (a.c_row_off + col) * a.ldc + j;
      if (!in_bounds(mo, 1, a.chk_c, a.status)) continue;
      a.C_hi[mo] = __float2bfloat16_rn(h);
      if (a.C_lo) a.C_lo[mo] = __float2bfloat16_rn(l);
    }
  }
}

// kEpiStore / kEpiSumSq / kEpiDotD: one pass over the tile's columns.
template <int kKind, int kBN>
__device__ __forceinline__ void epi_rows(const GemmArgs& a, uint32_t t_row, int j, int n0, int n_blk, int half) {
  float acc = 0.0f;
  const bool row_ok = j < a.M;
  constexpr int kHalfChunks = kBN / 32 / kEpiHalves;
#pragma unroll 1
  for (int c = half * kHalfChunks; c < (half + 1) * kHalfChunks; ++c) {
    const int col0 = n0 + c * 32;
    if (col0 >= a.N) break;  // warp-uniform
    uint32_t r[32];
    __syncwarp();
    tmem_ld_32cols(t_row + c * 32, r);
    tmem_ld_wait();
    if (!row_ok) continue;  // nothing warp-collective follows in this iteration
    const int nvalid = min(32, a.N - col0);  // a multiple of 8
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
    if ((kKind == kEpiStore || kKind == kEpiSumSq) && a.C_add) {
      // C += add_hi + add_lo (the pair's sum is exact in fp32), 8 columns at a time
      const int64_t offa = (a.c_row_off + j) * (a.ldc_add ? a.ldc_add : a.ldc) + col0;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q * 8 >= nvalid) break;
        float hv[8], lv[8];
        load_bf16x8(a.C_add + offa + q * 8, hv);
        if (a.C_add_lo) {
          load_bf16x8(a.C_add_lo + offa + q * 8, lv);
#pragma unroll
          for (int i = 0; i < 8; ++i) hv[i] = __fadd_rn(hv[i], lv[i]);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) x[q * 8 + i] = __fadd_rn(x[q * 8 + i], hv[i]);
      }
    }
    if (kKind == kEpiStore || kKind == kEpiSumSq) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nvalid) acc = fmaf(x[i], x[i], acc);
    }
    if (kKind == kEpiDotD) {
      const int64_t e = static_cast<int64_t>(j) * a.N + col0;
      float dh[32], dl[32];
      load_bf16x32(a.Dd_hi + e, dh);
      if (a.Dd_lo) {
        load_bf16x32(a.Dd_lo + e, dl);
#pragma unroll
        for (int i = 0; i < 32; ++i) dh[i] += dl[i];
      }
      if (a.diag_in) {
        float dg[32];
        load_f32x32(a.diag_in + col0, dg);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = fmaf(dh[i], dg[i], x[i]);
      }
      if (a.Cs) {  // full-precision target: + 2 D C^T
        float cs[32];
        load_f32x32(a.Cs + e, cs);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = fmaf(2.0f, cs[i], x[i]);
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) acc = fmaf(dh[i], x[i], acc);
    }
    if (kKind == kEpiStore) store_cols32(a, j, col0, nvalid, x);
  }
  if (kKind == kEpiDotD && row_ok && a.e_row && n_blk == 0 && half == 0) acc += a.e_row[j];
  if (row_ok && a.part) a.part[static_cast<int64_t>(j) * a.part_ld + n_blk * kEpiHalves + half] = acc;
}

// kEpiUpdate: one SignSGD step for the rows x columns of this G tile.
//
// The tile's groups are split between the two column halves (a group wider than
// half a tile stays with half 0).  Each chunk of kUC columns is processed while
// the next chunk's W, V and diagonal values are already on their way into
// registers, so the memory latency of one chunk overlaps the arithmetic of the
// previous one.
template <int kBN>
__device__ __forceinline__ void epi_group_range(const GemmArgs& a, int half, int& gl_begin, int& gl_end) {
  const int gpt = max(1, kBN / a.g);  // g divides kBN, or g == N <= kBN
  if (a.g <= kBN / kEpiHalves) {
    gl_begin = half * (gpt / kEpiHalves);
    gl_end = gl_begin + gpt / kEpiHalves;
  } else {
    gl_begin = 0;
    gl_end = half == 0 ? gpt : 0;
  }
}

// W, V and (Gram form) the exact Gram diagonal of one chunk.
__device__ __forceinline__ void load_upd_chunk(const GemmArgs& a, int64_t e0, int col, float (&w)[kUC],
                                               float (&v)[kUC], float (&dg)[kUC]) {
  load_w16(a.W, a.w_bf16, e0, w);
  load_f32x16(a.V_in + e0, v);
  if (a.diag_in) load_f32x16(a.diag_in + col, dg);
}

// Keep-best: the row's batch loss (sum of the per-n-tile partials in a fixed
// order, so every n-tile of the row reaches the same decision) against the best
// so far; the row's lead thread records the new best and the loss.  Direct form:
// the loss of this step (computed by the residual GEMM), snapshot of the state read
// now.  Gram form: the loss of the previous step (computed by the previous
// launch), snapshot of the previous state, which still sits in the output buffers
// until this epilogue overwrites it.
__device__ __forceinline__ bool row_better(const GemmArgs& a, int j, bool row_ok, int n_blk, int half) {
  bool better = false;
  if (row_ok && a.part_in) {
    // Sum in index order; eight loads are in flight at a time.
    float L = 0.0f;
    const float* p = a.part_in + static_cast<int64_t>(j) * a.nparts;
    int q = 0;
    for (; q + 8 <= a.nparts; q += 8) {
      float x[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) x[i] = p[q + i];
#pragma unroll
      for (int i = 0; i < 8; ++i) L += x[i];
    }
    for (; q < a.nparts; ++q) L += p[q];
    if (a.keep_best) {
      const float mean = L * a.inv_batch;
      better = mean < a.best_in[j];
      if (n_blk == 0 && half == 0) a.best_out[j] = better ? mean : a.best_in[j];
    }
    if (n_blk == 0 && half == 0) a.rowloss[j] = L;
  }
  return better;
}

// One element of the step: G (the accumulator, plus the exact Gram-diagonal term
// and, with a full-precision target, this block's C), the element's share of the
// row loss, its new V, and its terms of the group's d alpha and d beta.
template <bool kFp>
__device__ __forceinline__ float sign_step_elem(const GemmArgs& a, float w, float v, float acc, float dg, float cv,
                                                const GroupScale& gs, const GroupDeriv& gd, float Q, bool fast,
                                                float& loss_acc, float& dal, float& dbe) {
  const ElemQuant e = quant_elem(w, v, gs, Q, fast);
  const float d = __fsub_rn(e.wq, w);
  float G = a.diag_in ? fmaf(d, dg, acc) : acc;
  if (kFp) {
    // row loss: d H d^T + 2 d C^T (+ e_row once per row); gradient D H + C
    G = __fadd_rn(G, cv);
    loss_acc = fmaf(d, __fadd_rn(G, cv), loss_acc);
  } else {
    loss_acc = fmaf(d, G, loss_acc);
  }
  const float sg = e.m ? sgnf(G) : 0.0f;
  const float vn = fminf(fmaxf(__fsub_rn(v, __fmul_rn(a.lr, sg)), -0.5f), 0.5f);
  float dwa, dwb;
  if (e.m) {
    const float ru = e.r - e.u;
    dwa = gd.ds_a * ru;
    dwb = gd.ds_b * ru;
  } else {
    const float qz = e.q - gs.zp;
    dwa = gd.ds_a * qz - gs.s * gd.dzp_a;
    dwb = gd.ds_b * qz - gs.s * gd.dzp_b;
  }
  dal = fmaf(G, dwa, dal);
  dbe = fmaf(G, dwb, dbe);
  return vn;
}

// kFp: the full-precision-target terms (GemmArgs::Cc_hi set) are compiled in.
template <int kBN, bool kFp>
__device__ __forceinline__ void epi_update(const GemmArgs& a, uint32_t t_row, int j, int n0, int n_blk, int half) {
  const bool row_ok = j < a.M;
  const float Q = qmaxf(a.bits);
  const bool sym = a.sym != 0;
  const int64_t row_base = static_cast<int64_t>(j) * a.N;
  const bool better = row_better(a, j, row_ok, n_blk, half);
  const bool snap_now = better && !a.snap_prev;
  const bool snap_old = better && a.snap_prev;
  const bool fast = a.div_slow && *a.div_slow == 0;

  int gl_begin, gl_end;
  epi_group_range<kBN>(a, half, gl_begin, gl_end);
  const int cpg = a.g / kUC;  // chunks per group
  float loss_acc = 0.0f;
#pragma unroll 1
  for (int gl = gl_begin; gl < gl_end; ++gl) {
    const int gcol0 = n0 + gl * a.g;
    if (gcol0 >= a.N) break;  // warp-uniform
    const int64_t gidx = static_cast<int64_t>(j) * a.G + gcol0 / a.g;

    float wmn = 0.f, wmx = 0.f, al = 1.f, be = 1.f;
    if (row_ok) {
      wmn = a.wmin[gidx];
      wmx = a.wmax[gidx];
      al = a.alpha_in[gidx];
      be = a.beta_in[gidx];
    }
    const GroupScale gs = group_scale(wmn, wmx, al, be, a.bits, sym);
    const GroupDeriv gd = group_deriv(wmn, wmx, be, gs, Q, sym);

    // Pass 1: sign updates of V, and the group's d alpha, d beta.
    float dal = 0.f, dbe = 0.f;
    // The next chunk's W, V and diagonal are loaded one chunk ahead (the
    // full-precision-target instance loads this block's C instead, which needs
    // those registers).
    float w_nx[kUC], v_nx[kUC], dg_nx[kUC];
    if (!kFp && row_ok) load_upd_chunk(a, row_base + gcol0, gcol0, w_nx, v_nx, dg_nx);
#pragma unroll 1
    for (int cc = 0; cc < cpg; ++cc) {
      const int col = gcol0 + cc * kUC;
      const int64_t e0 = row_base + col;
      float w[kUC], v[kUC], dg[kUC];
      if (kFp) {
        if (row_ok) load_upd_chunk(a, e0, col, w, v, dg);
      } else {
#pragma unroll
        for (int i = 0; i < kUC; ++i) {
          w[i] = w_nx[i];
          v[i] = v_nx[i];
          dg[i] = dg_nx[i];
        }
        if (row_ok && cc + 1 < cpg) load_upd_chunk(a, e0 + kUC, col + kUC, w_nx, v_nx, dg_nx);
      }
      // Full-precision target: this block's C = W M_b (a bf16 pair) joins G.
      float cv[kUC];
      if (kFp && row_ok) {
        float clo[kUC];
        load_w16(a.Cc_hi, 1, e0, cv);
        load_w16(a.Cc_lo, 1, e0, clo);
#pragma unroll
        for (int i = 0; i < kUC; ++i) cv[i] = __fadd_rn(cv[i], clo[i]);
      }
      uint32_t r[kUC];
      __syncwarp();
      tmem_ld_16cols(t_row + (col - n0), r);
      tmem_ld_wait();
      if (!row_ok) continue;  // nothing warp-collective follows in this iteration
      const bool e_ok = in_bounds(e0, kUC, a.chk_elems, a.status);
      if (snap_old && e_ok) {
        float vo[kUC];
        load_f32x16(a.V_out + e0, vo);
        store_f32x16(a.V_best + e0, vo);
      }
      float vn[kUC];
#pragma unroll
      for (int i = 0; i < kUC; ++i)
        vn[i] = sign_step_elem<kFp>(a, w[i], v[i], __uint_as_float(r[i]), dg[i], kFp ? cv[i] : 0.0f, gs, gd, Q, fast,
                                    loss_acc, dal, dbe);
      if (e_ok) store_f32x16(a.V_out + e0, vn);
      if (snap_now && e_ok) store_f32x16(a.V_best + e0, v);
    }
    if (!row_ok) continue;

    const float al_n = clip_step(al, a.mlr, dal);
    const float be_n = sym ? be : clip_step(be, a.mlr, dbe);
    if (in_bounds(gidx, 1, a.chk_groups, a.status)) {
      if (snap_now) {
        a.alpha_best[gidx] = al;
        a.beta_best[gidx] = be;
      }
      if (snap_old) {
        a.alpha_best[gidx] = a.alpha_out[gidx];
        a.beta_best[gidx] = a.beta_out[gidx];
      }
      a.alpha_out[gidx] = al_n;
      a.beta_out[gidx] = be_n;
    }

    // Pass 2: D = W' - W of the next step, from the updated state, as a bf16 pair
    // (the values were written by this thread in pass 1).
    const GroupScale gn = group_scale(wmn, wmx, al_n, be_n, a.bits, sym);
    load_w16(a.W, a.w_bf16, row_base + gcol0, w_nx);
    load_f32x16(a.V_out + row_base + gcol0, v_nx);
#pragma unroll 1
    for (int cc = 0; cc < cpg; ++cc) {
      const int64_t e0 = row_base + gcol0 + cc * kUC;
      float w[kUC], v[kUC], d[kUC];
#pragma unroll
      for (int i = 0; i < kUC; ++i) {
        w[i] = w_nx[i];
        v[i] = v_nx[i];
      }
      if (cc + 1 < cpg) {
        load_w16(a.W, a.w_bf16, e0 + kUC, w_nx);
        load_f32x16(a.V_out + e0 + kUC, v_nx);
      }
#pragma unroll
      for (int i = 0; i < kUC; ++i) d[i] = __fsub_rn(quant_elem(w[i], v[i], gn, Q, fast).wq, w[i]);
      if (!in_bounds(e0, kUC, a.chk_elems, a.status)) continue;
#pragma unroll
      for (int q = 0; q < kUC / 8; ++q)
        store_pair8(d + q * 8, a.D_hi + e0 + q * 8, a.D_lo ? a.D_lo + e0 + q * 8 : nullptr);
    }
  }
  if (kFp && row_ok && a.e_row && n_blk == 0 && half == 0) loss_acc += a.e_row[j];
  if (row_ok && a.part_out) a.part_out[static_cast<int64_t>(j) * a.part_ld + n_blk * kEpiHalves + half] = loss_acc;
}

// kEpiUpdate*Wide: groups wider than a thread's columns, or not aligned to them.
// This thread walks its column half (kSegCols columns, one 128-column segment of
// the row) in chunks of kUC; a chunk lies in one group (g is a multiple of 16).
// Per element it does what epi_update's first pass does (G, the row loss, the new
// V, the V snapshot); the group's d alpha and d beta over this segment go to
// GemmArgs::gpart, and launch_group_finish completes the group.
template <int kBN, bool kFp>
__device__ __forceinline__ void epi_update_wide(const GemmArgs& a, uint32_t t_row, int j, int n0, int n_blk,
                                                int half) {
  static_assert(kBN / kEpiHalves == kSegCols, "one segment per thread");
  const bool row_ok = j < a.M;
  const float Q = qmaxf(a.bits);
  const bool sym = a.sym != 0;
  const int64_t row_base = static_cast<int64_t>(j) * a.N;
  const bool better = row_better(a, j, row_ok, n_blk, half);
  const bool snap_now = better && !a.snap_prev;
  const bool snap_old = better && a.snap_prev;
  const bool fast = a.div_slow && *a.div_slow == 0;
  const int c_begin = n0 + half * kSegCols;
  const int c_end = min(a.N, c_begin + kSegCols);
  const int seg = c_begin / kSegCols;

  float loss_acc = 0.0f;
  int cur = -1;  // group of the running sums
  float dal = 0.f, dbe = 0.f;
  GroupScale gs{1.f, 0.f, 1.f};
  GroupDeriv gd{0.f, 0.f, 0.f, 0.f};
  auto flush = [&]() {
    const int k = seg - static_cast<int>((static_cast<int64_t>(cur) * a.g) / kSegCols);
    float* p = a.gpart + ((static_cast<int64_t>(j) * a.G + cur) * a.gslots + k) * 2;
    p[0] = dal;
    p[1] = dbe;
  };
#pragma unroll 1
  for (int col = c_begin; col < c_end; col += kUC) {  // warp-uniform bounds
    const int gg = col / a.g;
    if (gg != cur) {
      if (cur >= 0 && row_ok) flush();
      cur = gg;
      dal = 0.f;
      dbe = 0.f;
      float wmn = 0.f, wmx = 0.f, al = 1.f, be = 1.f;
      if (row_ok) {
        const int64_t gidx = static_cast<int64_t>(j) * a.G + gg;
        wmn = a.wmin[gidx];
        wmx = a.wmax[gidx];
        al = a.alpha_in[gidx];
        be = a.beta_in[gidx];
      }
      gs = group_scale(wmn, wmx, al, be, a.bits, sym);
      gd = group_deriv(wmn, wmx, be, gs, Q, sym);
    }
    const int64_t e0 = row_base + col;
    float w[kUC], v[kUC], dg[kUC], cv[kUC];
    if (row_ok) {
      load_upd_chunk(a, e0, col, w, v, dg);
      if (kFp) {
        float clo[kUC];
        load_w16(a.Cc_hi, 1, e0, cv);
        load_w16(a.Cc_lo, 1, e0, clo);
#pragma unroll
        for (int i = 0; i < kUC; ++i) cv[i] = __fadd_rn(cv[i], clo[i]);
      }
    }
    uint32_t r[kUC];
    __syncwarp();
    tmem_ld_16cols(t_row + (col - n0), r);
    tmem_ld_wait();
    if (!row_ok) continue;  // nothing warp-collective follows in this iteration
    const bool e_ok = in_bounds(e0, kUC, a.chk_elems, a.status);
    if (snap_old && e_ok) {
      float vo[kUC];
      load_f32x16(a.V_out + e0, vo);
      store_f32x16(a.V_best + e0, vo);
    }
    float vn[kUC];
#pragma unroll
    for (int i = 0; i < kUC; ++i)
      vn[i] = sign_step_elem<kFp>(a, w[i], v[i], __uint_as_float(r[i]), dg[i], kFp ? cv[i] : 0.0f, gs, gd, Q, fast,
                                  loss_acc, dal, dbe);
    if (e_ok) store_f32x16(a.V_out + e0, vn);
    if (snap_now && e_ok) store_f32x16(a.V_best + e0, v);
  }
  if (cur >= 0 && row_ok) flush();
  if (kFp && row_ok && a.e_row && n_blk == 0 && half == 0) loss_acc += a.e_row[j];
  if (row_ok && a.part_out) a.part_out[static_cast<int64_t>(j) * a.part_ld + n_blk * kEpiHalves + half] = loss_acc;
}

// Before waiting for a tile's accumulator, ask L2 for the W and V row segments the
// update epilogue of that tile will read, so the wait covers their memory latency.
// (kWide: the thread's column half, which epi_update_wide walks.)
template <int kBN, bool kWide>
__device__ __forceinline__ void epi_update_prefetch(const GemmArgs& a, int j, int n0, int half) {
  if (j >= a.M) return;
  int c0, c1;
  if (kWide) {
    c0 = n0 + half * (kBN / kEpiHalves);
    c1 = min(a.N, c0 + kBN / kEpiHalves);
  } else {
    int gl_begin, gl_end;
    epi_group_range<kBN>(a, half, gl_begin, gl_end);
    c0 = n0 + gl_begin * a.g;
    c1 = min(a.N, n0 + gl_end * a.g);
  }
  if (c0 >= c1) return;
  const int64_t e0 = static_cast<int64_t>(j) * a.N + c0;
  const uint32_t cols = static_cast<uint32_t>(c1 - c0);  // a multiple of 8
  const int wsz = a.w_bf16 ? 2 : 4;
  prefetch_l2(static_cast<const uint8_t*>(a.W) + e0 * wsz, cols * wsz);
  prefetch_l2(a.V_in + e0, cols * 4);
  if (a.Cc_hi) {
    prefetch_l2(a.Cc_hi + e0, cols * 2);
    prefetch_l2(a.Cc_lo + e0, cols * 2);
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

// kPair: a cluster of two CTAs computes one 256 x kBN tile with tcgen05
// cta_group::2.  CTA `rank` loads its 128 A rows and B rows rank * kBN/2 ..
// + kBN/2 - 1 of the tile; its TMA bytes are counted on the leader's (rank 0)
// full barrier; the leader's MMA thread alone issues M = 256 MMAs and its commits
// arrive on both CTAs' barriers; each CTA's epilogue reads its own 128 accumulator
// rows and releases the accumulator with one arrive per warp on the leader.
// kMaj: bit 0 set when A is MN-major, bit 1 when B is (GemmArgs::a_mn, b_mn).
template <int kKind, int kBN, bool kPair, int kNA, int kNB, int kMaj>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                const __grid_constant__ CUtensorMap tmB0, const __grid_constant__ CUtensorMap tmB1,
                const __grid_constant__ GemmArgs args) {
  using C = Cfg<kBN, kPair, kNA, kNB>;
  constexpr bool kFused = C::kFused;
  // The Gram-matrix instance can sum K in chunks (GemmArgs::k_chunk): the MMAs of
  // each chunk accumulate afresh in accumulator 1, and the epilogue adds each chunk,
  // in fp32 round to nearest, to the tile's running sum kept in accumulator 0.
  constexpr bool kChunkable = (kKind == kEpiStore && kPair && kNA == 0 && kNB == 0 && kMaj == 3) ||
                              (kKind == kEpiUpdateExact && kPair && kNA == 2 && kNB == 2 && kMaj == 0);
  // The step instances on pair tiles may split the tiles of their last partial wave
  // into column halves (GemmArgs::split_tiles): a half unit issues N = kBN / 2 MMAs
  // into the half's own columns of the accumulator, and only that half's epilogue
  // warps run the epilogue, exactly as they do in a whole tile.  Each output element
  // is the same accumulation over K either way.
  constexpr bool kWideKind = kKind == kEpiUpdateWide || kKind == kEpiUpdateFpWide;
  constexpr bool kSplittable =
      kPair && kMaj == 0 && (kKind == kEpiUpdate || kKind == kEpiUpdateFp || kWideKind);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem* sm = reinterpret_cast<Smem*>(smem + C::kBarOffset);
  volatile int* abort_flag = &sm->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = kPair ? cluster_ctarank() : 0u;
  const int unit0 = kPair ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int unit_stride = kPair ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);

  if (warp == 1 && lane == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->tfull[b], 1);
      // 1-SM: every epilogue thread arrives; pair: one arrive per epilogue warp of
      // both CTAs, on the leader's barrier.
      mbar_init(&sm->tempty[b], kPair ? 2 * kEpiWarps : 32 * kEpiWarps);
    }
    mbar_init(&sm->drain, 1);
    sm->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    if (kPair) {
      tmem_alloc_pair(&sm->tmem_base, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(&sm->tmem_base, C::kTmemCols);
      tmem_relinquish();
    }
    if (lane == 0) {
      tma_prefetch_desc(&tmA0);
      tma_prefetch_desc(&tmB0);
      if (args.num_seg > 1) {
        tma_prefetch_desc(&tmA1);
        tma_prefetch_desc(&tmB1);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync_all();  // the peer's barriers are initialised before any remote arrive
  tc_fence_after();
  const uint32_t tmem_base = sm->tmem_base;
  // kFused: one stage per K block carries every segment; otherwise one per
  // (segment, K block), segments outermost.
  const int k_blocks = kFused ? args.num_k_blk : args.num_seg * args.num_k_blk;
  // K blocks per accumulator hand-off: the whole tile, or one chunk.
  // (kEpiUpdateExact always takes the chunked path, with one chunk when K is short.)
  const bool chunk_arg = args.k_chunk > 0 && args.k_chunk < k_blocks;
  const bool chunked = kChunkable && (kKind == kEpiUpdateExact || chunk_arg);
  const int k_chunk = chunked && chunk_arg ? args.k_chunk : k_blocks;
  // kFused: which of the two maps of A and of B the segments use.
  bool use_a1 = false, use_b1 = false;
  for (int s = 0; s < args.num_seg; ++s) {
    use_a1 = use_a1 || args.seg_a[s] != 0;
    use_b1 = use_b1 || args.seg_b[s] != 0;
  }
  // The pair-precision product (D_hi + D_lo)(H_hi + H_lo) of the Gram step on fused
  // stages: segments (A0, B0), (A1, B0), (A0, B1).  Per K16 step the MMA warp issues
  // the two products of A0 back to back, the first filling the A collector buffer and
  // the second reading it, so A0 leaves shared memory once per step (then A1's).
  const bool collect = kPair && kFused && kNA == 2 && kNB == 2 && args.num_seg == 3 && args.seg_a[0] == 0 &&
                       args.seg_b[0] == 0 && args.seg_a[1] == 1 && args.seg_b[1] == 0 && args.seg_a[2] == 0 &&
                       args.seg_b[2] == 1;
  // With one map of an operand staged, it is whichever one the segments use.
  const CUtensorMap* map_a0 = (kNA == 1 && use_a1) ? &tmA1 : &tmA0;
  const CUtensorMap* map_b0 = (kNB == 1 && use_b1) ? &tmB1 : &tmB0;
  constexpr int kBRows = kPair ? kBN / 2 : kBN;  // B rows this CTA stages
  // Operand majors: the instruction descriptor's bits, the shared-memory
  // descriptor, and its start-address step per K16 (32 B K-major, 2 KB MN-major).
  constexpr bool kAMn = (kMaj & 1) != 0, kBMn = (kMaj & 2) != 0;
  constexpr uint32_t idesc = C::kIdesc | (kAMn ? kIdescAMn : 0u) | (kBMn ? kIdescBMn : 0u);
  constexpr uint32_t idesc_half =
      umma_idesc_bf16(kPair ? 2 * kBM : kBM, kBN / 2) | (kAMn ? kIdescAMn : 0u) | (kBMn ? kIdescBMn : 0u);
  // A non-wide epilogue keeps groups inside a column half only when g <= kBN / 2.
  const int split_tiles =
      (kSplittable && (kWideKind || args.g <= kBN / kEpiHalves)) ? args.split_tiles : 0;
  const int num_units = args.num_tiles + split_tiles;
  constexpr uint32_t a_kstep = kAMn ? 128u : 2u, b_kstep = kBMn ? 128u : 2u;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int u = unit0; ok && u < num_units; u += unit_stride) {
        int nh;
        const int tile = unit_tile(args.num_tiles, split_tiles, u, nh);
        int m_blk, n_blk;
        tile_pos<kBN, kPair>(args, tile, m_blk, n_blk);
        const int a_row = (kPair ? 2 * m_blk + static_cast<int>(rank) : m_blk) * kBM;
        // A half unit's MMAs read the first kBN / 4 of the B rows each CTA stages
        // (the box is loaded whole).
        const int b_col = nh < 0 ? static_cast<int>(rank) * (kBN / 2)
                                 : nh * (kBN / 2) + static_cast<int>(rank) * (kBN / 4);
        const int b_row = n_blk * kBN + args.b_row_off + (kPair ? b_col : 0);
        for (int kb = 0; kb < k_blocks; ++kb) {
          const int seg = kb / args.num_k_blk;
          const int kk = kb - seg * args.num_k_blk;
          const CUtensorMap* mA = args.seg_a[seg] ? &tmA1 : &tmA0;
          const CUtensorMap* mB = args.seg_b[seg] ? &tmB1 : &tmB0;
          if (!mbar_wait<kPair>(&sm->empty[stage], phase ^ 1, abort_flag, args.status, args.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * C::kStageBytes;
          uint8_t* sB = sA + kTileABytes;
          if (kFused) {
            // every slot of the stage is filled: the host picks kNA, kNB as the
            // number of distinct maps the segments use
            if (!kPair || rank == 0) mbar_arrive_expect_tx(&sm->full[stage], (kPair ? 2 : 1) * C::kStageBytes);
            const int ka = kb * kBK + args.a_k_off, kbb = kb * kBK + args.b_k_off;
            const uint32_t leader_full = kPair ? mapa_shared(smem_u32(&sm->full[stage]), 0) : 0u;
            uint64_t* full = &sm->full[stage];
            load_tile<kPair>(sA, map_a0, kAMn, ka, a_row, kBM, full, leader_full);
            if (kNA == 2) load_tile<kPair>(sA + C::kOffA1, &tmA1, kAMn, ka, a_row, kBM, full, leader_full);
            load_tile<kPair>(sA + C::kOffB0, map_b0, kBMn, kbb, b_row, kBRows, full, leader_full);
            if (kNB == 2) load_tile<kPair>(sA + C::kOffB1, &tmB1, kBMn, kbb, b_row, kBRows, full, leader_full);
          } else {
            if (!kPair || rank == 0) mbar_arrive_expect_tx(&sm->full[stage], (kPair ? 2 : 1) * C::kStageBytes);
            const uint32_t leader_full = kPair ? mapa_shared(smem_u32(&sm->full[stage]), 0) : 0u;
            load_tile<kPair>(sA, mA, kAMn, kk * kBK + args.a_k_off, a_row, kBM, &sm->full[stage], leader_full);
            load_tile<kPair>(sB, mB, kBMn, kk * kBK + args.b_k_off, b_row, kBRows, &sm->full[stage], leader_full);
          }
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        if (kPair) {
          // The copies' completion is counted on the leader's barriers, which this
          // CTA cannot wait on: give anything in flight time to land.
          const uint64_t t0 = globaltimer_ns();
          while (globaltimer_ns() - t0 < 10000000ull) {
          }
        } else {
          // Let the copies already issued land before the CTA exits.
          for (int s = 0; s < C::kStages; ++s)
            if (issued_mask & (1u << s)) mbar_wait_drain(&sm->full[s], (issued_parity >> s) & 1u, args.timeout_ns);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      uint32_t chunk_phase = 0;  // chunked: phase of accumulator 1, the only one the MMAs use
      bool ok = true;
      for (int u = unit0; ok && u < num_units; u += unit_stride) {
       int nh;
       unit_tile(args.num_tiles, split_tiles, u, nh);
       const uint32_t idesc_u = nh < 0 ? idesc : idesc_half;
       for (int kb0 = 0; ok && kb0 < k_blocks; kb0 += k_chunk) {
        const int buf = chunked ? 1 : acc;
        if (!mbar_wait<kPair>(&sm->tempty[buf], (chunked ? chunk_phase : acc_phase) ^ 1, abort_flag, args.status,
                              args.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * kBN + (nh > 0 ? kBN / 2 : 0);
        const int kb1 = min(k_blocks, kb0 + k_chunk);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait<kPair>(&sm->full[stage], phase, abort_flag, args.status, args.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::kStageBytes);
          if (kFused && collect) {
            const uint64_t a0 = operand_desc(a_addr, kAMn), a1 = operand_desc(a_addr + C::kOffA1, kAMn);
            const uint64_t b0 = operand_desc(a_addr + C::kOffB0, kBMn);
            const uint64_t b1 = operand_desc(a_addr + C::kOffB1, kBMn);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint32_t accum = ((kb - kb0) | k) != 0 ? 1u : 0u;
              umma_bf16_pair_collect<true>(d_tmem, a0 + a_kstep * k, b0 + b_kstep * k, idesc_u, accum);
              umma_bf16_pair_collect<false>(d_tmem, a0 + a_kstep * k, b1 + b_kstep * k, idesc_u, 1u);
              umma_bf16_pair(d_tmem, a1 + a_kstep * k, b0 + b_kstep * k, idesc_u, 1u);
            }
          } else if (kFused) {
            for (int s = 0; s < args.num_seg; ++s) {
              const uint64_t a_desc =
                  operand_desc(a_addr + ((kNA == 2 && args.seg_a[s]) ? C::kOffA1 : 0), kAMn);
              const uint64_t b_desc =
                  operand_desc(a_addr + ((kNB == 2 && args.seg_b[s]) ? C::kOffB1 : C::kOffB0), kBMn);
#pragma unroll
              for (int k = 0; k < kBK / 16; ++k) {
                const uint32_t accum = ((kb - kb0) | s | k) != 0 ? 1u : 0u;
                if (kPair)
                  umma_bf16_pair(d_tmem, a_desc + a_kstep * k, b_desc + b_kstep * k, idesc_u, accum);
                else
                  umma_bf16(d_tmem, a_desc + a_kstep * k, b_desc + b_kstep * k, idesc_u, accum);
              }
            }
          } else {
            const uint64_t a_desc = operand_desc(a_addr, kAMn);
            const uint64_t b_desc = operand_desc(a_addr + kTileABytes, kBMn);
#pragma unroll
            for (int k = 0; k < kBK / 16; ++k) {
              const uint32_t accum = ((kb - kb0) | k) != 0 ? 1u : 0u;
              if (kPair)
                umma_bf16_pair(d_tmem, a_desc + a_kstep * k, b_desc + b_kstep * k, idesc_u, accum);
              else
                umma_bf16(d_tmem, a_desc + a_kstep * k, b_desc + b_kstep * k, idesc_u, accum);
            }
          }
          if (kPair)
            umma_commit_pair_both(&sm->empty[stage]);
          else
            umma_commit(&sm->empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        if (kPair)
          umma_commit_pair_both(&sm->tfull[buf]);
        else
          umma_commit(&sm->tfull[buf]);
        if (chunked) {
          chunk_phase ^= 1;
        } else {
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1;
        }
       }
      }
      // Every MMA this thread issued has completed once `drain` flips.
      if (kPair)
        umma_commit_pair_local(&sm->drain);
      else
        umma_commit(&sm->drain);
      mbar_wait_drain(&sm->drain, 0, args.timeout_ns);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    const int half = (warp - 2) >> 2;  // column half of the tile
    const int row_in_tile = quarter * 32 + lane;
    // Pair: the leader's accumulator-empty barriers, as shared::cluster addresses.
    const uint32_t leader_tempty0 = kPair ? mapa_shared(smem_u32(&sm->tempty[0]), 0) : 0u;
    const uint32_t leader_tempty1 = kPair ? mapa_shared(smem_u32(&sm->tempty[1]), 0) : 0u;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t chunk_phase = 0;  // chunked: phase of accumulator 1
    for (int u = unit0; u < num_units; u += unit_stride) {
      int nh;
      const int tile = unit_tile(args.num_tiles, split_tiles, u, nh);
      // A half unit's accumulator holds only its half's columns: the other half's
      // warps only hand the accumulator back.
      const bool active = nh < 0 || nh == half;
      int m_blk, n_blk;
      tile_pos<kBN, kPair>(args, tile, m_blk, n_blk);
      const int j = (kPair ? 2 * m_blk + static_cast<int>(rank) : m_blk) * kBM + row_in_tile;
      const int n0 = n_blk * kBN;
      if ((kKind == kEpiUpdate || kKind == kEpiUpdateFp || kKind == kEpiUpdateExact) && active)
        epi_update_prefetch<kBN, false>(args, j, n0, half);
      if (kWideKind && active) epi_update_prefetch<kBN, true>(args, j, n0, half);
      if constexpr (kChunkable) {
        if (chunked) {
          // Each chunk: accumulator 1 (the chunk) added into accumulator 0 (the
          // running sum) in fp32, then accumulator 1 released; after the last one the
          // sum is stored.  A warp touches only its own lanes and columns of both.
          const uint32_t lanes = static_cast<uint32_t>(quarter * 32) << 16;
          const uint32_t t_sum = tmem_base + lanes + half * (kBN / kEpiHalves);
          const uint32_t t_chunk = t_sum + kBN;
          bool ok = true;
          for (int kb0 = 0; kb0 < k_blocks; kb0 += k_chunk) {
            if (!mbar_wait<kPair>(&sm->tfull[1], chunk_phase, abort_flag, args.status, args.timeout_ns, false)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll 1
            for (int g = 0; g < kBN / kEpiHalves / 32; ++g) {
              uint32_t r[32];
              __syncwarp();
              tmem_ld_32cols(t_chunk + g * 32, r);
              tmem_ld_wait();
              if (kb0 > 0) {
                uint32_t q[32];
                tmem_ld_32cols(t_sum + g * 32, q);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__fadd_rn(__uint_as_float(q[i]), __uint_as_float(r[i])));
              }
              tmem_st_32cols(t_sum + g * 32, r);
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_tempty1);
            chunk_phase ^= 1;
          }
          if (!ok) break;
          if constexpr (kKind == kEpiUpdateExact) {
            // the step on the tile's sum in accumulator 0, which no MMA writes
            tc_fence_after();
            epi_update<kBN, false>(args, tmem_base + lanes, j, n0, n_blk, half);
            continue;
          } else {
            // the tile's sum, from accumulator 0
#pragma unroll 1
            for (int g = 0; g < kBN / kEpiHalves / 32; ++g) {
              uint32_t r[32];
              __syncwarp();
              tmem_ld_32cols(t_sum + g * 32, r);
              tmem_ld_wait();
              const int col0 = n0 + half * (kBN / kEpiHalves) + g * 32;
              if (j >= args.M || col0 >= args.N) continue;  // nothing warp-collective follows
              float x[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(r[i]);
              store_cols32(args, j, col0, min(32, args.N - col0), x);
            }
            continue;
          }
        }
      }
      // No early exit on another role's abort: every epilogue warp of the CTA takes
      // the same decision here (the phase completes for all of them, or for none).
      if (!mbar_wait<kPair>(&sm->tfull[acc], acc_phase, abort_flag, args.status, args.timeout_ns, false)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
      if (active) {
        if constexpr (kKind == kEpiUpdateExact) {
          // always chunked (above)
        } else if constexpr (kKind == kEpiUpdate)
          epi_update<kBN, false>(args, t_row, j, n0, n_blk, half);
        else if constexpr (kKind == kEpiUpdateFp)
          epi_update<kBN, true>(args, t_row, j, n0, n_blk, half);
        else if constexpr (kKind == kEpiUpdateWide)
          epi_update_wide<kBN, false>(args, t_row, j, n0, n_blk, half);
        else if constexpr (kKind == kEpiUpdateFpWide)
          epi_update_wide<kBN, true>(args, t_row, j, n0, n_blk, half);
        else
          epi_rows<kKind, kBN>(args, t_row, j, n0, n_blk, half);
      }
      tc_fence_before();
      if (kPair) {
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(acc ? leader_tempty1 : leader_tempty0);
      } else {
        mbar_arrive(&sm->tempty[acc]);
      }
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (kPair) cluster_sync_all();  // the leader's MMAs into this CTA's tensor memory are done
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    if (kPair)
      tmem_dealloc_pair(tmem_base, C::kTmemCols);
    else
      tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// The fused instances that the library's GEMMs use (the others are not compiled):
// pair 2+2 (the Gram step; the full-precision-target products with an fp32 W),
// pair 1+2 (those products with a bf16 W), pair 2+1 (direct form on pair tiles),
// 1-SM 2+1 (the direct form's residual, update and final MSE).
template <int kKind, int kBN, bool kPair, int kNA, int kNB>
constexpr bool stage_instance() {
  if (kNA == 0) return kNB == 0;
  if (kPair && kNA == 2 && kNB == 2)
    return kKind == kEpiUpdate || kKind == kEpiUpdateFp || kKind == kEpiStore || kKind == kEpiSumSq ||
           kKind == kEpiUpdateExact;
  if (kPair && kNA == 1 && kNB == 2) return kKind == kEpiStore || kKind == kEpiSumSq;
  if (kPair && kNA == 2 && kNB == 1) return kKind == kEpiStore || kKind == kEpiUpdate;
  if (!kPair && kBN == 256 && kNA == 2 && kNB == 1)
    return kKind == kEpiStore || kKind == kEpiUpdate || kKind == kEpiSumSq;
  return false;
}

// MN-major operands (the activations read in place): both for the Gram matrices
// and the full-precision-target M_b (kEpiStore), B for the direct update.
template <int kKind, int kBN, bool kPair, int kNA, int kNB, int kMaj>
constexpr bool kernel_instance() {
  // The chunked-accumulation step: the Gram step's pair tiles and fused 2 + 2 stages only.
  if (kKind == kEpiUpdateExact) return kPair && kBN == 256 && kNA == 2 && kNB == 2 && kMaj == 0;
  // Wide-group steps: the Gram step on pair tiles (pair or single operands, with or
  // without a full-precision target) and the direct update on 1-SM tiles.
  if (kKind == kEpiUpdateWide || kKind == kEpiUpdateFpWide) {
    if (kBN != 256 || !((kNA == 2 && kNB == 2) || (kNA == 0 && kNB == 0) || (kNA == 2 && kNB == 1))) return false;
    if (kPair) return kMaj == 0 && kNB != 1;
    return kKind == kEpiUpdateWide && kMaj == 2 && kNB != 2;
  }
  if (!stage_instance<kKind, kBN, kPair, kNA, kNB>()) return false;
  if (kMaj == 0) return true;
  if (kBN != 256) return false;
  if (kMaj == 3) return kKind == kEpiStore && ((kNA == 0 && kNB == 0) || (kNA == 1 && kNB == 2));
  if (kMaj == 2) return kKind == kEpiUpdate && ((kNA == 0 && kNB == 0) || (kNA == 2 && kNB == 1));
  return false;
}

template <int kKind, int kBN, bool kPair, int kNA, int kNB, int kMaj>
cudaError_t launch_kind(const GemmMaps& m, const GemmArgs& args, int num_sms, cudaStream_t stream) {
  if constexpr (!kernel_instance<kKind, kBN, kPair, kNA, kNB, kMaj>()) {
    return cudaErrorInvalidValue;
  } else {
    using C = Cfg<kBN, kPair, kNA, kNB>;
    auto* fn = gemm_kernel<kKind, kBN, kPair, kNA, kNB, kMaj>;
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    if (e != cudaSuccess) return e;
    if (!kPair) {
      const int grid = args.num_tiles < num_sms ? args.num_tiles : num_sms;
      if (grid <= 0) return cudaSuccess;
      fn<<<grid, kThreads, C::kSmemBytes, stream>>>(m.a0, m.a1, m.b0, m.b1, args);
      return cudaGetLastError();
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (num_sms / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // A persistent grid must not exceed the clusters that can be resident at once
    // (a pair needs two SMs of one GPC): queried once per device.
    // (One cache per kernel instance; host threads may launch concurrently.)
    static std::atomic<int> resident[64];  // 0: not yet known
    int dev = 0;
    e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int max_pairs = (dev >= 0 && dev < 64) ? resident[dev].load(std::memory_order_relaxed) : 0;
    if (max_pairs <= 0) {
      e = cudaOccupancyMaxActiveClusters(&max_pairs, fn, &cfg);
      if (e != cudaSuccess) return e;
      if (max_pairs <= 0) return cudaErrorInvalidConfiguration;
      if (dev >= 0 && dev < 64) resident[dev].store(max_pairs, std::memory_order_relaxed);
    }
    int pairs_max = num_sms / 2 < max_pairs ? num_sms / 2 : max_pairs;
    if (pairs_max <= 0 || args.num_tiles <= 0) return cudaSuccess;
    // A last partial wave of at most half the clusters: its tiles become two
    // column-half units each (the kernel ignores the request where it cannot split).
    GemmArgs a = args;
    a.split_tiles = 0;
    const int tail = args.num_tiles % pairs_max;
    constexpr bool kWideKind = kKind == kEpiUpdateWide || kKind == kEpiUpdateFpWide;
    constexpr bool kSplitKind = kMaj == 0 && (kKind == kEpiUpdate || kKind == kEpiUpdateFp || kWideKind);
    const bool can_split = kSplitKind && (kWideKind || args.g <= kBN / kEpiHalves);
    if (args.tail_split && can_split && tail > 0 && 2 * tail <= pairs_max) a.split_tiles = tail;
    const int units = a.num_tiles + a.split_tiles;
    const int pairs = units < pairs_max ? units : pairs_max;
    cfg.gridDim = dim3(2 * pairs, 1, 1);
    e = cudaLaunchKernelEx(&cfg, fn, m.a0, m.a1, m.b0, m.b1, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
}

template <int kBN, bool kPair, int kNA, int kNB, int kMaj>
cudaError_t launch_bn(EpiKind kind, const GemmMaps& m, const GemmArgs& args, int num_sms, cudaStream_t stream) {
  switch (kind) {
    case kEpiStore:
      return launch_kind<kEpiStore, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiSumSq:
      return launch_kind<kEpiSumSq, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiUpdate:
      return launch_kind<kEpiUpdate, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiDotD:
      return launch_kind<kEpiDotD, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiUpdateFp:
      return launch_kind<kEpiUpdateFp, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiUpdateWide:
      return launch_kind<kEpiUpdateWide, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiUpdateFpWide:
      return launch_kind<kEpiUpdateFpWide, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
    case kEpiUpdateExact:
      return launch_kind<kEpiUpdateExact, kBN, kPair, kNA, kNB, kMaj>(m, args, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

// The operand majors of a launch as the kernel's kMaj.
template <int kBN, bool kPair, int kNA = 0, int kNB = 0>
cudaError_t launch_major(EpiKind kind, const GemmMaps& m, const GemmArgs& args, int num_sms, cudaStream_t stream) {
  const int maj = (args.a_mn ? 1 : 0) | (args.b_mn ? 2 : 0);
  switch (maj) {
    case 0:
      return launch_bn<kBN, kPair, kNA, kNB, 0>(kind, m, args, num_sms, stream);
    case 2:
      return launch_bn<kBN, kPair, kNA, kNB, 2>(kind, m, args, num_sms, stream);
    case 3:
      return launch_bn<kBN, kPair, kNA, kNB, 3>(kind, m, args, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemm(EpiKind kind, int bn, const GemmMaps& maps, const GemmArgs& args, int num_sms,
                        cudaStream_t stream) {
  if (args.num_seg < 1 || args.num_seg > 3) return cudaErrorInvalidValue;
  // Fused stages: as many A (B) tiles per stage as the segments use distinct maps.
  int na = 0, nb = 0;
  if (args.fused) {
    bool a[2] = {false, false}, b[2] = {false, false};
    for (int s = 0; s < args.num_seg; ++s) {
      a[args.seg_a[s] ? 1 : 0] = true;
      b[args.seg_b[s] ? 1 : 0] = true;
    }
    na = a[0] + a[1];
    nb = b[0] + b[1];
  }
  if (args.pair) {
    // Pair tiles: 256 rows x 256 columns; K-major B maps with 128-row boxes.
    if (bn != 256) return cudaErrorInvalidValue;
    if (!args.fused) return launch_major<256, true>(kind, maps, args, num_sms, stream);
    if (na == 2 && nb == 2) return launch_major<256, true, 2, 2>(kind, maps, args, num_sms, stream);
    if (na == 2 && nb == 1) return launch_major<256, true, 2, 1>(kind, maps, args, num_sms, stream);
    if (na == 1 && nb == 2) return launch_major<256, true, 1, 2>(kind, maps, args, num_sms, stream);
    return cudaErrorInvalidValue;
  }
  if (args.fused) {
    if (bn == 256 && na == 2 && nb == 1 && !args.symmetric)
      return launch_major<256, false, 2, 1>(kind, maps, args, num_sms, stream);
    return cudaErrorInvalidValue;
  }
  if (bn == 256) return launch_major<256, false>(kind, maps, args, num_sms, stream);
  if (bn == 128) return launch_major<128, false>(kind, maps, args, num_sms, stream);
  return cudaErrorInvalidValue;
}

}  // namespace ar
