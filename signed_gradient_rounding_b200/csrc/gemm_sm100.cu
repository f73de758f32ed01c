// Persistent warp-specialised bf16 GEMM for sm_100a with fused epilogues.
//
//   C[M, N] = A[M, K] * B[N, K]^T      (A, B bf16 K-major; C fp32 in tensor memory)
//
// Roles (192 threads, one CTA per SM):
//   warp 0      TMA producer: 128x64 A tile + 256x64 B tile per stage, 4 stages,
//               128-byte swizzle, completion counted on the stage's mbarrier.
//   warp 1      MMA issuer: four tcgen05.mma (M=128, N=256, K=16) per stage into
//               one of two 256-column fp32 accumulators in tensor memory;
//               tcgen05.commit frees the stage and, after the last K block,
//               hands the accumulator to the epilogue.
//   warps 2..5  epilogue: each thread owns one accumulator row (its warp's
//               32-lane slice of tensor memory) and walks the tile's 256 columns
//               32 at a time with tcgen05.ld, while the MMA warp fills the other
//               accumulator with the next tile.
//
// Epilogues (the two contractions of one SignSGD step of the AutoRound loop,
// "[llm-compressor] AutoRound ...", "on_event with SEQUENTIAL_EPOCH_END"):
//   kEpiResidual  A = D = bf16(W' - W) [out, in], B = X_b [B, in]: C = R^T = (Y' - Y)^T.
//                 Stores R^T in bf16 and per-(row, n-tile) sums of R^2.
//   kEpiUpdate    A = R^T [out, B], B = X_b^T [in, B]: C = G = R^T X_b = dL/dW' * B*out/2.
//                 Straight-through sign updates of V (per element) and of alpha,
//                 beta (per group: a group lies inside one thread's 256 columns),
//                 the per-row keep-best snapshot, and the next step's D, so the
//                 gradient never goes to memory.
//   kEpiLoss      as kEpiResidual without storing R (final MSE over all rows).
//
// Every mbarrier wait is bounded (GemmArgs::timeout_ns); a role that gives up
// records the timeout in *status and the CTA drains its in-flight copies and
// MMAs before it frees tensor memory and exits.
#include "ar_device.cuh"
#include "ar_internal.h"

namespace ar {

namespace {

constexpr int kStages = 4;
constexpr int kThreads = 192;
constexpr int kTileABytes = kBM * kBK * 2;   // 16 KB
constexpr int kTileBBytes = kBN * kBK * 2;   // 32 KB
constexpr int kStageBytes = kTileABytes + kTileBBytes;
constexpr int kTmemCols = 2 * kBN;           // two accumulators
constexpr int kBarOffset = kStages * kStageBytes;
constexpr int kSmemBytes = kBarOffset + 1024 /* barriers etc. */ + 1024 /* alignment slack */;
constexpr uint32_t kIdesc = umma_idesc_bf16(kBM, kBN);

struct Smem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
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

__device__ __forceinline__ void store_f32x32(float* p, const float (&v)[32]) {
  float4* q4 = reinterpret_cast<float4*>(p);
#pragma unroll
  for (int q = 0; q < 8; ++q) q4[q] = make_float4(v[q * 4 + 0], v[q * 4 + 1], v[q * 4 + 2], v[q * 4 + 3]);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ---------------------------------------------------------------------------
// epilogues
// ---------------------------------------------------------------------------

// R^T tile: optional bf16 store, per-row sum of squares over the valid columns.
template <bool kStore>
__device__ __forceinline__ void epi_residual(const GemmArgs& a, uint32_t t_row, int j, int n0, int n_blk) {
  float sumsq = 0.0f;
  const bool row_ok = j < a.M;
#pragma unroll 1
  for (int c = 0; c < kBN / 32; ++c) {
    const int col0 = n0 + c * 32;
    if (col0 >= a.N) break;  // warp-uniform
    uint32_t r[32];
    __syncwarp();
    tmem_ld_32cols(t_row + c * 32, r);
    tmem_ld_wait();
    if (row_ok) {
      const int nvalid = min(32, a.N - col0);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float v = __uint_as_float(r[i]);
        if (i < nvalid) sumsq = fmaf(v, v, sumsq);
      }
      if (kStore) {
        __nv_bfloat16* dst = a.Rt + static_cast<int64_t>(j) * a.ldr + col0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (q * 8 < nvalid) {  // nvalid is a multiple of 8
            uint4 pk;
            pk.x = pack_bf16x2(__uint_as_float(r[q * 8 + 0]), __uint_as_float(r[q * 8 + 1]));
            pk.y = pack_bf16x2(__uint_as_float(r[q * 8 + 2]), __uint_as_float(r[q * 8 + 3]));
            pk.z = pack_bf16x2(__uint_as_float(r[q * 8 + 4]), __uint_as_float(r[q * 8 + 5]));
            pk.w = pack_bf16x2(__uint_as_float(r[q * 8 + 6]), __uint_as_float(r[q * 8 + 7]));
            reinterpret_cast<uint4*>(dst)[q] = pk;
          }
        }
      }
    }
  }
  if (row_ok) a.part[static_cast<int64_t>(j) * a.part_ld + n_blk] = sumsq;
}

// G tile: the SignSGD update of one step for the rows x columns of this tile.
__device__ __forceinline__ void epi_update(const GemmArgs& a, uint32_t t_row, int j, int n0, int n_blk) {
  const bool row_ok = j < a.M;
  const float Q = qmaxf(a.bits);
  const bool sym = a.sym != 0;
  const int64_t row_base = static_cast<int64_t>(j) * a.N;

  // Per-row batch loss of this step (sum over the residual GEMM's n-tiles, fixed
  // order) and the keep-best decision; identical in every n-tile of the row.
  bool better = false;
  if (row_ok) {
    float L = 0.0f;
    const float* p = a.part_in + static_cast<int64_t>(j) * a.nparts;
    for (int q = 0; q < a.nparts; ++q) L += p[q];
    if (a.keep_best) {
      const float mean = L * a.inv_batch;
      better = mean < a.best_in[j];
      if (n_blk == 0) a.best_out[j] = better ? mean : a.best_in[j];
    }
    if (n_blk == 0) a.rowloss[j] = L;
  }

  const int groups_in_tile = max(1, kBN / a.g);  // g divides 256, or g == N <= 256
  const int chunks_per_group = a.g / 32;
#pragma unroll 1
  for (int gl = 0; gl < groups_in_tile; ++gl) {
    const int gcol0 = n0 + gl * a.g;
    if (gcol0 >= a.N) break;  // warp-uniform
    const int64_t gidx = static_cast<int64_t>(j) * a.G + gcol0 / a.g;

    float wmn = 0.f, wmx = 0.f, al = 1.f, be = 1.f;
    if (row_ok) {
      wmn = a.wmin[gidx];
      wmx = a.wmax[gidx];
      al = a.alpha[gidx];
      be = a.beta[gidx];
    }
    const GroupScale gs = group_scale(wmn, wmx, al, be, a.bits, sym);
    // Straight-through derivatives of s and zp with respect to alpha and beta.
    float ds_a, ds_b, dzp_a = 0.f, dzp_b = 0.f;
    if (sym) {
      ds_a = __fdiv_rn(__fmul_rn(2.0f, fmaxf(-wmn, wmx)), Q);
      ds_b = 0.f;
    } else {
      ds_a = __fdiv_rn(wmx, Q);
      ds_b = __fdiv_rn(-wmn, Q);
      const float z0 = __fdiv_rn(-__fmul_rn(be, wmn), gs.s);
      const float rz = rintf(z0);
      if (rz >= 0.f && rz <= Q) {
        dzp_a = -z0 * ds_a / gs.s;
        dzp_b = -wmn / gs.s - z0 * ds_b / gs.s;
      }
    }

    float dal = 0.f, dbe = 0.f;
#pragma unroll 1
    for (int cc = 0; cc < chunks_per_group; ++cc) {
      const int tcol = gl * a.g + cc * 32;
      uint32_t r[32];
      __syncwarp();
      tmem_ld_32cols(t_row + tcol, r);
      tmem_ld_wait();
      if (!row_ok) continue;  // no warp-collective instruction follows in this iteration
      const int64_t e0 = row_base + n0 + tcol;
      float w[32], v[32], vn[32];
      load_w32(a.W, a.w_bf16, e0, w);
      load_f32x32(a.V + e0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float G = __uint_as_float(r[i]);
        const ElemQuant e = quant_elem(w[i], v[i], gs, Q);
        const float sg = e.m ? sgnf(G) : 0.0f;
        vn[i] = fminf(fmaxf(__fsub_rn(v[i], __fmul_rn(a.lr, sg)), -0.5f), 0.5f);
        float dwa, dwb;
        if (e.m) {
          const float d = e.r - e.u;
          dwa = ds_a * d;
          dwb = ds_b * d;
        } else {
          const float qz = e.q - gs.zp;
          dwa = ds_a * qz - gs.s * dzp_a;
          dwb = ds_b * qz - gs.s * dzp_b;
        }
        dal = fmaf(G, dwa, dal);
        dbe = fmaf(G, dwb, dbe);
      }
      store_f32x32(a.V + e0, vn);
      if (better) store_f32x32(a.V_best + e0, v);
    }
    if (!row_ok) continue;

    const float al_n = fminf(fmaxf(__fsub_rn(al, __fmul_rn(a.mlr, sgnf(dal))), 0.5f), 1.0f);
    const float be_n = sym ? be : fminf(fmaxf(__fsub_rn(be, __fmul_rn(a.mlr, sgnf(dbe))), 0.5f), 1.0f);
    a.alpha[gidx] = al_n;
    a.beta[gidx] = be_n;
    if (better) {
      a.alpha_best[gidx] = al;
      a.beta_best[gidx] = be;
    }

    // D for the next step from the updated state.
    const GroupScale gn = group_scale(wmn, wmx, al_n, be_n, a.bits, sym);
#pragma unroll 1
    for (int cc = 0; cc < chunks_per_group; ++cc) {
      const int64_t e0 = row_base + gcol0 + cc * 32;
      float w[32], v[32];
      load_w32(a.W, a.w_bf16, e0, w);
      load_f32x32(a.V + e0, v);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const ElemQuant e0q = quant_elem(w[2 * i], v[2 * i], gn, Q);
        const ElemQuant e1q = quant_elem(w[2 * i + 1], v[2 * i + 1], gn, Q);
        pk[i] = pack_bf16x2(__fsub_rn(e0q.wq, w[2 * i]), __fsub_rn(e1q.wq, w[2 * i + 1]));
      }
      uint4* dst = reinterpret_cast<uint4*>(a.D + e0);
#pragma unroll
      for (int q = 0; q < 4; ++q) dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
    }
  }
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------

template <int kKind>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ GemmArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Smem* sm = reinterpret_cast<Smem*>(smem + kBarOffset);
  volatile int* abort_flag = &sm->abort_flag;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 1 && lane == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm->tfull[b], 1);
      mbar_init(&sm->tempty[b], 128);
    }
    mbar_init(&sm->drain, 1);
    sm->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&sm->tmem_base, kTmemCols);
    tmem_relinquish();
    if (lane == 0) {
      tma_prefetch_desc(&tmA);
      tma_prefetch_desc(&tmB);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = sm->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_parity = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
        const int m_blk = tile % args.num_m_blk;
        const int n_blk = tile / args.num_m_blk;
        for (int kb = 0; kb < args.num_k_blk; ++kb) {
          if (!mbar_wait(&sm->empty[stage], phase ^ 1, abort_flag, args.status, args.timeout_ns)) {
            ok = false;
            break;
          }
          uint8_t* sA = smem + stage * kStageBytes;
          uint8_t* sB = sA + kTileABytes;
          mbar_arrive_expect_tx(&sm->full[stage], kStageBytes);
          tma_load_2d(sA, &tmA, kb * kBK, m_blk * kBM, &sm->full[stage]);
          tma_load_2d(sB, &tmB, kb * kBK + args.b_k_off, n_blk * kBN + args.b_row_off, &sm->full[stage]);
          issued_mask |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      if (!ok) {
        // Let the copies already issued land before the CTA exits.
        for (int s = 0; s < kStages; ++s)
          if (issued_mask & (1u << s)) mbar_wait_drain(&sm->full[s], (issued_parity >> s) & 1u, args.timeout_ns);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < args.num_tiles; tile += gridDim.x) {
        if (!mbar_wait(&sm->tempty[acc], acc_phase ^ 1, abort_flag, args.status, args.timeout_ns)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * kBN;
        for (int kb = 0; kb < args.num_k_blk; ++kb) {
          if (!mbar_wait(&sm->full[stage], phase, abort_flag, args.status, args.timeout_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * kStageBytes);
          const uint64_t a_desc = umma_desc_sw128(a_addr);
          const uint64_t b_desc = umma_desc_sw128(a_addr + kTileABytes);
#pragma unroll
          for (int k = 0; k < kBK / 16; ++k)
            umma_bf16(d_tmem, a_desc + 2 * k, b_desc + 2 * k, kIdesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(&sm->empty[stage]);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) break;
        umma_commit(&sm->tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1;
      }
      // Every MMA this thread issued has completed once `drain` flips.
      umma_commit(&sm->drain);
      mbar_wait_drain(&sm->drain, 0, args.timeout_ns);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // tensor-memory lanes this warp may access
    const int row_in_tile = quarter * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < args.num_tiles; tile += gridDim.x) {
      const int m_blk = tile % args.num_m_blk;
      const int n_blk = tile / args.num_m_blk;
      if (!mbar_wait(&sm->tfull[acc], acc_phase, abort_flag, args.status, args.timeout_ns)) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + acc * kBN;
      const int j = m_blk * kBM + row_in_tile;
      const int n0 = n_blk * kBN;
      if (kKind == kEpiResidual) epi_residual<true>(args, t_row, j, n0, n_blk);
      if (kKind == kEpiLoss) epi_residual<false>(args, t_row, j, n0, n_blk);
      if (kKind == kEpiUpdate) epi_update(args, t_row, j, n0, n_blk);
      tc_fence_before();
      mbar_arrive(&sm->tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int kKind>
cudaError_t launch_kind(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args, int num_sms,
                        cudaStream_t stream) {
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<kKind>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const int grid = args.num_tiles < num_sms ? args.num_tiles : num_sms;
  if (grid <= 0) return cudaSuccess;
  gemm_kernel<kKind><<<grid, kThreads, kSmemBytes, stream>>>(tmA, tmB, args);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gemm(EpiKind kind, const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmArgs& args,
                        int num_sms, cudaStream_t stream) {
  switch (kind) {
    case kEpiResidual:
      return launch_kind<kEpiResidual>(tmA, tmB, args, num_sms, stream);
    case kEpiUpdate:
      return launch_kind<kEpiUpdate>(tmA, tmB, args, num_sms, stream);
    case kEpiLoss:
      return launch_kind<kEpiLoss>(tmA, tmB, args, num_sms, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ar
