// Device helpers for libar: the fp32 quantiser arithmetic, and thin inline-PTX
// wrappers for sm_100a mbarriers, TMA tile loads and the tcgen05 tensor-core
// instructions (MMA into tensor memory, commit, tensor-memory loads).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ar {

// ---------------------------------------------------------------------------
// Quantiser arithmetic ("[llm-compressor] AutoRound ...", "논문 핵심 내용" and
// _fake_quantize_with_offset).  Every operation is a single IEEE fp32 operation
// with round-to-nearest-even, written with the _rn intrinsics so the compiler
// cannot contract or reorder them.  rintf rounds half to even (torch.round).
// ---------------------------------------------------------------------------

struct GroupScale {
  float s;    // scale
  float zp;   // zero-point (integer-valued)
  float rcp;  // 1/s correctly rounded (for div_rn_by)
};

__device__ __forceinline__ float qmaxf(int bits) { return (float)((1 << bits) - 1); }

// Scale and zero-point of one group from its min/max statistics and clip factors.
__device__ __forceinline__ GroupScale group_scale(float wmin, float wmax, float alpha,
                                                  float beta, int bits, bool sym) {
  const float Q = qmaxf(bits);
  GroupScale g;
  if (sym) {
    const float amax = fmaxf(-wmin, wmax);
    g.s = __fdiv_rn(__fmul_rn(2.0f, __fmul_rn(alpha, amax)), Q);
    if (g.s == 0.0f) g.s = 1.0f;
    g.zp = (float)(1 << (bits - 1));
  } else {
    g.s = __fdiv_rn(__fsub_rn(__fmul_rn(alpha, wmax), __fmul_rn(beta, wmin)), Q);
    if (g.s == 0.0f) g.s = 1.0f;
    g.zp = fminf(fmaxf(rintf(__fdiv_rn(-__fmul_rn(beta, wmin), g.s)), 0.0f), Q);
  }
  g.rcp = __frcp_rn(g.s);
  return g;
}

// Weights whose quotients by their group's scale div_rn_by may form: zero, or
// 2^-100 <= |w| <= 2^20.  With every weight of a group in that range the scale is a
// normal number below 2^21, and each quotient and each residual w - s*q of the
// division is a normal number.
__device__ __forceinline__ bool div_fast_ok(float w) {
  const float m = fabsf(w);
  return w == 0.0f || (m >= 0x1p-100f && m <= 0x1p20f);
}

// a / b correctly rounded, from y = 1/b correctly rounded, by one residual
// correction (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990; also Muller et al.,
// Handbook of Floating-Point Arithmetic, ch. "Newton-Raphson-based division with
// an FMA"): q = RN(a y) is within one ulp of a/b, the residual q b - a is exact in
// one fma, and RN(q - (q b - a) y) is the correctly rounded quotient.  (Writing the
// residual as q b - a keeps the sign of a zero quotient.)  Valid for b > 0 when
// a/b and the residual are normal numbers: for div_fast_ok weights divided by
// their group's (positive) scale.
__device__ __forceinline__ float div_rn_by(float a, float b, float y) {
  const float q = __fmul_rn(a, y);
  const float r = __fmaf_rn(q, b, -a);
  return __fmaf_rn(-r, y, q);
}

struct ElemQuant {
  float u;   // W / s
  float r;   // rint(W/s + V)
  float q;   // clamp(r + zp, 0, Q): the code
  bool m;    // 0 <= r + zp <= Q: the clamp passes the gradient
  float wq;  // s * (q - zp)
};

// fast: every weight of the layer is div_fast_ok, so W/s may use div_rn_by.
__device__ __forceinline__ ElemQuant quant_elem(float w, float v, GroupScale g, float Q, bool fast = false) {
  ElemQuant e;
  e.u = fast ? div_rn_by(w, g.s, g.rcp) : __fdiv_rn(w, g.s);
  e.r = rintf(__fadd_rn(e.u, v));
  const float p = __fadd_rn(e.r, g.zp);
  e.q = fminf(fmaxf(p, 0.0f), Q);
  e.m = (p >= 0.0f) && (p <= Q);
  e.wq = __fmul_rn(g.s, __fsub_rn(e.q, g.zp));
  return e;
}

__device__ __forceinline__ float sgnf(float x) { return (x > 0.0f) ? 1.0f : ((x < 0.0f) ? -1.0f : 0.0f); }

// Straight-through derivatives of a group's scale and zero-point with respect to
// its clip factors ("[llm-compressor] AutoRound ...": rint treated as identity,
// a clamp passing the gradient inside its range).
struct GroupDeriv {
  float ds_a, ds_b;    // ds/d alpha, ds/d beta
  float dzp_a, dzp_b;  // dzp/d alpha, dzp/d beta (0 when zp is clamped, and when symmetric)
};

__device__ __forceinline__ GroupDeriv group_deriv(float wmn, float wmx, float be, const GroupScale& gs, float Q,
                                                  bool sym) {
  GroupDeriv d;
  d.dzp_a = 0.f;
  d.dzp_b = 0.f;
  if (sym) {
    d.ds_a = __fdiv_rn(__fmul_rn(2.0f, fmaxf(-wmn, wmx)), Q);
    d.ds_b = 0.f;
  } else {
    d.ds_a = __fdiv_rn(wmx, Q);
    d.ds_b = __fdiv_rn(-wmn, Q);
    const float z0 = __fdiv_rn(-__fmul_rn(be, wmn), gs.s);
    const float rz = rintf(z0);
    if (rz >= 0.f && rz <= Q) {
      d.dzp_a = -z0 * d.ds_a / gs.s;
      d.dzp_b = -wmn / gs.s - z0 * d.ds_b / gs.s;
    }
  }
  return d;
}

// A clip factor after one sign step of size mlr against its gradient, clamped to
// [0.5, 1].
__device__ __forceinline__ float clip_step(float c, float mlr, float grad) {
  return fminf(fmaxf(__fsub_rn(c, __fmul_rn(mlr, sgnf(grad))), 0.5f), 1.0f);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(((uint32_t)b) << 16);
}

// ---------------------------------------------------------------------------
// Shared-memory addresses, mbarriers, bounded waits.
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Same test with acquire semantics at cluster scope: for barriers whose phase is
// completed by the peer CTA of a pair (remote arrivals, the peer's TMA bytes).
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar_addr, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return ok != 0;
}

// Device status words (first int of the workspace).
enum : int { kDevOk = 0, kDevTimeout = 5, kDevCheck = 6 };

// Bounds check of the AR_CHECKS mode: true if [idx, idx + n) lies inside a buffer
// of cap elements, or if checks are off (cap == 0).  Otherwise records kDevCheck
// in *status (the first error recorded stays) and returns false: the caller skips
// the access.  Never traps.
__device__ __forceinline__ bool in_bounds(int64_t idx, int n, int64_t cap, int* status) {
  if (cap == 0 || (idx >= 0 && idx + n <= cap)) return true;
  if (status) atomicCAS(status, kDevOk, kDevCheck);
  return false;
}

// Wait until the phase with the given parity of `bar` has completed.  Gives up
// after timeout_ns (checked every few hundred polls), or as soon as another role
// of the CTA has given up (*abort != 0); on giving up it records kDevTimeout in
// *status, raises *abort and returns false.
// With kCluster the test acquires at cluster scope.  With use_abort false the
// wait ignores *abort and ends only on completion or its own timeout, so that
// warps waiting on the same phase always take the same decision.
template <bool kCluster = false>
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status, uint64_t timeout_ns, bool use_abort = true) {
  const uint32_t addr = smem_u32(bar);
  auto test = [&]() { return kCluster ? mbar_try_wait_cluster(addr, parity) : mbar_try_wait(addr, parity); };
#pragma unroll 1
  for (int i = 0; i < 32; ++i)
    if (test()) return true;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 256; ++i)
      if (test()) return true;
    if (use_abort && *abort) return false;
    if (globaltimer_ns() - t0 > timeout_ns) {
      atomicCAS(status, kDevOk, kDevTimeout);
      *abort = 1;
      return false;
    }
  }
}

// Same wait without an abort flag, for the drain phase after an abort.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  while (!mbar_try_wait(addr, parity)) {
    if (globaltimer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// ---------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor) tile loads, no multicast.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Load the box at (x = inner coordinate, y = row) into shared memory; completes
// `bytes` of transaction count on `bar`.  x * 2 bytes must be a multiple of 16.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------------------
// Thread-block clusters of two CTAs (the tcgen05 cta_group::2 pair).
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

// Every thread of both CTAs: release this CTA's prior writes, acquire the peer's.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Arrive (release, cluster scope) on an mbarrier given by its shared::cluster address.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is counted on the
// pair leader's mbarrier (`leader_bar` is a shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map, int32_t x, int32_t y,
                                                 uint32_t leader_bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(leader_bar)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads.
// ---------------------------------------------------------------------------

__device__ __forceinline__ void tmem_alloc(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// Pair versions (cta_group::2): one warp of each CTA allocates the same columns in
// both CTAs' tensor memory; the leader's thread issues an M = 256 MMA whose A rows
// and B columns are split between the two CTAs' shared memory, each CTA's tensor
// memory holding its 128 accumulator rows.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_result, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_result)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// The same MMA with the A collector buffer: kFill reads A from shared memory and
// keeps it in the tensor core's A collector; !kFill (lastuse) takes A from the
// collector, filled by the MMA issued just before with the same A descriptor, and
// releases it.  Two products that share their A tile read it from shared memory once.
template <bool kFill>
__device__ __forceinline__ void umma_bf16_pair_collect(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                       uint32_t idesc, uint32_t accumulate) {
  if (kFill)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::fill [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16.collector::a::lastuse [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the mbarrier at the same shared-memory offset in both CTAs of the pair
// once the pair MMAs issued so far have completed.
__device__ __forceinline__ void umma_commit_pair_both(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}

// Arrive on this CTA's mbarrier only.
__device__ __forceinline__ void umma_commit_pair_local(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D, both
// operands K-major, tile M x N.
// Instruction-descriptor bits that mark A (bit 15) or B (bit 16) as MN-major.
constexpr uint32_t kIdescAMn = 1u << 15;
constexpr uint32_t kIdescBMn = 1u << 16;

__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4)                          // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Shared-memory matrix descriptor for a K-major operand tile stored as rows of
// 64 bf16 (128 bytes) in the 128-byte swizzle pattern that TMA writes with
// CU_TENSOR_MAP_SWIZZLE_128B; eight-row core groups are 1024 bytes apart.  The
// tile base must be 1024-byte aligned.  Advancing K by 16 elements inside the
// 128-byte row adds 32 bytes (2 units) to the start address.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);   // start address
  d |= (uint64_t)1 << 16;                        // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1 << 46;                        // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                        // layout: 128-byte swizzle
  return d;
}

// Shared-memory matrix descriptor for an MN-major operand tile (the operand read
// from a row-major [K, M or N] tensor without a transpose).  TMA writes it as
// 64 x 64 boxes in the 128-byte swizzle pattern: each box holds 64 K rows of 64
// consecutive M (or N) elements, 128 bytes a row, 8 KB a box.  In the canonical
// MN-major layout the 64-element blocks along M or N are then 8 KB apart (leading
// byte offset) and the eight-row K groups 1 KB apart (stride byte offset).
// Advancing K by 16 rows adds 2 KB (128 units) to the start address.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);   // start address
  d |= (uint64_t)(8192 >> 4) << 16;              // leading byte offset: next 64 along M/N
  d |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: next 8 K rows
  d |= (uint64_t)1 << 46;                        // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                        // layout: 128-byte swizzle
  return d;
}

// 32 consecutive fp32 columns of one tensor-memory lane per thread (lane = warp's
// 32-lane slice + thread index).
__device__ __forceinline__ void tmem_ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 16 consecutive fp32 columns of one tensor-memory lane per thread.
__device__ __forceinline__ void tmem_ld_16cols(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Ask L2 to fetch [p, p + bytes) from memory (p 16-byte aligned, bytes a multiple
// of 16).  A hint: nothing waits for it.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Store 32 consecutive columns of this warp's 32 lanes into tensor memory (the
// counterpart of tmem_ld_32cols); tmem_st_wait orders them before later accesses.
__device__ __forceinline__ void tmem_st_32cols(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
      :
      : "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

}  // namespace ar
