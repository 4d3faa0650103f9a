// Thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers (with bounded waits), TMA tensor loads, and the 5th-generation
// tensor core (tcgen05: TMEM allocation, MMA, commit, TMEM loads/stores).
//
// Every wait here is bounded by wall-clock time (%globaltimer); a wait that
// runs out returns false so the caller can record an error and leave.
#pragma once
#include <cstdint>
#include <cuda.h>

namespace sa {

// Status bits a kernel may OR into the caller's device status word.
enum : uint32_t {
  kDevErrTimeoutLoad = 1u << 0,   // a wait for TMA data ran out
  kDevErrTimeoutMma = 1u << 1,    // a wait for tensor-core results ran out
  kDevErrTimeoutSoftmax = 1u << 2,// a wait for the softmax warps ran out
  kDevErrBadIndex = 1u << 3,      // a block index outside [0, nb)
};

// ~1 second; long enough for any legitimate wait, short enough to keep a
// broken pipeline from holding the GPU.
constexpr uint64_t kWaitLimitNs = 1000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the async proxy (TMA, tensor core).
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Arrive without release ordering: the thread's earlier memory operations
// (e.g. global reductions still in flight) are not waited for. Only for
// barriers that guard TMEM accesses the thread has already completed
// (tcgen05.wait::ld / ::st before the arrive).
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t* bar) {
  asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of the phase (no suspend window).
__device__ __forceinline__ bool mbar_peek(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking probe of three barriers at once: the three test_waits issue
// back to back, so their shared-memory latency is paid once. Bit i of the
// result is set when barrier i's phase with parity i has completed.
__device__ __forceinline__ uint32_t mbar_peek3(uint64_t* b0, uint32_t p0, uint64_t* b1, uint32_t p1,
                                               uint64_t* b2, uint32_t p2) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred q0, q1, q2;\n\t.reg .u32 t0, t1, t2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q0, [%1], %2;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q1, [%3], %4;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 q2, [%5], %6;\n\t"
      "selp.u32 t0, 1, 0, q0;\n\t"
      "selp.u32 t1, 2, 0, q1;\n\t"
      "selp.u32 t2, 4, 0, q2;\n\t"
      "or.b32 t0, t0, t1;\n\t"
      "or.b32 %0, t0, t2;\n\t}"
      : "=r"(r)
      : "r"(smem_u32(b0)), "r"(p0), "r"(smem_u32(b1)), "r"(p1), "r"(smem_u32(b2)), "r"(p2)
      : "memory");
  return r;
}

// Waits until the barrier's phase with the given parity has completed.
// Gives up after kWaitLimitNs, or early once *abort is non-zero.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          const volatile int* abort) {
  if (mbar_peek(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_test(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3), "r"(c4)
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// Untiled bulk copy global -> shared (both 16-byte aligned, bytes a multiple
// of 16), completing on *bar's transaction count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// *p += (a, b, c, d) as one vector reduction (relaxed, GPU scope).
__device__ __forceinline__ void red_add_f32x4(float* p, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(a), "f"(b), "f"(c),
               "f"(d)
               : "memory");
}

// Generic-proxy writes to shared memory -> visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05
// Allocation is warp-wide; the TMEM base address is written to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulation.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Eight back-to-back MMAs over K = 8 x 16 in one asm block (no compiler
// instructions between them): D[tmem] (+)= A * B^T with A and B both
// 128-byte-swizzled K-major shared-memory tiles whose 64-element K chunks are
// kChunk bytes apart. Descriptors are passed as 32-bit halves; the per-MMA
// offsets move only the start-address field (low word, no carry). The first
// MMA accumulates iff acc != 0, the other seven always do.
template <uint32_t kChunk>
__device__ __forceinline__ void mma_ss_k8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t acc) {
  const uint32_t alo = uint32_t(a_desc), ahi = uint32_t(a_desc >> 32);
  const uint32_t blo = uint32_t(b_desc), bhi = uint32_t(b_desc >> 32);
#define SA_MMA_SS_STEP(KK, PRED)                                                     \
  "add.u32 la, %1, " #KK ";\n\t"                                                   \
  "add.u32 lb, %3, " #KK ";\n\t"                                                   \
  "mov.b64 da, {la, %2};\n\t"                                                      \
  "mov.b64 db, {lb, %4};\n\t"                                                      \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], da, db, %5, " PRED ";\n\t"
  asm volatile(
      "{\n\t.reg .pred p0, p1;\n\t.reg .u32 la, lb;\n\t.reg .b64 da, db;\n\t"
      "setp.ne.b32 p0, %6, 0;\n\t"
      "setp.eq.b32 p1, 0, 0;\n\t"
      SA_MMA_SS_STEP(%7, "p0") SA_MMA_SS_STEP(%8, "p1") SA_MMA_SS_STEP(%9, "p1")
      SA_MMA_SS_STEP(%10, "p1") SA_MMA_SS_STEP(%11, "p1") SA_MMA_SS_STEP(%12, "p1")
      SA_MMA_SS_STEP(%13, "p1") SA_MMA_SS_STEP(%14, "p1") "}"
      ::"r"(d_tmem), "r"(alo), "r"(ahi), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc),
      "n"(0), "n"(2), "n"(4), "n"(6), "n"(kChunk / 16), "n"(kChunk / 16 + 2),
      "n"(kChunk / 16 + 4), "n"(kChunk / 16 + 6)
      : "memory");
#undef SA_MMA_SS_STEP
}

// NK (4 or 8) back-to-back MMAs with A from TMEM (8 columns of bf16 pairs per
// K step of 16) and B an MN-major shared-memory tile advancing 2048 bytes per
// K step; the first accumulates iff acc != 0, the others always do.
template <int NK>
__device__ __forceinline__ void mma_ts_k(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                         uint32_t idesc, uint32_t acc) {
  static_assert(NK == 4 || NK == 8, "NK is 4 or 8");
  const uint32_t blo = uint32_t(b_desc), bhi = uint32_t(b_desc >> 32);
#define SA_MMA_TS_STEP(TOFF, BOFF, PRED)                                             \
  "add.u32 ta, %1, " #TOFF ";\n\t"                                                  \
  "add.u32 lb, %2, " #BOFF ";\n\t"                                                  \
  "mov.b64 db, {lb, %3};\n\t"                                                      \
  "tcgen05.mma.cta_group::1.kind::f16 [%0], [ta], db, %4, " PRED ";\n\t"
  if constexpr (NK == 8) {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 ta, lb;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p0, %5, 0;\n\t"
        "setp.eq.b32 p1, 0, 0;\n\t"
        SA_MMA_TS_STEP(0, 0, "p0") SA_MMA_TS_STEP(8, 128, "p1") SA_MMA_TS_STEP(16, 256, "p1")
        SA_MMA_TS_STEP(24, 384, "p1") SA_MMA_TS_STEP(32, 512, "p1") SA_MMA_TS_STEP(40, 640, "p1")
        SA_MMA_TS_STEP(48, 768, "p1") SA_MMA_TS_STEP(56, 896, "p1") "}"
        ::"r"(d_tmem), "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc)
        : "memory");
  } else {
    asm volatile(
        "{\n\t.reg .pred p0, p1;\n\t.reg .b32 ta, lb;\n\t.reg .b64 db;\n\t"
        "setp.ne.b32 p0, %5, 0;\n\t"
        "setp.eq.b32 p1, 0, 0;\n\t"
        SA_MMA_TS_STEP(0, 0, "p0") SA_MMA_TS_STEP(8, 128, "p1") SA_MMA_TS_STEP(16, 256, "p1")
        SA_MMA_TS_STEP(24, 384, "p1") "}"
        ::"r"(d_tmem), "r"(a_tmem), "r"(blo), "r"(bhi), "r"(idesc), "r"(acc)
        : "memory");
  }
#undef SA_MMA_TS_STEP
}

// Arrives once on *bar when every tensor-core op issued so far by this thread
// has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
// a_mn / b_mn select MN-major (1) instead of K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, int a_mn, int b_mn) {
  return (1u << 4)                            // D format: f32
         | (1u << 7)                          // A format: bf16
         | (1u << 10)                         // B format: bf16
         | (uint32_t(a_mn) << 15) | (uint32_t(b_mn) << 16) |
         (uint32_t(N >> 3) << 17)             // N / 8
         | (uint32_t(M >> 4) << 24);          // M / 16
}

// Shared-memory operand descriptor for a 128-byte-swizzled bf16 tile
// (the layout TMA writes with CU_TENSOR_MAP_SWIZZLE_128B: rows of 128 bytes,
// 8-row / 1024-byte swizzle atoms). For K-major operands lbo is unused and
// sbo is the byte stride between 8-row groups; for MN-major operands lbo is
// the stride between 64-element column chunks and sbo the stride between
// groups of 8 K-rows.
// Instruction descriptor, kind::tf32 with TF32 A/B (format code 2, as the
// CUTLASS UMMA descriptor defines it) and fp32 D, both operands K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int M, int N) {
  return (1u << 4)                            // D format: f32
         | (2u << 7)                          // A format: tf32
         | (2u << 10)                         // B format: tf32
         | (uint32_t(N >> 3) << 17)           // N / 8
         | (uint32_t(M >> 4) << 24);          // M / 16
}

// D[tmem] (+)= A[smem] * B[smem]^T on 32-bit TF32 operands (K = 8 per MMA).
__device__ __forceinline__ void mma_tf32_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return uint64_t((saddr & 0x3FFFFu) >> 4) | (uint64_t((lbo >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo >> 4) & 0x3FFFu) << 32) | (uint64_t(1) << 46)  // sm100 descriptor
         | (uint64_t(2) << 61);                                         // SWIZZLE_128B
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (warp's quadrant base + i), columns [col, col + 32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
      "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %2, %1;" : "=r"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Warpgroup-wide register reallocation; every warp of the warpgroup must
// execute the same call.
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

__device__ __forceinline__ void named_barrier_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

}  // namespace sa
