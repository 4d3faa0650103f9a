// Mask build (NABLA, Metodologia 2 "Attenzione Ridotta" + "CDF Thresholding",
// Metodologia 3 STA union), three kernels after the pooling:
//
//  logits_tc_kernel  L[bh][r][j] = Qbar[r] . Kbar[j] / sqrt(d) for every pair
//                 of blocks of a head on the TF32 tensor cores (three products
//                 of a hi / lo split: fp32-level accuracy), a persistent
//                 kernel over 128 x 256 output tiles, stored in the workspace;
//  select_kernel  one warp per q-block row, the row held in registers:
//                 softmax, then the CDF threshold without sorting. k-block j
//                 is kept iff the probability mass ranked before it (descending
//                 order, ties by index) is < 1 - thr. With masses in 2^-30
//                 fixed point (integer sums, so the result is bit-identical
//                 run to run), a leading-bit histogram and a bitwise search
//                 over the compacted octave find the mass tau of the last
//                 kept block; of
//                 the blocks whose mass equals tau, those that keep the
//                 running mass below the threshold are kept in ascending index
//                 order. Then the OR with the static STA window, the ascending
//                 kept list and the row's keep bitmap (select_pair_kernel:
//                 the same with two warps per row, for rows of 1025..2048
//                 blocks);
//  union_kernel   one warp per query tile (two q-blocks): the union of the
//                 two bitmaps as a list of k-blocks tagged with which q-block
//                 keeps each, first the steps that pair one patch in frames t
//                 and t+1 (one two-frame TMA box each in the attention
//                 kernel), then the remaining blocks in ascending order.
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

namespace {

constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ void fail_status(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// ------------------------------------------------------------------ logits
// L = Qbar Kbar^T / sqrt(d) per head on the TF32 tensor cores, in three
// products of the pooled means' hi / lo split (hi*hi + hi*lo + lo*hi), fp32
// accumulation in TMEM. A persistent kernel, one CTA per SM, walks the
// 128 x 256 output tiles (column tiles fastest, so neighbouring CTAs share
// the query rows in L2): warp 0 loads 32-channel K-chunks of the four
// operands by TMA into a 2-stage ring, warp 1 issues the MMAs (M=128, N=256,
// K=8) into one of two TMEM accumulators, and warps 2-5 read the other one,
// scale it and store it (staged through shared memory, 32 x 32 per warp, so
// that the global stores are whole 128-byte rows) while the next tile's
// products run.
constexpr int kLtM = 128, kLtN = 256, kLtK = 32;  // tile rows, columns, K-chunk (128 B of fp32)
constexpr int kLtThreads = 192;
constexpr int kLtStagePitch = 36;  // floats per staged 32-column row (float4 stores conflict-free)
constexpr uint32_t kLtStageBytes = 2u * kLtM * kLtK * 4u + 2u * kLtN * kLtK * 4u;  // 96 KB

struct __align__(1024) LogitsSmem {
  float a[2][2][kLtM * kLtK];  // [stage][hi, lo]: 128 rows x 128 B, 128-byte swizzle
  float b[2][2][kLtN * kLtK];  // [stage][hi, lo]: 256 rows x 128 B
  float out[4][32 * kLtStagePitch];  // per epilogue warp: 32 rows x 32 columns
  uint64_t full[2], empty[2], acc_full[2], acc_empty[2], drain;
  uint32_t tmem_base;
  int abort;
};

struct LtTile {
  int bh, r0, c0;
};
__device__ __forceinline__ LtTile lt_tile(int t, int nrt, int nct) {
  const int ct = t % nct, rest = t / nct;
  return {rest / nrt, (rest % nrt) * kLtM, ct * kLtN};
}

template <int D>
__global__ void __launch_bounds__(kLtThreads, 1)
    logits_tc_kernel(const __grid_constant__ MaskArgs a, Geometry g, int ld) {
  extern __shared__ uint8_t lt_raw[];
  LogitsSmem& sm = *reinterpret_cast<LogitsSmem*>(
      (reinterpret_cast<uintptr_t>(lt_raw) + 1023) & ~uintptr_t(1023));
  constexpr int kChunks = D / kLtK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nrt = (g.nb + kLtM - 1) / kLtM, nct = ld / kLtN;
  const int ntiles = g.BH * nrt * nct;
  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], 4);  // one arrival per epilogue warp
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&a.map_qhi);
      prefetch_tensormap(&a.map_qlo);
      prefetch_tensormap(&a.map_khi);
      prefetch_tensormap(&a.map_klo);
      int q = 0, issued = -1;  // chunks over this CTA's tiles
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x) {
        const LtTile tl = lt_tile(t, nrt, nct);
        const int row_base = tl.bh * g.nb;  // first row of this head in the [BH*nb][d] operands
        for (int c = 0; c < kChunks; ++c, ++q) {
          const int s = q & 1;
          if (q >= 2 && !mbar_wait(&sm.empty[s], ((q >> 1) - 1) & 1, abort)) {
            if (!*abort) fail_status(a.status, &sm.abort, kDevErrTimeoutLoad);
            break;
          }
          if (*abort) break;
          mbar_arrive_expect_tx(&sm.full[s], kLtStageBytes);
          tma_load_2d(sm.a[s][0], &a.map_qhi, &sm.full[s], c * kLtK, row_base + tl.r0);
          tma_load_2d(sm.a[s][1], &a.map_qlo, &sm.full[s], c * kLtK, row_base + tl.r0);
          tma_load_2d(sm.b[s][0], &a.map_khi, &sm.full[s], c * kLtK, row_base + tl.c0);
          tma_load_2d(sm.b[s][1], &a.map_klo, &sm.full[s], c * kLtK, row_base + tl.c0);
          issued = q;
        }
      }
      if (*abort) {  // let this thread's copies land before the CTA can exit
        int never = 0;
        for (int c = issued; c >= 0 && c > issued - 2; --c)
          mbar_wait(&sm.full[c & 1], (c >> 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_tf32_f32(kLtM, kLtN);
      bool ok = true;
      int q = 0, i = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++i) {
        const int buf = i & 1;
        if (i >= 2) ok = mbar_wait(&sm.acc_empty[buf], ((i >> 1) - 1) & 1, abort);
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t acc = tmem + uint32_t(buf * kLtN);
        for (int c = 0; c < kChunks; ++c, ++q) {
          const int s = q & 1;
          ok = mbar_wait(&sm.full[s], (q >> 1) & 1, abort);
          if (!ok) break;
          tc_fence_after_sync();
          const uint64_t ahi = sw128_desc(smem_u32(sm.a[s][0]), 16, 1024);
          const uint64_t alo = sw128_desc(smem_u32(sm.a[s][1]), 16, 1024);
          const uint64_t bhi = sw128_desc(smem_u32(sm.b[s][0]), 16, 1024);
          const uint64_t blo = sw128_desc(smem_u32(sm.b[s][1]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kLtK / 8; ++kk) {  // K = 8 tf32 = 32 B per MMA
            const uint32_t off = uint32_t(kk) * 2u;  // 32 B in 16-byte units
            mma_tf32_ss(acc, ahi + off, bhi + off, idesc, (c | kk) != 0 ? 1u : 0u);
            mma_tf32_ss(acc, ahi + off, blo + off, idesc, 1u);
            mma_tf32_ss(acc, alo + off, bhi + off, idesc, 1u);
          }
          mma_commit(&sm.empty[s]);
        }
        if (ok) mma_commit(&sm.acc_full[buf]);
      }
      if (!ok && !*abort) fail_status(a.status, &sm.abort, kDevErrTimeoutMma);
      // no MMA of this thread may be in flight when the TMEM is freed
      mma_commit(&sm.drain);
      int never = 0;
      mbar_wait(&sm.drain, 0, &never);
    }
  } else {
    // epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 = tile rows
    const int quad = warp & 3;
    float* stage = sm.out[warp - 2];
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      const int buf = i & 1;
      const bool ok = __all_sync(kFull, mbar_wait(&sm.acc_full[buf], (i >> 1) & 1, abort));
      if (!ok || *abort) {
        if (lane == 0 && !*abort) fail_status(a.status, &sm.abort, kDevErrTimeoutMma);
        break;
      }
      tc_fence_after_sync();
      const LtTile tl = lt_tile(t, nrt, nct);
      const uint32_t t_row = tmem + (uint32_t(quad * 32) << 16) + uint32_t(buf * kLtN);
      const int row0 = tl.r0 + quad * 32;  // this warp's first tile row
      float* out = a.logits + (size_t(tl.bh) * g.nb + row0) * ld + tl.c0;
#pragma unroll 1
      for (int cc = 0; cc < kLtN / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(t_row + 32 * cc, v);
        tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(stage + lane * kLtStagePitch);
#pragma unroll
        for (int k = 0; k < 8; ++k)
          dst[k] = make_float4(__uint_as_float(v[4 * k]) * a.scale,
                               __uint_as_float(v[4 * k + 1]) * a.scale,
                               __uint_as_float(v[4 * k + 2]) * a.scale,
                               __uint_as_float(v[4 * k + 3]) * a.scale);
        __syncwarp();
        // four whole 128-byte row segments per store instruction
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = 4 * k + (lane >> 3), c4 = lane & 7;
          if (row0 + rr < g.nb)
            reinterpret_cast<float4*>(out + size_t(rr) * ld + 32 * cc)[c4] =
                reinterpret_cast<const float4*>(stage + rr * kLtStagePitch)[c4];
        }
        __syncwarp();
      }
      tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[buf]);
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ select
constexpr int kSelWarps = 8;
constexpr int kCandCap = 256;      // compacted search window per warp (8 per lane)
constexpr int kMaxRowWords = 192;  // keep-bitmap words of a row (nb <= 6144)
constexpr int kRegVPL = 96;        // longest row held in registers (nb <= 3072)
// Per-warp shared work area, used in turn by the leading-bit histogram
// (32 buckets x 32 lanes, words 0..1023), then the packed window (words
// 0..255) and the keep bitmap (256..447).
constexpr int kSelWork = 32 * 32;
constexpr int kDenseAt = 0;
constexpr int kRbitsAt = kDenseAt + kCandCap;
static_assert(kRbitsAt + kMaxRowWords <= kSelWork, "select work area");

// A row's integer masses, VPL per lane (column j in lane j % 32, slot
// j / 32): in registers, or, for rows too long for the register file, in the
// warp's own shared-memory slice [VPL][32].
template <int VPL, bool kSmem>
struct RowStore;
template <int VPL>
struct RowStore<VPL, false> {
  uint32_t v[VPL];
  __device__ __forceinline__ uint32_t get(int i) const { return v[i]; }
  __device__ __forceinline__ void set(int i, uint32_t x) { v[i] = x; }
};
template <int VPL>
struct RowStore<VPL, true> {
  uint32_t* p;  // this lane's column of the slice
  __device__ __forceinline__ uint32_t get(int i) const { return p[i * 32]; }
  __device__ __forceinline__ void set(int i, uint32_t x) { p[i * 32] = x; }
};

// Sum over the warp of the masses >= c; eight independent partial sums keep
// the adds pipelined. (The sum of the masses > c is the one at c + 1.)
template <int N, class Store>
__device__ __forceinline__ uint32_t mass_at_least(const Store& m, uint32_t c) {
  constexpr int kAcc = N < 8 ? N : 8;
  uint32_t acc[kAcc];
#pragma unroll
  for (int i = 0; i < kAcc; ++i) acc[i] = 0u;
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const uint32_t x = m.get(i);
    acc[i % kAcc] += x >= c ? x : 0u;
  }
#pragma unroll
  for (int w = 1; w < kAcc; w <<= 1)
#pragma unroll
    for (int i = 0; i + w < kAcc; i += 2 * w) acc[i] += acc[i + w];
  return __reduce_add_sync(kFull, acc[0]);
}

// The bits of tau below its leading bit e, one by one, over the packed
// window (wcnt masses in [2^e, 2^(e+1)), N per lane: the first n0 in d0, the
// rest in d1); `above` is the mass above the window. Also counts the masses
// equal to tau.
template <int N>
__device__ __forceinline__ void window_search(const uint32_t* d0, int n0, const uint32_t* d1,
                                              int wcnt, int lane, int e, uint32_t above,
                                              uint32_t tgt, uint32_t& tau, uint32_t& keep_ties,
                                              uint32_t& n_tau) {
  RowStore<N, false> cwr;
#pragma unroll
  for (int k = 0; k < N; ++k) {
    const int at = 32 * k + lane;
    // 0 is below every candidate
    cwr.set(k, at < n0 ? d0[at] : (at < wcnt ? d1[at - n0] : 0u));
  }
  uint32_t x = 1u << e;
#pragma unroll 1
  for (int b = e - 1; b >= 0; --b) {
    const uint32_t t = x | (1u << b);
    if (above + mass_at_least<N>(cwr, t) >= tgt) x = t;
  }
  tau = x;
  uint32_t eq = 0;
#pragma unroll
  for (int k = 0; k < N; ++k) eq += cwr.get(k) == tau ? 1u : 0u;
  n_tau = __reduce_add_sync(kFull, eq);
  keep_ties = (tgt - above - mass_at_least<N>(cwr, tau + 1) + tau - 1) / tau;
}

// VPL = values per lane: column j of the row sits in lane j % 32, slot j / 32.
// kSmem: the masses live in dynamic shared memory (VPL * 32 words per warp).
template <int VPL, bool kSmem>
__global__ void __launch_bounds__(kSelWarps * 32, VPL <= 32 ? 4 : (VPL <= 64 ? 2 : 1))
    select_kernel(const float* __restrict__ L, MaskArgs a, Geometry g, int ld) {
  __shared__ __align__(16) uint32_t work_all[kSelWarps][kSelWork];
  extern __shared__ uint32_t sel_slice[];  // kSmem only: [warp][VPL][32]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long row = long(blockIdx.x) * kSelWarps + warp;
  if (row >= long(g.BH) * g.nb) return;
  const int nb = g.nb;
  const int qb = int(row % nb);
  const float* Lr = L + size_t(row) * ld;
  uint32_t* work = work_all[warp];
  constexpr float kLog2e = 1.4426950408889634f;

  // ---- row softmax; each probability as an integer mass m = p * 2^30
  // (the same operations, in the same order, whichever storage holds them)
  RowStore<VPL, kSmem> m;
  if constexpr (kSmem) m.p = sel_slice + size_t(warp) * VPL * 32 + lane;
  {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const int j = lane + 32 * i;
      const float v = j < nb ? __ldg(Lr + j) : -INFINITY;
      m.set(i, __float_as_uint(v));
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    const float shift = -mx * kLog2e;
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      // exactly 0 in the padding slots
      const float v = ex2_approx(fmaf(__uint_as_float(m.get(i)), kLog2e, shift));
      m.set(i, __float_as_uint(v));
      sum += v;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    const float to_fx = 1073741824.0f / sum;  // 2^30 / sum
#pragma unroll
    for (int i = 0; i < VPL; ++i) m.set(i, __float2uint_rn(__uint_as_float(m.get(i)) * to_fx));
  }

  // ---- CDF threshold. In descending mass order (ties by index), block j is
  // kept iff the mass ranked before it is < target. tau, the mass of the last
  // kept block, is the largest x with G(x) = (sum of the masses >= x) >=
  // target; G does not increase with x, so tau is one of the masses.
  //  1. The leading bit e of tau from one histogram of the masses by leading
  //     bit (each lane adds into its own column of a 32 x 32 table; lane b
  //     then sums row b, and a suffix scan over the lanes gives G(2^b) in
  //     lane b): e is the highest b with G(2^b) >= target, and G(2^(e+1)),
  //     the mass above the window [2^e, 2^(e+1)), comes with it.
  //  2. The window's masses are compacted to shared memory (if at most 256)
  //     and the lower bits of tau found one by one over them alone (1, 2, 4
  //     or 8 per lane), the mass
  //     above the window entering as a constant; a longer window is searched
  //     bit by bit over the whole row.
  // Blocks with mass > tau are kept, and of those with mass == tau the first
  // ceil((target - G(tau + 1)) / tau) in index order.
  bool keep_all = a.dense != 0;
  uint32_t tau = 0, keep_ties = 0, n_tau = 0;  // n_tau: masses equal to tau (0: not counted)
  if (!keep_all) {
    const uint32_t tgt = a.target_fx;
    uint4* work4 = reinterpret_cast<uint4*>(work);
#pragma unroll
    for (int k = lane; k < kSelWork / 4; k += 32) work4[k] = make_uint4(0u, 0u, 0u, 0u);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      const uint32_t mi = m.get(i);
      if (mi != 0u) atomicAdd(work + (31 - __clz(mi)) * 32 + lane, mi);
    }
    __syncwarp();
    uint32_t gs = 0;  // this lane's row; four words per load, the loads of a
                      // quarter-warp on distinct banks
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint4 q = work4[lane * 8 + ((lane + s) & 7)];
      gs += (q.x + q.y) + (q.z + q.w);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFull, gs, o);
      if (lane + o < 32) gs += t;
    }
    // lane b: G(2^b); lane 0: the total (masses are < 2^31, so lane 31: 0)
    const uint32_t total = __shfl_sync(kFull, gs, 0);
    __syncwarp();  // the table is read before the window overwrites it
    if (total < tgt) {  // total mass below the target (rounding): keep all
      keep_all = true;
    } else {
      const int e = 31 - __clz(__ballot_sync(kFull, gs >= tgt));
      const uint32_t above = __shfl_sync(kFull, gs, e + 1);
      uint32_t x = 1u << e;
      // compact the window [x, 2x); order does not matter for sums
      int wcnt = 0;
      uint32_t* dense = work + kDenseAt;
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        const uint32_t mi = m.get(i);
        const bool in = (mi - x) < x;  // unsigned: x <= m < 2x
        const unsigned bal = __ballot_sync(kFull, in);
        const int at = wcnt + __popc(bal & lanemask_lt());
        if (in && at < kCandCap) dense[at] = mi;
        wcnt += __popc(bal);
      }
      __syncwarp();
      if (wcnt <= kCandCap) {
        if (wcnt <= 32)
          window_search<1>(dense, wcnt, dense, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
        else if (wcnt <= 64)
          window_search<2>(dense, wcnt, dense, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
        else if (wcnt <= 128)
          window_search<4>(dense, wcnt, dense, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
        else
          window_search<8>(dense, wcnt, dense, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
      } else {
#pragma unroll 1
        for (int b = e - 1; b >= 0; --b) {
          const uint32_t t = x | (1u << b);
          if (mass_at_least<VPL>(m, t) >= tgt) x = t;
        }
        tau = x;
        keep_ties = (tgt - mass_at_least<VPL>(m, tau + 1) + tau - 1) / tau;
      }
    }
  }

  // ---- keep bitmap in shared memory: the NABLA bits by ballot (ties in
  // index order, unless every mass equal to tau is kept), then OR the STA
  // box, clipped to the grid. Padding slots hold mass 0 < tau.
  uint32_t* rbits = work + kRbitsAt;
  if (keep_all || n_tau == keep_ties) {
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (32 * i < nb) {  // warp-uniform
        const bool nab = keep_all ? lane + 32 * i < nb : m.get(i) >= tau;
        const unsigned kb = __ballot_sync(kFull, nab);
        if (lane == 0) rbits[i] = kb;
      }
    }
  } else {
    uint32_t ties = 0;
#pragma unroll
    for (int i = 0; i < VPL; ++i) {
      if (32 * i < nb) {  // warp-uniform
        const uint32_t mi = m.get(i);
        bool nab = mi > tau;
        const bool tie = mi == tau;
        const unsigned tb = __ballot_sync(kFull, tie);
        if (tie) nab = (ties + __popc(tb & lanemask_lt())) < keep_ties;
        ties += __popc(tb);
        const unsigned kb = __ballot_sync(kFull, nab);
        if (lane == 0) rbits[i] = kb;
      }
    }
  }
  __syncwarp();
  if (a.sta_t >= 0) {
    int tq, hq, wq;
    block_coords(g, qb, tq, hq, wq);
    const int t0 = max(tq - a.sta_t, 0), t1 = min(tq + a.sta_t, g.nt - 1);
    const int h0 = max(hq - a.sta_h, 0), h1 = min(hq + a.sta_h, g.nh - 1);
    const int w0 = max(wq - a.sta_w, 0), w1 = min(wq + a.sta_w, g.nw - 1);
    const int nw_ = w1 - w0 + 1, nhw = (h1 - h0 + 1) * nw_;
    const int cells = (t1 - t0 + 1) * nhw;
    for (int cidx = lane; cidx < cells; cidx += 32) {
      const int ct = cidx / nhw, r = cidx - ct * nhw, ch = r / nw_, cw = r - ch * nw_;
      const int j = ((t0 + ct) * g.nh + h0 + ch) * g.nw + w0 + cw;
      atomicOr(&rbits[j >> 5], 1u << (j & 31));
    }
    __syncwarp();
  }

  // ---- ascending kept list, bitmap and count to global: lane per word
  const int nwords = bitmap_words(g);
  uint32_t* bits = a.bits + size_t(row) * nwords;
  int32_t* out_idx = a.idx + size_t(row) * nb;
  int pos = 0;
  for (int base = 0; base < nwords; base += 32) {
    const int wi = base + lane;
    uint32_t w = wi < nwords ? rbits[wi] : 0u;
    if (wi < nwords) bits[wi] = w;
    const int cnt = __popc(w);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += t;
    }
    int o = pos + inc - cnt;
    while (w) {
      out_idx[o++] = 32 * wi + __ffs(w) - 1;
      w &= w - 1u;
    }
    pos += __shfl_sync(kFull, inc, 31);
  }
  if (lane == 0) a.cnt[row] = pos;
}

// ------------------------------------------------------------------ select, two warps per row
// Rows of 1025..2048 blocks: a pair of warps per row, 32 masses per lane each
// (warp h holds columns 1024 h + lane + 32 i), so that twice as many rows are
// in flight per SM as with one warp holding 64 masses per lane (registers
// bound the occupancy). The operations are those of select_kernel in the same
// order: the row sum continues warp 0's per-lane partial sums in warp 1, and
// integer sums are exact, so the kept sets are identical. The two warps meet
// at a named barrier of their own.
constexpr int kPairs = 4;      // rows per CTA
constexpr int kPairHV = 32;    // masses per lane and warp
constexpr int kPairRbitsAt = 2 * kCandCap;  // bitmap after the two window halves
static_assert(kPairRbitsAt + 64 <= kSelWork, "pair work area");

__global__ void __launch_bounds__(kPairs * 64, 4)
    select_pair_kernel(const float* __restrict__ L, MaskArgs a, Geometry g, int ld) {
  __shared__ __align__(16) uint32_t work_all[kPairs][kSelWork];
  __shared__ uint32_t xch_all[kPairs][64];  // per pair: values passed between the warps
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pr = warp >> 1, h = warp & 1;
  const long row = long(blockIdx.x) * kPairs + pr;
  if (row >= long(g.BH) * g.nb) return;  // both warps of the pair
  const uint32_t bar_id = 1u + uint32_t(pr);
  const int nb = g.nb;
  const int qb = int(row % nb);
  const float* Lr = L + size_t(row) * ld;
  uint32_t* work = work_all[pr];
  uint32_t* xch = xch_all[pr];  // [0..2]: maxima, sum; [8..39]: partial sums; [48..]: integers
  float* xf = reinterpret_cast<float*>(xch);
  const int j0 = h * 32 * kPairHV;
  constexpr float kLog2e = 1.4426950408889634f;

  // ---- row softmax to integer masses m = p * 2^30
  RowStore<kPairHV, false> m;
  {
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPairHV; ++i) {
      const int j = j0 + lane + 32 * i;
      const float v = j < nb ? __ldg(Lr + j) : -INFINITY;
      m.set(i, __float_as_uint(v));
      mx = fmaxf(mx, v);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    if (lane == 0) xf[h] = mx;
    named_barrier_sync(bar_id, 64);
    mx = fmaxf(xf[0], xf[1]);
    const float shift = -mx * kLog2e;
#pragma unroll
    for (int i = 0; i < kPairHV; ++i)  // exactly 0 in the padding slots
      m.set(i, __float_as_uint(ex2_approx(fmaf(__uint_as_float(m.get(i)), kLog2e, shift))));
    if (h == 0) {
      float sum = 0.f;
#pragma unroll
      for (int i = 0; i < kPairHV; ++i) sum += __uint_as_float(m.get(i));
      xf[8 + lane] = sum;
    }
    named_barrier_sync(bar_id, 64);
    if (h == 1) {
      float sum = xf[8 + lane];
#pragma unroll
      for (int i = 0; i < kPairHV; ++i) sum += __uint_as_float(m.get(i));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
      if (lane == 0) xf[2] = sum;
    }
    named_barrier_sync(bar_id, 64);
    const float to_fx = 1073741824.0f / xf[2];  // 2^30 / sum
#pragma unroll
    for (int i = 0; i < kPairHV; ++i) m.set(i, __float2uint_rn(__uint_as_float(m.get(i)) * to_fx));
  }

  // ---- CDF threshold, as in select_kernel: the leading-bit histogram (one
  // table for the pair), the window compacted by each warp into its own half,
  // searched by warp 0
  bool keep_all = a.dense != 0;
  uint32_t tau = 0, keep_ties = 0, n_tau = 0;
  if (!keep_all) {
    const uint32_t tgt = a.target_fx;
    uint4* work4 = reinterpret_cast<uint4*>(work);
#pragma unroll
    for (int k = h * 32 + lane; k < kSelWork / 4; k += 64) work4[k] = make_uint4(0u, 0u, 0u, 0u);
    named_barrier_sync(bar_id, 64);
#pragma unroll
    for (int i = 0; i < kPairHV; ++i) {
      const uint32_t mi = m.get(i);
      if (mi != 0u) atomicAdd(work + (31 - __clz(mi)) * 32 + lane, mi);
    }
    named_barrier_sync(bar_id, 64);
    uint32_t gs = 0;
#pragma unroll
    for (int s = 0; s < 8; ++s) {
      const uint4 q = work4[lane * 8 + ((lane + s) & 7)];
      gs += (q.x + q.y) + (q.z + q.w);
    }
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(kFull, gs, o);
      if (lane + o < 32) gs += t;
    }
    const uint32_t total = __shfl_sync(kFull, gs, 0);
    named_barrier_sync(bar_id, 64);  // both warps have read the table
    if (total < tgt) {
      keep_all = true;
    } else {
      const int e = 31 - __clz(__ballot_sync(kFull, gs >= tgt));
      const uint32_t above = __shfl_sync(kFull, gs, e + 1);
      uint32_t x = 1u << e;
      uint32_t* half = work + h * kCandCap;
      int wc = 0;
#pragma unroll
      for (int i = 0; i < kPairHV; ++i) {
        const uint32_t mi = m.get(i);
        const bool in = (mi - x) < x;  // unsigned: x <= m < 2x
        const unsigned bal = __ballot_sync(kFull, in);
        const int at = wc + __popc(bal & lanemask_lt());
        if (in && at < kCandCap) half[at] = mi;
        wc += __popc(bal);
      }
      if (lane == 0) xch[48 + h] = uint32_t(wc);
      named_barrier_sync(bar_id, 64);
      const int wc0 = int(xch[48]), wcnt = wc0 + int(xch[49]);
      if (wcnt <= kCandCap) {
        if (h == 0) {
          const uint32_t* d1 = work + kCandCap;
          if (wcnt <= 32)
            window_search<1>(work, wc0, d1, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
          else if (wcnt <= 64)
            window_search<2>(work, wc0, d1, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
          else if (wcnt <= 128)
            window_search<4>(work, wc0, d1, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
          else
            window_search<8>(work, wc0, d1, wcnt, lane, e, above, tgt, tau, keep_ties, n_tau);
          if (lane == 0) {
            xch[50] = tau;
            xch[51] = keep_ties;
            xch[52] = n_tau;
          }
        }
        named_barrier_sync(bar_id, 64);
        tau = xch[50];
        keep_ties = xch[51];
        n_tau = xch[52];
      } else {  // a long window: bit by bit over both warps' masses
#pragma unroll 1
        for (int b = e - 1; b >= 0; --b) {
          const uint32_t t = x | (1u << b);
          const uint32_t part = mass_at_least<kPairHV>(m, t);
          uint32_t* slot = xch + 56 + 2 * (b & 1);  // alternate slots: no overwrite before read
          if (lane == 0) slot[h] = part;
          named_barrier_sync(bar_id, 64);
          if (slot[0] + slot[1] >= tgt) x = t;
        }
        tau = x;
        const uint32_t part = mass_at_least<kPairHV>(m, tau + 1);
        if (lane == 0) xch[60 + h] = part;
        named_barrier_sync(bar_id, 64);
        keep_ties = (tgt - (xch[60] + xch[61]) + tau - 1) / tau;
      }
    }
  }

  // ---- keep bitmap: warp h writes words 32 h .. 32 h + 31; ties in index
  // order (warp 0's columns first) unless every mass equal to tau is kept
  uint32_t* rbits = work + kPairRbitsAt;
  if (keep_all || n_tau == keep_ties) {
#pragma unroll
    for (int i = 0; i < kPairHV; ++i) {
      if (j0 + 32 * i < nb) {  // warp-uniform
        const bool nab = keep_all ? j0 + lane + 32 * i < nb : m.get(i) >= tau;
        const unsigned kb = __ballot_sync(kFull, nab);
        if (lane == 0) rbits[h * kPairHV + i] = kb;
      }
    }
  } else {
    uint32_t ties = 0;
    if (h == 1) named_barrier_sync(bar_id, 64);  // warp 0's tie count first
    if (h == 1) ties = xch[62];
#pragma unroll
    for (int i = 0; i < kPairHV; ++i) {
      if (j0 + 32 * i < nb) {  // warp-uniform
        const uint32_t mi = m.get(i);
        bool nab = mi > tau;
        const bool tie = mi == tau;
        const unsigned tb = __ballot_sync(kFull, tie);
        if (tie) nab = (ties + __popc(tb & lanemask_lt())) < keep_ties;
        ties += __popc(tb);
        const unsigned kb = __ballot_sync(kFull, nab);
        if (lane == 0) rbits[h * kPairHV + i] = kb;
      }
    }
    if (h == 0) {
      if (lane == 0) xch[62] = ties;
      named_barrier_sync(bar_id, 64);
    }
  }
  named_barrier_sync(bar_id, 64);  // the bitmap is complete
  if (a.sta_t >= 0) {
    int tq, hq, wq;
    block_coords(g, qb, tq, hq, wq);
    const int t0 = max(tq - a.sta_t, 0), t1 = min(tq + a.sta_t, g.nt - 1);
    const int h0 = max(hq - a.sta_h, 0), h1 = min(hq + a.sta_h, g.nh - 1);
    const int w0 = max(wq - a.sta_w, 0), w1 = min(wq + a.sta_w, g.nw - 1);
    const int nw_ = w1 - w0 + 1, nhw = (h1 - h0 + 1) * nw_;
    const int cells = (t1 - t0 + 1) * nhw;
    for (int cidx = h * 32 + lane; cidx < cells; cidx += 64) {
      const int ct = cidx / nhw, r = cidx - ct * nhw, ch = r / nw_, cw = r - ch * nw_;
      const int j = ((t0 + ct) * g.nh + h0 + ch) * g.nw + w0 + cw;
      atomicOr(&rbits[j >> 5], 1u << (j & 31));
    }
    named_barrier_sync(bar_id, 64);
  }

  // ---- ascending kept list, bitmap and count: warp h takes words 32 h ..
  const int nwords = bitmap_words(g);
  uint32_t* bits = a.bits + size_t(row) * nwords;
  int32_t* out_idx = a.idx + size_t(row) * nb;
  int pos = 0;
  if (h == 1) pos = int(__reduce_add_sync(kFull, uint32_t(__popc(rbits[lane]))));
  {
    const int wi = 32 * h + lane;
    uint32_t w = wi < nwords ? rbits[wi] : 0u;
    if (wi < nwords) bits[wi] = w;
    const int cnt = __popc(w);
    int inc = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kFull, inc, o);
      if (lane >= o) inc += t;
    }
    int o = pos + inc - cnt;
    while (w) {
      out_idx[o++] = 32 * wi + __ffs(w) - 1;
      w &= w - 1u;
    }
    pos += __shfl_sync(kFull, inc, 31);
  }
  if (h == 1 && lane == 0) a.cnt[row] = pos;
}

// ------------------------------------------------------------------ union
constexpr int kUnionMaxWarps = 8;

// Shared words per warp: the two rows' bitmaps (+1 zero word each, read by
// the funnel shift below) and, frame-major ([T][fw] words, fw = words per
// frame), the first blocks of the temporal pairs and the unpaired blocks.
SA_HD int union_words_per_warp(const Geometry& g) {
  const int fw = (g.nh * g.nw + 31) / 32;
  return 2 * (bitmap_words(g) + 1) + 2 * g.nt * fw;
}

__global__ void __launch_bounds__(kUnionMaxWarps * 32) union_kernel(MaskArgs a, Geometry g) {
  extern __shared__ uint32_t ush[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwords = bitmap_words(g);
  const int pf = g.nh * g.nw, fw = (pf + 31) >> 5, nf = g.nt * fw;
  const long item = long(blockIdx.x) * (blockDim.x >> 5) + warp;  // (bh, tile)
  if (item >= long(g.BH) * g.ntile) return;
  const int bh = int(item / g.ntile), tile = int(item - long(bh) * g.ntile);
  int qa, qb;
  tile_blocks(g, tile, qa, qb);
  const uint32_t* ba = a.bits + (size_t(bh) * g.nb + qa) * nwords;
  const uint32_t* bb = qb >= 0 ? a.bits + (size_t(bh) * g.nb + qb) * nwords : nullptr;
  uint32_t* ua = ush + size_t(warp) * union_words_per_warp(g);
  uint32_t* ub = ua + nwords + 1;
  uint32_t* firstF = ub + nwords + 1;
  uint32_t* leftF = firstF + nf;
  for (int w = lane; w <= nwords; w += 32) {
    ua[w] = w < nwords ? ba[w] : 0u;
    ub[w] = (bb != nullptr && w < nwords) ? bb[w] : 0u;
  }
  __syncwarp();

  // Bits [t * pf + 32 w, +32) of the union, clipped to frame t.
  auto frame_word = [&](int t, int w) -> uint32_t {
    const int s = t * pf + 32 * w;
    const int q = s >> 5, off = s & 31;
    uint32_t x = ua[q] | ub[q];
    if (off) x = (x >> off) | ((ua[q + 1] | ub[q + 1]) << (32 - off));
    const int nbits = pf - 32 * w;
    return nbits < 32 ? x & ((1u << nbits) - 1u) : x;
  };
  // Greedy pairing along time: a block present in frame t whose frame t - 1
  // block is present and not already the second of a pair becomes the second
  // of a pair. Per bit, pair_t = a_t & ~pair_(t-1) with a_t = in_(t-1) & in_t:
  // each frame applies x -> (x & k) ^ v to the previous frame's pair bits
  // (k = v = a_t), and these maps compose associatively, so the pair bits of
  // 32 frames come from one scan over the lanes (lane = frame), 32 patches
  // per word at once. firstF[t] marks the first blocks of the pairs (t, t+1)
  // (= pair_(t+1)); leftF first holds in_t, then keeps the unpaired blocks.
  for (int w = 0; w < fw; ++w) {
    uint32_t carry_in = 0u, carry_pair = 0u;  // frame 32 c - 1: presence, pair bits
    for (int t0 = 0; t0 < g.nt; t0 += 32) {
      const int t = t0 + lane;
      const uint32_t in = t < g.nt ? frame_word(t, w) : 0u;
      uint32_t prev = __shfl_up_sync(kFull, in, 1);
      if (lane == 0) prev = carry_in;
      uint32_t k = prev & in, v = k;  // a_t
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t ke = __shfl_up_sync(kFull, k, o), ve = __shfl_up_sync(kFull, v, o);
        if (lane >= o) {  // this map after the earlier composite
          v = (ve & k) ^ v;
          k = ke & k;
        }
      }
      const uint32_t pair = (carry_pair & k) ^ v;
      if (t < g.nt) {
        if (t > 0) firstF[(t - 1) * fw + w] = pair;
        leftF[t * fw + w] = in;
      }
      carry_in = __shfl_sync(kFull, in, 31);
      carry_pair = __shfl_sync(kFull, pair, 31);
    }
    if (lane == 0) firstF[(g.nt - 1) * fw + w] = 0u;
  }
  __syncwarp();
  for (int i = lane; i < nf; i += 32)  // unpaired: in_t & ~pair_t & ~pair_(t+1)
    leftF[i] &= ~firstF[i] & (i >= fw ? ~firstF[i - fw] : ~0u);
  __syncwarp();

  // Emission in ascending block order (frame-major words are in block
  // order): first the pairs, two entries each, then the unpaired blocks.
  // Each lane takes one word of a 32-word group; a warp scan places it.
  int32_t* out = a.tidx + size_t(item) * g.nb;
  auto flags = [&](int b) {
    return int(((ua[b >> 5] >> (b & 31)) & 1u) << 16) | int(((ub[b >> 5] >> (b & 31)) & 1u) << 17);
  };
  int pos = 0;
  for (int pass = 0; pass < 2; ++pass) {
    const uint32_t* src = pass == 0 ? firstF : leftF;
    for (int base = 0; base < nf; base += 32) {
      const int it = base + lane;
      uint32_t x = it < nf ? src[it] : 0u;
      const int c = (pass == 0 ? 2 : 1) * __popc(x);
      int inc = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, inc, o);
        if (lane >= o) inc += v;
      }
      int o = pos + inc - c;
      const int t = it / fw;
      const int b0 = t * pf + 32 * (it - t * fw);
      while (x) {
        const int b = b0 + __ffs(x) - 1;
        x &= x - 1u;
        if (pass == 0) {
          out[o] = b | flags(b) | kEntryTPair;
          out[o + 1] = (b + pf) | flags(b + pf);
          o += 2;
        } else {
          out[o++] = b | flags(b);
        }
      }
      pos += __shfl_sync(kFull, inc, 31);
    }
  }
  if (lane == 0) a.tcnt[item] = pos;
}

template <int VPL>
cudaError_t launch_select(const MaskArgs& a, const Geometry& g, int ld, cudaStream_t stream) {
  const long rows = long(g.BH) * g.nb;
  constexpr bool kSmem = VPL > kRegVPL;
  const size_t smem = kSmem ? size_t(kSelWarps) * VPL * 32 * sizeof(uint32_t) : 0;
  if (kSmem) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel<VPL, kSmem>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  select_kernel<VPL, kSmem><<<unsigned((rows + kSelWarps - 1) / kSelWarps), kSelWarps * 32, smem,
                              stream>>>(a.logits, a, g, ld);
  return cudaGetLastError();
}

cudaError_t launch_select_pair(const MaskArgs& a, const Geometry& g, int ld, cudaStream_t stream) {
  const long rows = long(g.BH) * g.nb;
  select_pair_kernel<<<unsigned((rows + kPairs - 1) / kPairs), kPairs * 64, 0, stream>>>(
      a.logits, a, g, ld);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_logits(const MaskArgs& a, const Geometry& g, int ld, cudaStream_t stream) {
  const int smem = int(sizeof(LogitsSmem) + 1024);
  cudaError_t e = cudaFuncSetAttribute(logits_tc_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, nsm = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
    return e;
  const long ntiles = long(g.BH) * ((g.nb + kLtM - 1) / kLtM) * (ld / kLtN);
  const unsigned grid = unsigned(ntiles < nsm ? ntiles : nsm);  // one CTA per SM
  logits_tc_kernel<D><<<grid, kLtThreads, smem, stream>>>(a, g, ld);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mask(const MaskArgs& a, const Geometry& g, cudaStream_t stream,
                        cudaEvent_t* marks) {
  const int ld = logits_ld(g);
  cudaError_t e = g.d == 128 ? launch_logits<128>(a, g, ld, stream)
                             : launch_logits<64>(a, g, ld, stream);
  if (e != cudaSuccess) return e;
  if (marks != nullptr && (e = cudaEventRecord(marks[0], stream)) != cudaSuccess) return e;
  const int vpl = (g.nb + 31) / 32;  // nb <= 6144 (checked by the entry points)
  if (vpl <= 4) e = launch_select<4>(a, g, ld, stream);
  else if (vpl <= 8) e = launch_select<8>(a, g, ld, stream);
  else if (vpl <= 16) e = launch_select<16>(a, g, ld, stream);
  else if (vpl <= 32) e = launch_select<32>(a, g, ld, stream);
  else if (vpl <= 64) e = launch_select_pair(a, g, ld, stream);
  else if (vpl <= 96) e = launch_select<96>(a, g, ld, stream);
  else e = launch_select<192>(a, g, ld, stream);
  if (e != cudaSuccess) return e;
  if (marks != nullptr && (e = cudaEventRecord(marks[1], stream)) != cudaSuccess) return e;
  return launch_union(a, g, stream);
}

cudaError_t launch_union(const MaskArgs& a, const Geometry& g, cudaStream_t stream) {
  const long items = long(g.BH) * g.ntile;
  const size_t warp_bytes = size_t(union_words_per_warp(g)) * sizeof(uint32_t);
  int wpc = int((48 * 1024) / warp_bytes);  // warps per CTA within 48 KB
  wpc = wpc < 1 ? 1 : (wpc > kUnionMaxWarps ? kUnionMaxWarps : wpc);
  union_kernel<<<unsigned((items + wpc - 1) / wpc), unsigned(wpc * 32), wpc * warp_bytes,
                 stream>>>(a, g);
  return cudaGetLastError();
}

// One CTA per head: bitonic sort of the head's tiles by descending union
// length, so that the attention grid meets the heaviest tiles of a head first
// (longest-processing-time order) while concurrently running CTAs still share
// one head's K/V in L2.
__global__ void __launch_bounds__(1024) tile_order_kernel(const int32_t* __restrict__ tcnt,
                                                          int32_t* __restrict__ order, Geometry g) {
  __shared__ uint32_t key[4096];
  const int bh = blockIdx.x;
  int n = 1;
  while (n < g.ntile) n <<= 1;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    // ascending key = descending count, then ascending tile; padding sorts last
    key[i] = i < g.ntile ? (uint32_t(g.nb - tcnt[size_t(bh) * g.ntile + i]) << 16) | uint32_t(i)
                         : 0xFFFFFFFFu;
  }
  __syncthreads();
  for (int size = 2; size <= n; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int partner = i ^ stride;
        if (partner > i) {
          const bool up = (i & size) == 0;
          const uint32_t x = key[i], y = key[partner];
          if ((x > y) == up) {
            key[i] = y;
            key[partner] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int i = threadIdx.x; i < g.ntile; i += blockDim.x)
    order[size_t(bh) * g.ntile + i] = int32_t(key[i] & 0xFFFFu);
}

cudaError_t launch_tile_order(const int32_t* tcnt, int32_t* order, const Geometry& g,
                              cudaStream_t stream) {
  tile_order_kernel<<<unsigned(g.BH), 1024, 0, stream>>>(tcnt, order, g);
  return cudaGetLastError();
}

}  // namespace sa
