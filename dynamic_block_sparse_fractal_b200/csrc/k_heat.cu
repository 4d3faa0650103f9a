// Exact block max-pooled attention map (the reference target of the page
// "Veda: Video Generation with Efficient Sparse Attention", section 2.1,
// "Costruzione dell'Obiettivo"): for every (q-block, k-block) pair of a head,
// the largest probability of the full, unmasked softmax attention inside the
// N x N block. A quality signal for a block mask: how much of the real
// attention its kept blocks carry.
//
// One CTA per pair of consecutive q-blocks (a 128-row query tile), two dense
// passes over all k-block pairs with S = Q K^T on the tensor cores:
//   pass 1  the row's log-sum-exp: online max and sum of 2^x,
//           x = s * log2(e) / sqrt(d), lse2 = m + log2(l);
//   pass 2  per 64-key half (one k-block) the row max of x - lse2, reduced
//           over the 64 rows of each q-block; H = 2^max.
// warp 0: TMA (Q tile, then K pairs into a 3-slot ring, both passes);
// warp 1: TMEM owner and MMA issuer (S double-buffered in TMEM);
// warps 2-5: one thread per tile row (TMEM lane). All waits are bounded.
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

namespace {

constexpr int kHThreads = 192;
constexpr int kHSlots = 3;
constexpr int kHChunk = 128 * 128;  // 128 rows x 128 B (64 bf16 channels)

template <int D>
struct __align__(1024) HeatSmem {
  uint8_t q[D / 64][kHChunk];
  uint8_t slot[kHSlots][D / 64][kHChunk];
  uint64_t q_full, full[kHSlots], empty[kHSlots], s_full[2], s_free[2], drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail_h(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kHThreads, 1)
    heat_kernel(const __grid_constant__ HeatArgs a, const Geometry g) {
  extern __shared__ uint8_t h_raw[];
  HeatSmem<D>& sm = *reinterpret_cast<HeatSmem<D>*>(
      (reinterpret_cast<uintptr_t>(h_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qa = 2 * blockIdx.x, qb = qa + 1 < g.nb ? qa + 1 : -1;
  const int nsteps = (g.nb + 1) / 2;  // k-block pairs per pass
  const int nops = 2 * nsteps;
  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kHSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.s_full[b], 1);
      mbar_init(&sm.s_free[b], 128);
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort = &sm.abort;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&a.map_q);
      prefetch_tensormap(&a.map_k);
      mbar_arrive_expect_tx(&sm.q_full, 128u * D * 2u);
      for (int e = 0; e < 2; ++e) {
        const int blk = (e == 0 || qb < 0) ? qa : qb;
        int t, hp, wp;
        block_coords(g, blk, t, hp, wp);
        for (int c = 0; c < D / 64; ++c)
          tma_load_5d(&sm.q[c][e * 8192], &a.map_q, &sm.q_full, c * 64, wp * g.pw, hp * g.ph,
                      t * g.pt, bh);
      }
      int issued = -1;
      for (int m = 0; m < nops; ++m) {
        const int s = m % kHSlots, use = m / kHSlots;
        if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort)) {
          fail_h(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        if (*abort) break;
        const int j = m % nsteps;
        const int nblk = 2 * j + 1 < g.nb ? 2 : 1;
        mbar_arrive_expect_tx(&sm.full[s], uint32_t(nblk) * 64u * D * 2u);
        for (int e = 0; e < nblk; ++e) {
          int t, hp, wp;
          block_coords(g, 2 * j + e, t, hp, wp);
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.slot[s][c][e * 8192], &a.map_k, &sm.full[s], c * 64, wp * g.pw,
                        hp * g.ph, t * g.pt, bh);
        }
        issued = m;
      }
      if (*abort && issued >= 0) {  // let this thread's copies land before the CTA exits
        int never = 0;
        for (int m = issued; m >= 0 && m > issued - kHSlots; --m)
          mbar_wait(&sm.full[m % kHSlots], (m / kHSlots) & 1, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id2 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint64_t qd = sw128_desc(smem_u32(&sm.q[0][0]), 16, 1024);
      const uint64_t kd0 = sw128_desc(smem_u32(&sm.slot[0][0][0]), 16, 1024);
      constexpr uint32_t kSlotStep = (D / 64) * kHChunk / 16;
      bool ok = mbar_wait(&sm.q_full, 0, abort);
      for (int m = 0; ok && m < nops; ++m) {
        const int s = m % kHSlots, buf = m & 1;
        const int j = m % nsteps;
        ok = mbar_wait(&sm.full[s], (m / kHSlots) & 1, abort) &&
             (m < 2 || mbar_wait(&sm.s_free[buf], ((m >> 1) - 1) & 1, abort));
        if (!ok) break;
        tc_fence_after_sync();
        const uint64_t kd = kd0 + uint64_t(s) * kSlotStep;
        const uint32_t id = 2 * j + 1 < g.nb ? id2 : id1;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t(kk >> 2) * kHChunk + uint32_t(kk & 3) * 32u) >> 4;
          mma_ss(tmem + uint32_t(buf) * 128u, qd + off, kd + off, id, kk > 0);
        }
        mma_commit(&sm.empty[s]);
        mma_commit(&sm.s_full[buf]);
      }
      if (!ok) {
        fail_h(a.status, &sm.abort, kDevErrTimeoutMma);
        mma_commit(&sm.drain);  // wait (bounded) for this thread's MMAs before exit
        int never = 0;
        mbar_wait(&sm.drain, 0, &never);
      }
    }
  } else {
    // processing: thread = tile row r (TMEM lane); rows 0-63 = qa, 64-127 = qb
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int half = r >> 6;
    const bool row_valid = half == 0 || qb >= 0;
    const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f, lse2 = 0.f;
    bool ok = true;
    for (int op = 0; op < nops; ++op) {
      const int buf = op & 1, j = op % nsteps;
      const int nblk = 2 * j + 1 < g.nb ? 2 : 1;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[buf], (op >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      uint32_t sv[128];
      tmem_ld32(t_lane + buf * 128u + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      tmem_ld32(t_lane + buf * 128u + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      if (nblk == 2) {
        tmem_ld32(t_lane + buf * 128u + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
        tmem_ld32(t_lane + buf * 128u + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      }
      tmem_wait_ld();
      tc_fence_before_sync();
      mbar_arrive(&sm.s_free[buf]);
      if (op < nsteps) {
        // pass 1: online log-sum-exp of x = s * log2(e) / sqrt(d)
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < 64 * nblk) mx = fmaxf(mx, __uint_as_float(sv[i]) * sl2);
        const float m_new = fmaxf(m, mx);
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < 64 * nblk) sum += ex2_approx(__uint_as_float(sv[i]) * sl2 - m_new);
        l = l * ex2_approx(m - m_new) + sum;  // m = -inf at first: 2^-inf = 0
        m = m_new;
        if (op == nsteps - 1) lse2 = m + __log2f(l);
      } else {
        // pass 2: per k-block, the max over this row of x - lse2, then over
        // the warp's 32 rows; the two warps of a q-block meet in an atomic max
        // on the (non-negative) probability's bits, on a zeroed map
        float bm[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i < 64 * nblk) bm[i >> 6] = fmaxf(bm[i >> 6], __uint_as_float(sv[i]) * sl2);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float v = bm[e] - lse2;
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
          bm[e] = v;
        }
        if (lane < nblk && row_valid) {
          const int qblk = half ? qb : qa;
          const float p = ex2_approx(lane == 0 ? bm[0] : bm[1]);
          atomicMax(reinterpret_cast<int*>(a.heat) + (size_t(bh) * g.nb + qblk) * g.nb + 2 * j +
                        lane,
                    __float_as_int(p));
        }
      }
    }
    if (!ok) fail_h(a.status, &sm.abort, kDevErrTimeoutSoftmax);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 256);
}

template <int D>
static cudaError_t launch_heat_d(const HeatArgs& a, const Geometry& g, cudaStream_t stream) {
  const int smem = int(sizeof(HeatSmem<D>) + 1024);
  cudaError_t e = cudaMemsetAsync(a.heat, 0, size_t(g.BH) * g.nb * g.nb * sizeof(float), stream);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(heat_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned((g.nb + 1) / 2), unsigned(g.BH));
  heat_kernel<D><<<grid, kHThreads, smem, stream>>>(a, g);
  return cudaGetLastError();
}

cudaError_t launch_heat(const HeatArgs& a, const Geometry& g, cudaStream_t stream) {
  return g.d == 128 ? launch_heat_d<128>(a, g, stream) : launch_heat_d<64>(a, g, stream);
}

}  // namespace sa
