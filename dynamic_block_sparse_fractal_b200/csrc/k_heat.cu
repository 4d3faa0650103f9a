// Exact block max-pooled attention map (the reference target of the page
// "Veda - Diffusione Video Scalabile tramite Attenzione Sparsa Distillata",
// gist.science/it/paper/2605.30325, section 2.1, "Costruzione
// dell'Obiettivo"): for every (q-block, k-block) pair of a head,
// the largest probability of the full, unmasked softmax attention inside the
// N x N block. A quality signal for a block mask: how much of the real
// attention its kept blocks carry.
//
// One dense pass over every key with S = Q K^T on the tensor cores. For a
// query row r and a k-block b, H depends on the row only through
//   max_{k in b} s[r][k]  and  lse2[r] = log2 sum_k 2^(x[r][k]),
// x = s * log2(e) / sqrt(d):  H[qb][b] = max_{r in qb} 2^(xmax[r][b] - lse2[r]).
// So each row keeps its online log-sum-exp (max m, sum l) and writes its raw
// block maxima to a per-CTA fp32 scratch laid out [b][row]; once the row's
// lse2 is final, its thread reads back its own entries, and the rows of a
// q-block are reduced by a butterfly across the warp and an atomic max
// (probabilities are non-negative, so their bits order like integers) on a
// zeroed map.
//
// Persistent grid of at most kHeatCtas CTAs; a CTA's unit of work is four
// consecutive q-blocks of one head as two 128-row query tiles A and B that
// share every K pair. warp 0: TMA (Q tiles, K pairs into a 3-slot ring);
// warp 1: TMEM owner (512 columns: S of A and B, double-buffered) and MMA
// issuer; warps 2-9 / 10-17: tile A / B, two threads per row, one per k-block
// of each K pair (their running sums meet once per unit). All waits are
// bounded.
#include <cuda_runtime.h>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

namespace {

constexpr int kHThreads = 576;  // 2 control warps + 16 row warps
constexpr int kHSlots = 3;
constexpr int kHChunk = 128 * 128;   // 128 rows x 128 B (64 bf16 channels)
constexpr int kHRows = 256;          // scratch rows per CTA (two tiles)
// Of every 8 column pairs of a row, this many take the FMA-pipe exp2 (degree
// 5, fp32-level accuracy); the rest the special-function unit, which alone
// would bound the pass.
constexpr int kHeatPolyPairsPer8 = 2;

template <int D>
struct __align__(1024) HeatSmem {
  uint8_t q[2][D / 64][kHChunk];           // tiles A, B
  uint8_t slot[kHSlots][D / 64][kHChunk];  // one K pair (128 keys) per slot
  uint64_t q_full, q_empty, full[kHSlots], empty[kHSlots];
  uint64_t s_full[2][2], s_free[2][2];  // [tile][TMEM buffer]
  uint64_t lse_bar[2];                  // [tile]: both halves' (max, sum) written
  uint64_t drain;
  float2 ml[2][2][2][128];              // [unit parity][tile][half][row]: (max, sum)
  float xs[2][2][2][128];               // the same: sum of 2^(x - max) (x - max)
  uint32_t tmem_base;
  int abort;
};

// Sum over the 64 columns of 2^(s * sl2 - m), two columns per packed op;
// kHeatPolyPairsPer8 of every 8 pairs take the FMA-pipe exp2. With ENT, also
// the sum of 2^(x - m) * (x - m) (x = s * sl2), for the row's entropy.
template <bool ENT>
__device__ __forceinline__ float exp2_row_sum(const uint32_t (&sv)[64], uint64_t sl2x2, float m,
                                              float& xsum) {
  const uint64_t negm2 = f2_pack(-m, -m);
  uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
  uint64_t xs2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const uint64_t x2 = f2_fma(
        f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2x2, negm2);
    float x0, x1;
    f2_unpack(x2, x0, x1);
    uint64_t e2;
    if ((i & 7) >= 8 - kHeatPolyPairsPer8)
      e2 = exp2_poly5_x2(f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f)));
    else
      e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
    rs2[i & 3] = f2_add(rs2[i & 3], e2);
    if (ENT) xs2[i & 3] = f2_fma(e2, x2, xs2[i & 3]);
  }
  float lo, hi;
  if (ENT) {
    f2_unpack(f2_add(f2_add(xs2[0], xs2[1]), f2_add(xs2[2], xs2[3])), lo, hi);
    xsum = lo + hi;
  }
  f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), lo, hi);
  return lo + hi;
}

__device__ __forceinline__ void fail_h(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

// Unit u of the persistent loop: head bh, first q-block base (tile x, half h
// holds q-block base + 2x + h, absent when >= nb).
__device__ __forceinline__ void heat_unit(const Geometry& g, long u, int& bh, int& base) {
  const int per_head = (g.nb + 3) / 4;
  bh = int(u / per_head);
  base = 4 * int(u - long(bh) * per_head);
}

}  // namespace

// MAP: write the block max-pooled map (scratch + reduction); ENT: write each
// query row's entropy. At least one of the two.
template <int D, bool MAP, bool ENT>
__global__ void __launch_bounds__(kHThreads, 1)
    heat_kernel(const __grid_constant__ HeatArgs a, const Geometry g) {
  extern __shared__ uint8_t h_raw[];
  HeatSmem<D>& sm = *reinterpret_cast<HeatSmem<D>*>(
      (reinterpret_cast<uintptr_t>(h_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long units = long(g.BH) * ((g.nb + 3) / 4);
  const int nsteps = (g.nb + 1) / 2;  // K pairs per unit
  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kHSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int x = 0; x < 2; ++x)
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[x][b], 1);
        mbar_init(&sm.s_free[x][b], 256);
      }
    for (int x = 0; x < 2; ++x) mbar_init(&sm.lse_bar[x], 256);
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
    // ---------------------------------------------------------------- TMA
    if (lane == 0) {
      prefetch_tensormap(&a.map_q);
      prefetch_tensormap(&a.map_k);
      int it = 0, op = 0, last_op = -1, last_q = -1;
      for (long u = blockIdx.x; u < units && !*abort; u += gridDim.x, ++it) {
        int bh, base;
        heat_unit(g, u, bh, base);
        if (it > 0 && !mbar_wait(&sm.q_empty, (it - 1) & 1, abort)) {
          fail_h(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        mbar_arrive_expect_tx(&sm.q_full, 2u * 128u * D * 2u);
        for (int x = 0; x < 2; ++x)
          for (int e = 0; e < 2; ++e) {
            const int blk = min(base + 2 * x + e, g.nb - 1);  // absent: any valid block
            int t, hp, wp;
            block_coords(g, blk, t, hp, wp);
            for (int c = 0; c < D / 64; ++c)
              tma_load_5d(&sm.q[x][c][e * 8192], &a.map_q, &sm.q_full, c * 64, wp * g.pw,
                          hp * g.ph, t * g.pt, bh);
          }
        last_q = it;
        bool ok = true;
        for (int j = 0; j < nsteps; ++j, ++op) {
          const int s = op % kHSlots, use = op / kHSlots;
          if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort)) {
            fail_h(a.status, &sm.abort, kDevErrTimeoutLoad);
            ok = false;
            break;
          }
          if (*abort) {
            ok = false;
            break;
          }
          if (op == 0 && (a.debug_flags & SA_DEBUG_STALL_LOADER)) continue;  // test hook
          const int nblk = 2 * j + 1 < g.nb ? 2 : 1;
          mbar_arrive_expect_tx(&sm.full[s], uint32_t(nblk) * 64u * D * 2u);
          for (int e = 0; e < nblk; ++e) {
            int t, hp, wp;
            block_coords(g, 2 * j + e, t, hp, wp);
            for (int c = 0; c < D / 64; ++c)
              tma_load_5d(&sm.slot[s][c][e * 8192], &a.map_k, &sm.full[s], c * 64, wp * g.pw,
                          hp * g.ph, t * g.pt, bh);
          }
          last_op = op;
        }
        if (!ok) break;
      }
      if (*abort) {
        // let this thread's copies land before the CTA can exit (time-bounded,
        // ignoring the abort flag); at most one op per slot can be in flight
        int never = 0;
        for (int o = last_op; o >= 0 && o > last_op - kHSlots; --o)
          mbar_wait(&sm.full[o % kHSlots], (o / kHSlots) & 1, &never);
        if (last_q >= 0) mbar_wait(&sm.q_full, last_q & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0) {
      const uint32_t id2 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint64_t qd0 = sw128_desc(smem_u32(&sm.q[0][0][0]), 16, 1024);
      const uint64_t kd0 = sw128_desc(smem_u32(&sm.slot[0][0][0]), 16, 1024);
      constexpr uint32_t kTileStep = (D / 64) * kHChunk / 16;  // descriptor units
      bool ok = true;
      int it = 0, op = 0;
      for (long u = blockIdx.x; ok && u < units; u += gridDim.x, ++it) {
        ok = mbar_wait(&sm.q_full, it & 1, abort);
        for (int j = 0; ok && j < nsteps; ++j, ++op) {
          const int s = op % kHSlots, buf = op & 1;
          ok = mbar_wait(&sm.full[s], (op / kHSlots) & 1, abort);
          const uint32_t id = 2 * j + 1 < g.nb ? id2 : id1;
          const uint64_t kd = kd0 + uint64_t(s) * kTileStep;
          for (int x = 0; ok && x < 2; ++x) {
            ok = op < 2 || mbar_wait(&sm.s_free[x][buf], ((op >> 1) - 1) & 1, abort);
            if (!ok) break;
            tc_fence_after_sync();
            const uint64_t qd = qd0 + uint64_t(x) * kTileStep;
            const uint32_t d_tmem = tmem + uint32_t(x) * 256u + uint32_t(buf) * 128u;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t off = (uint32_t(kk >> 2) * kHChunk + uint32_t(kk & 3) * 32u) >> 4;
              mma_ss(d_tmem, qd + off, kd + off, id, kk > 0);
            }
            mma_commit(&sm.s_full[x][buf]);
          }
          if (ok) mma_commit(&sm.empty[s]);
        }
        if (ok) mma_commit(&sm.q_empty);
      }
      if (!ok) {
        fail_h(a.status, &sm.abort, kDevErrTimeoutMma);
        mma_commit(&sm.drain);  // wait (bounded) for this thread's MMAs before exit
        int never = 0;
        mbar_wait(&sm.drain, 0, &never);
      }
    }
  } else {
    // ---------------------------------------------------------------- rows
    // thread = row r of tile x (TMEM lane r), columns of k-block 2j + e of
    // each step (e = which half of the K pair); rows 0-63 / 64-127 of a tile
    // are its two q-blocks
    const int pw = warp - 2;
    const int x = pw >> 3, e = (pw >> 2) & 1, quad = warp & 3;
    const int r = quad * 32 + lane;
    const int half = r >> 6;
    const uint32_t t_lane =
        tmem + (uint32_t(quad * 32) << 16) + uint32_t(x) * 256u + uint32_t(e) * 64u;
    // this thread's scratch column: entry b at mine[b * kHRows]
    float* mine = MAP ? a.scratch + size_t(blockIdx.x) * kHRows * g.nb + x * 128 + r : nullptr;
    const float sl2 = a.scale_log2;
    const uint64_t sl2x2 = f2_pack(sl2, sl2);
    bool ok = true;
    int op = 0, it = 0;
    for (long u = blockIdx.x; ok && u < units; u += gridDim.x, ++it) {
      int bh, base;
      heat_unit(g, u, bh, base);
      // log2-domain running max and sum over this half; xs = sum of
      // 2^(x - m) (x - m) for the entropy (relative to m, so that no large
      // values cancel)
      float m = -INFINITY, l = 0.f, xs = 0.f;
      for (int j = 0; j < nsteps; ++j, ++op) {
        const int buf = op & 1;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[x][buf], (op >> 1) & 1, abort));
        if (!ok) break;
        tc_fence_after_sync();
        if (2 * j + e >= g.nb) {  // the lone last k-block: nothing in this half
          mbar_arrive(&sm.s_free[x][buf]);
          continue;
        }
        uint32_t sv[64];
        tmem_ld32(t_lane + uint32_t(buf) * 128u, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(t_lane + uint32_t(buf) * 128u + 32u,
                  *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_ld();
        tc_fence_before_sync();
        mbar_arrive(&sm.s_free[x][buf]);
        // raw maximum of the row over k-block 2j + e (four chains)
        float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int i = 0; i < 64; i += 2)
          mq[(i >> 1) & 3] =
              max3(mq[(i >> 1) & 3], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
        const float bmax = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        if (MAP) mine[size_t(2 * j + e) * kHRows] = bmax;
        const float m_new = fmaxf(m, bmax * sl2);
        const float alpha = ex2_approx(m - m_new);  // m = -inf at first: 2^-inf = 0
        if (ENT) xs = l > 0.f ? alpha * fmaf(l, m - m_new, xs) : 0.f;
        l *= alpha;
        m = m_new;
        float xsj = 0.f;
        l += exp2_row_sum<ENT>(sv, sl2x2, m, xsj);
        if (ENT) xs += xsj;
      }
      if (!ok) break;
      // ---- the row's two halves meet: lse2 over all keys (both threads of
      // the row compute the same value)
      sm.ml[it & 1][x][e][r] = make_float2(m, l);
      if (ENT) sm.xs[it & 1][x][e][r] = xs;
      mbar_arrive(&sm.lse_bar[x]);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.lse_bar[x], it & 1, abort));
      if (!ok) break;
      const float2 o = sm.ml[it & 1][x][e ^ 1][r];
      const float mm = fmaxf(m, o.x);
      const float ll = (e == 0 ? l * ex2_approx(m - mm) + o.y * ex2_approx(o.x - mm)
                               : o.y * ex2_approx(o.x - mm) + l * ex2_approx(m - mm));
      const float lse2 = mm + __log2f(ll);
      const int qblk = base + 2 * x + half;  // uniform across the warp
      if (qblk >= g.nb) continue;
      if (ENT && e == 0) {
        // H = -sum p ln p with p = 2^(x - lse2): ln 2 (log2 L - XS / L), L and
        // XS the row's sums relative to mm (the halves rescaled, XS shifted)
        const float ox = sm.xs[it & 1][x][1][r];
        const float a0 = ex2_approx(m - mm), a1 = ex2_approx(o.x - mm);
        const float X0 = l > 0.f ? a0 * fmaf(l, m - mm, xs) : 0.f;
        const float X1 = o.y > 0.f ? a1 * fmaf(o.y, o.x - mm, ox) : 0.f;
        const float H = 0.6931471805599453f * (__log2f(ll) - (X0 + X1) / ll);
        a.entropy[size_t(bh) * g.S + block_row_token(g, qblk, r & 63)] = H;
      }
      if (!MAP) continue;
      // ---- this unit's map rows, blocks 2i + e
      int* out = reinterpret_cast<int*>(a.heat) + (size_t(bh) * g.nb + qblk) * g.nb + e;
      const int nbe = (g.nb - e + 1) / 2;  // blocks of this parity
      for (int b0 = 0; b0 < nbe; b0 += 32) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i)
          v[i] = b0 + i < nbe ? fmaf(mine[size_t(2 * (b0 + i) + e) * kHRows], sl2, -lse2)
                              : -INFINITY;
        // butterfly reduce-scatter over the warp's 32 rows: after the stage
        // of width w, lane l holds in v[0..w) the maxima for the blocks whose
        // index bits above w agree with l's; at the end v[0] = block b0 + lane
#pragma unroll
        for (int w = 16; w >= 1; w >>= 1) {
          const bool upper = (lane & w) != 0;
#pragma unroll
          for (int i = 0; i < w; ++i) {
            const float keep = upper ? v[i + w] : v[i];
            const float send = upper ? v[i] : v[i + w];
            v[i] = fmaxf(keep, __shfl_xor_sync(0xFFFFFFFFu, send, w));
          }
        }
        if (b0 + lane < nbe) atomicMax(out + 2 * (b0 + lane), __float_as_int(ex2_approx(v[0])));
      }
    }
    if (!ok) fail_h(a.status, &sm.abort, kDevErrTimeoutSoftmax);
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D, bool MAP, bool ENT>
static cudaError_t launch_heat_k(const HeatArgs& a, const Geometry& g, cudaStream_t stream) {
  // at least half the shared memory of an SM, so that one CTA (with its 512
  // TMEM columns) is resident per SM whatever the register count
  const int smem = max(int(sizeof(HeatSmem<D>) + 1024), 116 * 1024);
  cudaError_t e;
  if (MAP) {
    e = cudaMemsetAsync(a.heat, 0, size_t(g.BH) * g.nb * g.nb * sizeof(float), stream);
    if (e != cudaSuccess) return e;
  }
  e = cudaFuncSetAttribute(heat_kernel<D, MAP, ENT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem);
  if (e != cudaSuccess) return e;
  heat_kernel<D, MAP, ENT><<<unsigned(heat_ctas(g)), kHThreads, smem, stream>>>(a, g);
  return cudaGetLastError();
}

template <int D>
static cudaError_t launch_heat_d(const HeatArgs& a, const Geometry& g, cudaStream_t stream) {
  if (a.heat != nullptr && a.entropy != nullptr) return launch_heat_k<D, true, true>(a, g, stream);
  if (a.heat != nullptr) return launch_heat_k<D, true, false>(a, g, stream);
  if (a.entropy != nullptr) return launch_heat_k<D, false, true>(a, g, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_heat(const HeatArgs& a, const Geometry& g, cudaStream_t stream) {
  return g.d == 128 ? launch_heat_d<128>(a, g, stream) : launch_heat_d<64>(a, g, stream);
}

}  // namespace sa
