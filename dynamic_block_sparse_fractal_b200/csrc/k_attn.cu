// Block-sparse attention forward over the kept (q-block, k-block) pairs
// ("Espansione", NABLA Metodologia 2: every dropped N x N block is -inf), on
// the sm_100a tensor cores.
//
// A query tile is 128 rows = two q-blocks (64 rows each) of one head; it runs
// over the union of the two blocks' kept k-block lists, two k-blocks (128
// keys) per step. Rows of a q-block that does not keep a k-block see it as
// -inf and evaluate no exponentials for it.
//
// A CTA holds two tiles, A and B (consecutive entries of the head's
// heaviest-first tile order), so that the tensor core works on one tile while
// the softmax warps of the other run:
//
//   producers   the two Q tiles, then one 32 KB ring slot per MMA (a K pair
//               for S, a V pair for PV) in exactly the order the MMA warp
//               consumes them. Q/K/V are read in natural layout
//               through 5-D tensor maps whose box is one 8x8 patch of one
//               frame, so the fractal flattening is pure addressing.
//   warp 1      owns TMEM (S_A, S_B, O_A, O_B: 4 x 128 columns) and issues
//               tcgen05.mma in the order
//                 S_A0 S_B0 | PV_A0 S_A1 PV_B0 S_B1 | PV_A1 S_A2 PV_B1 S_B2 | ...
//               S_X = Q_X K^T (SS, M=128, N=64*nblk, K=d) -> TMEM S_X;
//               O_X += P_X V (TS: P from TMEM over S_X, V MN-major in smem).
//   warps 4-7   softmax of tile A, warps 8-11 softmax of tile B: one thread
//               per query row (TMEM lane), online softmax in fp32 in the exp2
//               domain, P written back as bf16 over S in TMEM, O rescaled in
//               TMEM only when the running max grows by more than 2^8 (exact
//               after the final 1/l), epilogue O / l -> natural token position.
//   warps 0,2,3 TMA producers (every third op each): one issuing thread
//               keeps too few boxes in flight to feed the tensor core.
//
// Ordering facts the pipeline relies on: tcgen05.mma ops issued by one thread
// execute in order, and a tcgen05.commit tracks every op issued before it. So
// when the softmax of tile X sees S_X(j) complete, PV_X(j-1) (issued before
// S_X(j)) is complete too, and O_X may be rescaled without another wait.
//
// All waits are bounded (sm100.cuh); a wait that runs out records a status
// bit, raises a CTA-wide abort flag, drains its own in-flight work and lets
// the CTA free TMEM and exit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "exp2_poly.cuh"
#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

// Timeline trace (a diagnostics build with -DSA_TRACE=1 only): clock64
// stamps of one CTA's MMA issuer (per unit: wait start, operands ready,
// issued) and of its eight softmax warps (per step: S seen, P arrived).
#ifndef SA_TRACE
#define SA_TRACE 0
#endif
#if SA_TRACE
constexpr int kTraceUnits = 1300, kTraceSteps = 500;
constexpr int kTraceSoftmax = 4096, kTraceWords = kTraceSoftmax + 8 * 2 * kTraceSteps;
__device__ long long g_attn_trace[kTraceWords];
__device__ int g_attn_trace_cta[2] = {100, 3};
#endif

namespace {

constexpr int kThreads = 384;
constexpr int kSlots = 4;
constexpr int kProducers = 3;  // TMA-issuing warps (0, 2, 3)
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 128 B (64 bf16 channels)
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;  // log2 units
// Column pairs (of every 8) whose exp2 runs on the FMA pipe instead of the
// SFU. Measured on the HunyuanVideo-like workload: 1 of 8 made the attention
// 7% slower and 2 of 8 17% slower (the softmax warps are limited by issue and
// latency, not by the SFU's rate), so all go to the SFU.
constexpr int kPolyPairsPer8 = 0;
// Union entries staged in shared memory per tile; longer unions (heads of
// more than 2880 blocks) read the rest from global memory (L2).
constexpr int kMaxList = 2880;

__host__ __device__ constexpr uint32_t col_s(int x) { return uint32_t(x) * 128u; }
__host__ __device__ constexpr uint32_t col_o(int x) { return 256u + uint32_t(x) * 128u; }

template <int D>
struct __align__(1024) AttnSmem {
  uint8_t q[2][D / 64][kChunkBytes];
  uint8_t slot[kSlots][D / 64][kChunkBytes];
  int32_t list[2][kMaxList];  // the two tiles' union lists, staged once
  uint64_t q_full[2];
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t p_full[2];
  uint64_t o_final[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct Tile {
  int qa, qb;           // q-blocks (qb = -1: lone block)
  int n_u;              // union length
  int nsteps;           // ceil(n_u / 2)
  const int32_t* list;   // union entries (shared-memory copy of the first kMaxList)
  const int32_t* glist;  // the same entries in global memory
};

__device__ __forceinline__ int list_at(const Tile& t, int i) {
  return i < kMaxList ? t.list[i] : __ldg(t.glist + i);
}

// The MMA issue order shared by the loader and the MMA warp.
struct OpIter {
  int n[2];
  int j, sub;
  __device__ OpIter(int na, int nb_) : j(0), sub(-2) {
    n[0] = na;
    n[1] = nb_;
  }
  // kind: 0 = S (consumes a K pair), 1 = PV (consumes a V pair)
  __device__ bool next(int& kind, int& x, int& step) {
    while (true) {
      if (sub == -2) {
        sub = -1;
        if (n[0] > 0) { kind = 0; x = 0; step = 0; return true; }
        continue;
      }
      if (sub == -1) {
        sub = 0;
        if (n[1] > 0) { kind = 0; x = 1; step = 0; return true; }
        continue;
      }
      if (j >= (n[0] > n[1] ? n[0] : n[1])) return false;
      const int s = sub, jj = j;
      if (++sub == 4) {
        sub = 0;
        ++j;
      }
      const int t = s >> 1;
      const int nt = t ? n[1] : n[0];
      if ((s & 1) == 0) {
        if (jj < nt) { kind = 1; x = t; step = jj; return true; }
      } else {
        if (jj + 1 < nt) { kind = 0; x = t; step = jj + 1; return true; }
      }
    }
  }
};

__device__ __forceinline__ void fail(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

// Ring position of S_X(step) in the MMA issue order
//   S_A0 S_B0 | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) | ...
// (n0, n1 = the tiles' step counts). The commit that frees this K slot is
// also the softmax's signal that S_X(step) is complete.
__device__ __forceinline__ int s_op_index(int x, int step, int n0, int n1) {
  if (step == 0) return x == 0 ? 0 : (n0 > 0 ? 1 : 0);
  const int i = step - 1;  // the loop iteration that issues S_X(step)
  const int c = min(i, n0) + min(i, max(n0 - 1, 0)) + min(i, n1) + min(i, max(n1 - 1, 0));
  const int base = (n0 > 0) + (n1 > 0) + c;
  return x == 0 ? base + 1 : base + (i < n0) + (i + 1 < n0) + 1;
}

__device__ __forceinline__ int step_blocks(const Tile& t, int step) {
  return (t.n_u - 2 * step) >= 2 ? 2 : 1;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const Geometry g) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int pair = blockIdx.x;
#if SA_TRACE
  const bool tr = int(blockIdx.x) == g_attn_trace_cta[0] && int(blockIdx.y) == g_attn_trace_cta[1];
  if (tr && threadIdx.x == 0) g_attn_trace[kTraceSoftmax - 1] = clock64();
#endif

  Tile tile[2];
#pragma unroll
  for (int x = 0; x < 2; ++x) {
    const int pos = 2 * pair + x;  // position in the head's tile order
    tile[x].qa = tile[x].qb = -1;
    tile[x].n_u = tile[x].nsteps = 0;
    tile[x].list = nullptr;
    tile[x].glist = nullptr;
    if (pos < g.ntile) {
      const int t = a.order[size_t(bh) * g.ntile + pos];
      tile_blocks(g, t, tile[x].qa, tile[x].qb);
      tile[x].n_u = a.tcnt[size_t(bh) * g.ntile + t];
      tile[x].nsteps = (tile[x].n_u + 1) >> 1;
      const int32_t* src = a.tidx + (size_t(bh) * g.ntile + t) * g.nb;
      tile[x].glist = src;
      // every warp reads the lists at each step: stage them in shared memory
      const int staged = tile[x].n_u < kMaxList ? tile[x].n_u : kMaxList;
      for (int i = threadIdx.x; i < staged; i += kThreads) sm.list[x][i] = src[i];
    }
    tile[x].list = sm.list[x];
  }
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int x = 0; x < 2; ++x) {
      mbar_init(&sm.q_full[x], 1);
      mbar_init(&sm.p_full[x], 128);
      mbar_init(&sm.o_final[x], 1);
    }
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  const uint32_t tmem = sm.tmem_base;

  // Warpgroup 0 (three producers and the MMA issuer) gives registers to the
  // softmax warpgroups: 128 x 72 + 256 x 216 = 384 x 168, the launch's
  // allocation.
  if (warp < 4) {
    setmaxnreg_dec<72>();
  if (warp != 1) {
    // -------------------------------------------------------------- producers
    // Warps 0, 2 and 3 each issue every third op's TMA loads: a single
    // issuing thread cannot keep enough boxes in flight to feed the MMAs.
    const int prod = warp == 0 ? 0 : warp - 1;  // 0, 1, 2
    if (lane == 0) {
      if (prod == 0) {
        prefetch_tensormap(&a.map_q);
        prefetch_tensormap(&a.map_k);
        prefetch_tensormap(&a.map_v);
        prefetch_tensormap(&a.map_k2);
        prefetch_tensormap(&a.map_v2);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (tile[x].nsteps == 0) continue;
          mbar_arrive_expect_tx(&sm.q_full[x], 128u * D * 2u);
          for (int e = 0; e < 2; ++e) {
            const int blk = (e == 0 || tile[x].qb < 0) ? tile[x].qa : tile[x].qb;
            int t, hp, wp;
            block_coords(g, blk, t, hp, wp);
            for (int c = 0; c < D / 64; ++c)
              tma_load_5d(&sm.q[x][c][e * 8192], &a.map_q, &sm.q_full[x], c * 64, wp * g.pw, hp * g.ph,
                          t * g.pt, bh);
          }
        }
      }
      OpIter it(tile[0].nsteps, tile[1].nsteps);
      int kind, x, step, k = 0, last_issued = -1;
      while (it.next(kind, x, step)) {
        if (k % kProducers != prod) {
          ++k;
          continue;
        }
        const int s = k % kSlots, use = k / kSlots;
        if (use > 0 && !mbar_wait(&sm.empty[s], (use - 1) & 1, abort)) {
          fail(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        if (*abort) break;
        if (k == 0 && (a.debug_flags & SA_DEBUG_STALL_LOADER)) {
          ++k;  // test hook: never fill the first slot
          continue;
        }
        const Tile t = x ? tile[1] : tile[0];
        const int nblk = step_blocks(t, step);
        mbar_arrive_expect_tx(&sm.full[s], uint32_t(nblk) * 64u * D * 2u);
        const int e0 = list_at(t, 2 * step);
        if (nblk == 2 && (e0 & kEntryTPair) && (e0 & kEntryBlockMask) + g.nh * g.nw < g.nb) {
          // the same patch in frames t, t+1: one two-frame box per channel half
          int tt, hp, wp;
          block_coords(g, e0 & kEntryBlockMask, tt, hp, wp);
          const CUtensorMap* map = kind == 0 ? &a.map_k2 : &a.map_v2;
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.slot[s][c][0], map, &sm.full[s], c * 64, wp * g.pw, hp * g.ph, tt * g.pt, bh);
        } else {
          const CUtensorMap* map = kind == 0 ? &a.map_k : &a.map_v;
          for (int e = 0; e < nblk; ++e) {
            int kb = list_at(t, 2 * step + e) & kEntryBlockMask;
            if (kb >= g.nb) {
              atomicOr(a.status, kDevErrBadIndex);
              kb = 0;
            }
            int tt, hp, wp;
            block_coords(g, kb, tt, hp, wp);
            for (int c = 0; c < D / 64; ++c)
              tma_load_5d(&sm.slot[s][c][e * 8192], map, &sm.full[s], c * 64, wp * g.pw, hp * g.ph,
                          tt * g.pt, bh);
          }
        }
        last_issued = k;
        ++k;
      }
      if (*abort && last_issued >= 0) {
        // let this warp's own copies land before the CTA can exit
        // (time-bounded, ignoring the abort flag); at most one op per slot
        // can still be in flight
        int never = 0;
        for (int kk = last_issued; kk >= 0 && kk > last_issued - kSlots; kk -= kProducers)
          mbar_wait(&sm.full[kk % kSlots], (kk / kSlots) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    // One thread issues every MMA; its SMSP is shared with two busy softmax
    // warps, so the bookkeeping between MMA batches is kept to a minimum
    // (each instruction here idles the tensor core once its short queue
    // drains), and each op's MMAs go out from one asm block with no compiler
    // instructions between them (3-4 % faster than one asm per MMA).
    if (lane == 0) {
      const uint32_t id_s2 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_pv = idesc_bf16_f32(128, D, 0, 1);
      // Descriptors differ only in the start-address field (bits 0-13, in
      // 16-byte units), so each MMA below is one 32-bit add from a base.
      const uint64_t kdesc0 = sw128_desc(smem_u32(&sm.slot[0][0][0]), 16, 1024);
      const uint64_t vdesc0 = sw128_desc(smem_u32(&sm.slot[0][0][0]), kChunkBytes, 1024);
      const uint64_t qdesc0 = sw128_desc(smem_u32(&sm.q[0][0][0]), 16, 1024);
      const uint64_t qdesc1 = sw128_desc(smem_u32(&sm.q[1][0][0]), 16, 1024);
      constexpr uint32_t kSlotStep = (D / 64) * kChunkBytes / 16;  // one slot, 16 B units
      const int n0 = tile[0].nsteps, n1 = tile[1].nsteps;
      const int u0 = tile[0].n_u, u1 = tile[1].n_u;
      bool ok = mbar_wait(&sm.q_full[0], 0, abort);
      if (ok && n1 > 0) ok = mbar_wait(&sm.q_full[1], 0, abort);
      int k = 0;  // op index (ring position)
#if SA_TRACE
      int tr_u = 0;
#endif
      // S_X(step) = Q_X K^T into tile X's S columns, the K pair in slot s
      auto mma_s = [&](int x, int step, int s) {
        const uint64_t qd = x ? qdesc1 : qdesc0;
        const uint64_t kd = kdesc0 + uint64_t(s) * kSlotStep;
        const uint32_t id = ((x ? u1 : u0) - 2 * step) >= 2 ? id_s2 : id_s1;
        const uint32_t d_tmem = tmem + col_s(x);
        if constexpr (D == 128) {
          mma_ss_k8<kChunkBytes>(d_tmem, qd, kd, id, 0u);
        } else {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (uint32_t(kk >> 2) * kChunkBytes + uint32_t(kk & 3) * 32u) >> 4;
            mma_ss(d_tmem, qd + off, kd + off, id, kk > 0);
          }
        }
      };
      // O_X += P_X V, P from tile X's S columns in TMEM, the V pair in slot s
      auto mma_pv = [&](int x, int step, int s) {
        const uint64_t vd = vdesc0 + uint64_t(s) * kSlotStep;
        const uint32_t o_tmem = tmem + col_o(x);
        const uint32_t p_tmem = tmem + col_s(x);
        if (((x ? u1 : u0) - 2 * step) >= 2)
          mma_ts_k<8>(o_tmem, p_tmem, vd, id_pv, step > 0 ? 1u : 0u);
        else
          mma_ts_k<4>(o_tmem, p_tmem, vd, id_pv, step > 0 ? 1u : 0u);
      };
      // the order the producers fill: S_A0 S_B0 | PV_A(j) S_A(j+1) PV_B(j) S_B(j+1) | ...
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if (!ok || (x ? n1 : n0) == 0) continue;
        const int s = k & (kSlots - 1);
        ok = mbar_wait(&sm.full[s], (k / kSlots) & 1, abort);
        if (!ok) break;
        mma_s(x, 0, s);
        mma_commit(&sm.empty[s]);  // also tells the softmax that S_X(0) is complete
        ++k;
      }
      // One unit per tile and step: PV_X(j) and S_X(j+1) issued back to back
      // behind one round of waits (an idle tensor core between the two would
      // cost more than waiting for the K pair a little earlier).
      const int nmax = n0 > n1 ? n0 : n1;
      for (int j = 0; ok && j < nmax; ++j) {
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int nx = x ? n1 : n0;
          if (!ok || j >= nx) continue;
          const bool has_s = j + 1 < nx;
#if SA_TRACE
          const long long tr_t0 = clock64();
#endif
          const int s_pv = k & (kSlots - 1), s_s = (k + 1) & (kSlots - 1);
          const uint32_t par_pv = (k / kSlots) & 1, par_s = ((k + 1) / kSlots) & 1;
          // one round trip for all three barriers; a bounded wait only for
          // those not yet complete
          const uint32_t ready = mbar_peek3(&sm.p_full[x], j & 1, &sm.full[s_pv], par_pv,
                                            has_s ? &sm.full[s_s] : &sm.full[s_pv],
                                            has_s ? par_s : par_pv);
          if (ready != 7u) {
            ok = ((ready & 1u) || mbar_wait(&sm.p_full[x], j & 1, abort)) &&
                 ((ready & 2u) || mbar_wait(&sm.full[s_pv], par_pv, abort)) &&
                 ((ready & 4u) || !has_s || mbar_wait(&sm.full[s_s], par_s, abort));
            if (!ok) break;
          }
#if SA_TRACE
          const long long tr_t1 = clock64();
#endif
          tc_fence_after_sync();  // P was written by the softmax threads
          mma_pv(x, j, s_pv);
          mma_commit(&sm.empty[s_pv]);
          if (has_s) {
            mma_s(x, j + 1, s_s);
            mma_commit(&sm.empty[s_s]);  // also tells the softmax that S_X(j+1) is complete
            k += 2;
          } else {
            mma_commit(&sm.o_final[x]);
            k += 1;
          }
#if SA_TRACE
          if (tr && tr_u < kTraceUnits) {
            g_attn_trace[3 * tr_u] = tr_t0;
            g_attn_trace[3 * tr_u + 1] = tr_t1;
            g_attn_trace[3 * tr_u + 2] = clock64();
          }
          ++tr_u;
#endif
        }
      }
      if (!ok) {
        fail(a.status, &sm.abort, kDevErrTimeoutMma);
        mma_commit(&sm.drain);  // wait for this thread's in-flight MMAs
        int never = 0;
        mbar_wait(&sm.drain, 0, &never);
      }
    }
  }
  } else {
    setmaxnreg_inc<216>();
    // -------------------------------------------------------------- softmax
    const int x = (warp - 4) >> 2;  // 0: tile A, 1: tile B
    const Tile t = x ? tile[1] : tile[0];
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // tile row == TMEM lane
    const int half = r >> 6;
    const bool row_valid = t.nsteps > 0 && (half == 0 || t.qb >= 0);
    const int keep_bit = half ? kEntryKeepB : kEntryKeepA;
    const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
    const uint32_t s_col = t_lane + col_s(x);
    const uint32_t o_col = t_lane + col_o(x);
    const float sl2 = a.scale_log2;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < t.nsteps; ++j) {
      const int nblk = step_blocks(t, j);
      const int e0 = list_at(t, 2 * j);
      const int e1 = nblk == 2 ? list_at(t, 2 * j + 1) : 0;
      const bool keep0 = row_valid && (e0 & keep_bit);
      const bool keep1 = row_valid && nblk == 2 && (e1 & keep_bit);
      const int ks = s_op_index(x, j, tile[0].nsteps, tile[1].nsteps);
      ok = __all_sync(0xFFFFFFFFu,
                      mbar_wait(&sm.empty[ks & (kSlots - 1)], (ks / kSlots) & 1, abort));
      if (!ok) break;
#if SA_TRACE
      if (tr && lane == 0 && j < kTraceSteps)
        g_attn_trace[kTraceSoftmax + (warp - 4) * 2 * kTraceSteps + 2 * j] = clock64();
#endif
      tc_fence_after_sync();
      // keep0 / keep1 are uniform across a warp (a warp's rows lie in one
      // q-block), so the warp-collective loads may be skipped per block
      uint32_t sv[128];
      if (keep0) {
        tmem_ld32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      }
      if (keep1) {
        tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
        tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
      }
      tmem_wait_ld();
      // row max over four independent chains (a single chain of 64 dependent
      // max3 would cost its full latency)
      float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (keep0) {
#pragma unroll
        for (int i = 0; i < 64; i += 2)
          mq[(i >> 1) & 3] = max3(mq[(i >> 1) & 3], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
      }
      if (keep1) {
#pragma unroll
        for (int i = 64; i < 128; i += 2)
          mq[(i >> 1) & 3] = max3(mq[(i >> 1) & 3], __uint_as_float(sv[i]), __uint_as_float(sv[i + 1]));
      }
      float mx = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
      mx *= sl2;
      const bool need = mx > m + kRescaleThreshold;  // false while mx = -inf
      const float m_new = need ? mx : m;
      const float alpha = need ? ex2_approx(m - m_new) : 1.f;  // m = -inf -> 0
      if (__any_sync(0xFFFFFFFFu, need) && j > 0) {
        // PV_X(j-1) was issued before S_X(j): it is complete here.
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(o_col + 32 * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(o_col + 32 * c, o);
        }
      }
      m = m_new;
      l *= alpha;
      // p = 2^(s * log2(e)/sqrt(d) - m), two columns per packed op;
      // kPolyPairsPer8 of every 8 column pairs take the FMA-pipe exp2.
      const uint64_t sl2x2 = f2_pack(sl2, sl2);
      const uint64_t negm2 = f2_pack(-m, -m);
      uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};  // four independent packed sums
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const bool kp = (2 * i) < 64 ? keep0 : keep1;
        uint32_t packed = 0u;
        if (kp) {
          const uint64_t x2 =
              f2_fma(f2_pack(__uint_as_float(sv[2 * i]), __uint_as_float(sv[2 * i + 1])), sl2x2,
                     negm2);
          float x0, x1;
          f2_unpack(x2, x0, x1);
          uint64_t e2;
          if ((i & 7) >= 8 - kPolyPairsPer8) {
            e2 = exp2_poly_x2(f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f)));
          } else {
            e2 = f2_pack(ex2_approx(x0), ex2_approx(x1));
          }
          rs2[i & 3] = f2_add(rs2[i & 3], e2);
          float p0, p1;
          f2_unpack(e2, p0, p1);
          packed = pack_bf16x2(p0, p1);
        }
        sv[i] = packed;
      }
      float rs_lo, rs_hi;
      f2_unpack(f2_add(f2_add(rs2[0], rs2[1]), f2_add(rs2[2], rs2[3])), rs_lo, rs_hi);
      const float rs = rs_lo + rs_hi;
      l += rs;
      tmem_st32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
      if (nblk == 2) tmem_st32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&sm.p_full[x]);
#if SA_TRACE
      if (tr && lane == 0 && j < kTraceSteps)
        g_attn_trace[kTraceSoftmax + (warp - 4) * 2 * kTraceSteps + 2 * j + 1] = clock64();
#endif
    }
    if (t.nsteps > 0) {
      if (!ok) {
        fail(a.status, &sm.abort, kDevErrTimeoutSoftmax);
      } else if (__all_sync(0xFFFFFFFFu, mbar_wait(&sm.o_final[x], 0, abort))) {
        tc_fence_after_sync();
        // ---- epilogue: O / l -> natural token position
        if (row_valid) {
          const int blk = half ? t.qb : t.qa;
          int tt, hp, wp;
          block_coords(g, blk, tt, hp, wp);
          // row i of the block: frame tt*pt + (i >> (lph + lpw)), row
          // hp*ph + ((i >> lpw) & (ph - 1)), column wp*pw + (i & (pw - 1))
          const int i = r & 63;
          const int run = i >> g.lpw;
          const size_t tok = (size_t(tt) * g.pt + (run >> g.lph)) * g.Hh * g.Ww +
                             size_t(hp * g.ph + (run & (g.ph - 1))) * g.Ww +
                             size_t(wp * g.pw + (i & (g.pw - 1)));
          const size_t row = size_t(bh) * g.S + tok;
          const float inv = l > 0.f ? 1.0f / l : 0.f;
          // log-sum-exp of the row's kept scaled scores (natural log): m is
          // in log2 units and l is the sum relative to 2^m
          if (a.lse != nullptr)
            a.lse[row] = l > 0.f ? (m + __log2f(l)) * 0.6931471805599453f : -INFINITY;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(o_col + 32 * c, o);
            tmem_wait_ld();
            if (a.out_fp32) {
              float4* dst =
                  reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * D + 32 * c);
#pragma unroll
              for (int v4 = 0; v4 < 8; ++v4)
                dst[v4] = make_float4(__uint_as_float(o[4 * v4]) * inv,
                                      __uint_as_float(o[4 * v4 + 1]) * inv,
                                      __uint_as_float(o[4 * v4 + 2]) * inv,
                                      __uint_as_float(o[4 * v4 + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.out) + row * D +
                                                    32 * c);
#pragma unroll
              for (int v8 = 0; v8 < 4; ++v8)
                dst[v8] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * v8]) * inv,
                                                 __uint_as_float(o[8 * v8 + 1]) * inv),
                                     pack_bf16x2(__uint_as_float(o[8 * v8 + 2]) * inv,
                                                 __uint_as_float(o[8 * v8 + 3]) * inv),
                                     pack_bf16x2(__uint_as_float(o[8 * v8 + 4]) * inv,
                                                 __uint_as_float(o[8 * v8 + 5]) * inv),
                                     pack_bf16x2(__uint_as_float(o[8 * v8 + 6]) * inv,
                                                 __uint_as_float(o[8 * v8 + 7]) * inv));
            }
          }
        }
      } else {
        fail(a.status, &sm.abort, kDevErrTimeoutSoftmax);
      }
    }
  }

  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

template <int D>
static cudaError_t launch_attn_d(const AttnArgs& a, const Geometry& g, cudaStream_t stream) {
  // At least 120 KB so that one CTA occupies an SM: each CTA allocates all
  // 512 TMEM columns.
  const size_t need = sizeof(AttnSmem<D>) + 1024;
  const size_t smem = need > 120 * 1024 ? need : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned((g.ntile + 1) / 2), unsigned(g.BH));
  attn_kernel<D><<<grid, kThreads, smem, stream>>>(a, g);
  return cudaGetLastError();
}

cudaError_t launch_attn(const AttnArgs& a, const Geometry& g, cudaStream_t stream) {
  return g.d == 128 ? launch_attn_d<128>(a, g, stream) : launch_attn_d<64>(a, g, stream);
}

}  // namespace sa

#if SA_TRACE
// Diagnostics build only: choose the traced CTA, read the stamps back.
extern "C" int sparse_attn_trace_select(int bx, int by) {
  const int v[2] = {bx, by};
  long long zero[sa::kTraceWords] = {};
  if (cudaMemcpyToSymbol(sa::g_attn_trace, zero, sizeof(zero)) != cudaSuccess) return 1;
  return cudaMemcpyToSymbol(sa::g_attn_trace_cta, v, sizeof(v)) != cudaSuccess;
}
extern "C" int sparse_attn_trace_read(long long* dst, int n) {
  if (n > sa::kTraceWords) n = sa::kTraceWords;
  return cudaMemcpyFromSymbol(dst, sa::g_attn_trace, sizeof(long long) * n) != cudaSuccess;
}
#endif
