// Block-sparse attention forward over the kept (q-block, k-block) pairs
// ("Espansione", NABLA Metodologia 2: every dropped N x N block is -inf), on
// the sm_100a tensor cores.
//
// A CTA computes one query tile of 128 rows = two q-blocks (64 rows each) of
// one head, iterating over the union of their kept k-block lists two
// k-blocks (128 keys) per step. Rows of a q-block that does not keep a
// k-block see it as -inf (no exponentials are evaluated for it).
//
//   warp 0      TMA producer: Q tile once, then K/V of each step into a
//               2-stage ring. Q/K/V are read in natural layout through 5-D
//               tensor maps whose box is one 8x8 patch of one frame, so the
//               fractal flattening is pure addressing.
//   warp 1      owns TMEM (512 columns) and issues tcgen05.mma:
//                 S_j  = Q K_j^T  (SS, M=128, N=64*nblk, K=d) -> TMEM S[j%2]
//                 O   += P_j V_j  (TS: P from TMEM, V MN-major from smem)
//               S_{j+1} is issued before PV_j so the tensor core works while
//               the softmax warps process S_j.
//   warps 2-5   one thread per query row (TMEM lane): online softmax in fp32
//               (exp2 domain), P written back as bf16 over S in TMEM, O
//               rescaled in TMEM only when the running max grows by more than
//               2^8 (exact after the final 1/l), epilogue stores O / l to the
//               row's natural token position.
//
// All waits are bounded (sm100.cuh); a wait that runs out records a status
// bit, raises a CTA-wide abort flag, drains its own in-flight work and lets
// the CTA free TMEM and exit.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

namespace {

constexpr int kThreads = 192;
constexpr int kChunkBytes = 128 * 128;  // 128 rows x 128 B (64 bf16 channels)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO = 256;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

template <int D>
struct __align__(1024) AttnSmem {
  uint8_t q[D / 64][kChunkBytes];
  uint8_t k[2][D / 64][kChunkBytes];
  uint8_t v[2][D / 64][kChunkBytes];
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t pv_done;
  uint64_t o_final;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_kernel(const __grid_constant__ AttnArgs a, const Geometry g) {
  const CUtensorMap* map_q = &a.map_q;
  const CUtensorMap* map_k = &a.map_k;
  const CUtensorMap* map_v = &a.map_v;
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D>& sm = *reinterpret_cast<AttnSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  int qa, qb;
  tile_blocks(g, tile, qa, qb);
  const int n_u = a.tcnt[size_t(bh) * g.ntile + tile];
  const int32_t* list = a.tidx + (size_t(bh) * g.ntile + tile) * g.nb;
  const int nsteps = (n_u + 1) >> 1;
  volatile int* abort = &sm.abort;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
    }
    mbar_init(&sm.pv_done, 1);
    mbar_init(&sm.o_final, 1);
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

  if (nsteps > 0) {
    if (warp == 0) {
      // ------------------------------------------------------------ producer
      if (lane == 0) {
        prefetch_tensormap(map_q);
        prefetch_tensormap(map_k);
        prefetch_tensormap(map_v);
        mbar_arrive_expect_tx(&sm.q_full, 128u * D * 2u);
        for (int e = 0; e < 2; ++e) {
          const int blk = (e == 0 || qb < 0) ? qa : qb;
          int t, hp, wp;
          block_coords(g, blk, t, hp, wp);
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.q[c][e * 8192], map_q, &sm.q_full, c * 64, wp * 8, hp * 8, t, bh);
        }
        int issued_hi = -1;  // last step whose loads were issued
        for (int j = 0; j < nsteps; ++j) {
          const int s = j & 1;
          if (j >= 2 && !mbar_wait(&sm.kv_empty[s], ((j >> 1) - 1) & 1, abort)) {
            fail(a.status, &sm.abort, kDevErrTimeoutLoad);
            break;
          }
          if (*abort) break;
          if (j == 0 && (a.debug_flags & SA_DEBUG_STALL_LOADER)) continue;
          const int nblk = (n_u - 2 * j) >= 2 ? 2 : 1;
          mbar_arrive_expect_tx(&sm.kv_full[s], uint32_t(nblk) * 2u * 64u * D * 2u);
          for (int e = 0; e < nblk; ++e) {
            int kb = list[2 * j + e] & kEntryBlockMask;
            if (kb >= g.nb) {
              atomicOr(a.status, kDevErrBadIndex);
              kb = 0;
            }
            int t, hp, wp;
            block_coords(g, kb, t, hp, wp);
            for (int c = 0; c < D / 64; ++c) {
              tma_load_5d(&sm.k[s][c][e * 8192], map_k, &sm.kv_full[s], c * 64, wp * 8, hp * 8, t,
                          bh);
              tma_load_5d(&sm.v[s][c][e * 8192], map_v, &sm.kv_full[s], c * 64, wp * 8, hp * 8, t,
                          bh);
            }
          }
          issued_hi = j;
        }
        if (*abort) {
          // let this CTA's own copies land before the CTA can exit (the wait
          // ignores the abort flag but is still time-bounded)
          int never = 0;
          for (int j = (issued_hi > 0 ? issued_hi - 1 : 0); j <= issued_hi; ++j)
            mbar_wait(&sm.kv_full[j & 1], (j >> 1) & 1, &never);
        }
      }
    } else if (warp == 1) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint32_t id_s2 = idesc_bf16_f32(128, 128, 0, 0);
        const uint32_t id_s1 = idesc_bf16_f32(128, 64, 0, 0);
        const uint32_t id_pv = idesc_bf16_f32(128, D, 0, 1);
        const uint32_t q_addr = smem_u32(&sm.q[0][0]);
        bool ok = mbar_wait(&sm.q_full, 0, abort);
        auto issue_s = [&](int j) {
          const int s = j & 1;
          const int nblk = (n_u - 2 * j) >= 2 ? 2 : 1;
          const uint32_t k_addr = smem_u32(&sm.k[s][0][0]);
          const uint32_t d_tmem = tmem + (s ? kColS1 : kColS0);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = uint32_t(kk >> 2) * kChunkBytes + uint32_t(kk & 3) * 32u;
            mma_ss(d_tmem, sw128_desc(q_addr + off, 16, 1024), sw128_desc(k_addr + off, 16, 1024),
                   nblk == 2 ? id_s2 : id_s1, kk > 0);
          }
          mma_commit(&sm.s_full[s]);
        };
        if (ok) ok = mbar_wait(&sm.kv_full[0], 0, abort);
        if (ok) {
          tc_fence_after_sync();
          issue_s(0);
        }
        for (int j = 0; ok && j < nsteps; ++j) {
          if (j + 1 < nsteps) {
            ok = mbar_wait(&sm.kv_full[(j + 1) & 1], ((j + 1) >> 1) & 1, abort);
            if (!ok) break;
            tc_fence_after_sync();
            issue_s(j + 1);
          }
          ok = mbar_wait(&sm.p_full[j & 1], (j >> 1) & 1, abort);
          if (!ok) break;
          tc_fence_after_sync();
          const int s = j & 1;
          const int nblk = (n_u - 2 * j) >= 2 ? 2 : 1;
          const uint32_t v_addr = smem_u32(&sm.v[s][0][0]);
          const uint32_t p_tmem = tmem + (s ? kColS1 : kColS0);
          for (int kk = 0; kk < 4 * nblk; ++kk)
            mma_ts(tmem + kColO, p_tmem + uint32_t(kk) * 8u,
                   sw128_desc(v_addr + uint32_t(kk) * 2048u, kChunkBytes, 1024), id_pv,
                   (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.pv_done);
          mma_commit(&sm.kv_empty[s]);
        }
        if (ok) {
          mma_commit(&sm.o_final);
        } else {
          fail(a.status, &sm.abort, kDevErrTimeoutMma);
          mma_commit(&sm.drain);  // wait for this thread's in-flight MMAs
          int never = 0;
          mbar_wait(&sm.drain, 0, &never);
        }
      }
    } else {
      // ------------------------------------------------------------ softmax
      const int quad = warp & 3;
      const int r = quad * 32 + lane;  // tile row == TMEM lane
      const int half = r >> 6;
      const bool row_valid = half == 0 || qb >= 0;
      const int keep_bit = half ? kEntryKeepB : kEntryKeepA;
      const uint32_t t_lane = tmem + (uint32_t(quad * 32) << 16);
      const float sl2 = a.scale_log2;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      for (int j = 0; j < nsteps; ++j) {
        const int s = j & 1;
        const int nblk = (n_u - 2 * j) >= 2 ? 2 : 1;
        const int e0 = list[2 * j];
        const int e1 = nblk == 2 ? list[2 * j + 1] : 0;
        const bool keep0 = row_valid && (e0 & keep_bit);
        const bool keep1 = row_valid && nblk == 2 && (e1 & keep_bit);
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full[s], (j >> 1) & 1, abort));
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t s_col = t_lane + (s ? kColS1 : kColS0);
        uint32_t sv[128];
        tmem_ld32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        tmem_ld32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        if (nblk == 2) {
          tmem_ld32(s_col + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
          tmem_ld32(s_col + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
        }
        tmem_wait_ld();
        float mx = -INFINITY;
        if (keep0) {
#pragma unroll
          for (int i = 0; i < 64; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
        }
        if (keep1) {
#pragma unroll
          for (int i = 64; i < 128; ++i) mx = fmaxf(mx, __uint_as_float(sv[i]));
        }
        mx *= sl2;
        const bool need = mx > m + kRescaleThreshold;  // false while mx = -inf
        const float m_new = need ? mx : m;
        const float alpha = need ? ex2_approx(m - m_new) : 1.f;  // m = -inf -> 0
        if (__any_sync(0xFFFFFFFFu, need) && j > 0) {
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.pv_done, (j - 1) & 1, abort));
          if (!ok) break;
          tc_fence_after_sync();
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_lane + kColO + 32 * c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_lane + kColO + 32 * c, o);
          }
        }
        m = m_new;
        l *= alpha;
        const float neg_m = -m;
        float rs = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          float p0 = 0.f, p1 = 0.f;
          const int base = 2 * i;
          const bool kp = base < 64 ? keep0 : keep1;
          if (kp) {
            p0 = ex2_approx(fmaf(__uint_as_float(sv[base]), sl2, neg_m));
            p1 = ex2_approx(fmaf(__uint_as_float(sv[base + 1]), sl2, neg_m));
          }
          rs += p0 + p1;
          sv[i] = pack_bf16x2(p0, p1);
        }
        l += rs;
        tmem_st32(s_col + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
        if (nblk == 2) tmem_st32(s_col + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
        tmem_wait_st();
        tc_fence_before_sync();
        mbar_arrive(&sm.p_full[s]);
      }
      if (!ok) {
        fail(a.status, &sm.abort, kDevErrTimeoutSoftmax);
      } else if (__all_sync(0xFFFFFFFFu, mbar_wait(&sm.o_final, 0, abort))) {
        tc_fence_after_sync();
        // ---- epilogue: O / l -> natural token position
        const int blk = half ? qb : qa;
        if (row_valid) {
          int t, hp, wp;
          block_coords(g, blk, t, hp, wp);
          const int i = r & 63;
          const size_t tok = size_t(t) * g.Hh * g.Ww + size_t(hp * 8 + (i >> 3)) * g.Ww +
                             size_t(wp * 8 + (i & 7));
          const size_t row = size_t(bh) * g.S + tok;
          const float inv = l > 0.f ? 1.0f / l : 0.f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(t_lane + kColO + 32 * c, o);
            tmem_wait_ld();
            if (a.out_fp32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.out) + row * D + 32 * c);
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
  const size_t smem = sizeof(AttnSmem<D>) + 1024 > 120 * 1024 ? sizeof(AttnSmem<D>) + 1024
                                                               : 120 * 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  const dim3 grid(unsigned(g.ntile), unsigned(g.BH));
  attn_kernel<D><<<grid, kThreads, smem, stream>>>(a, g);
  return cudaGetLastError();
}

cudaError_t launch_attn(const AttnArgs& a, const Geometry& g, cudaStream_t stream) {
  return g.d == 128 ? launch_attn_d<128>(a, g, stream) : launch_attn_d<64>(a, g, stream);
}

}  // namespace sa
