// Gradients of the block-sparse attention, for the training use of the mask
// (the NABLA page trains a DiT with the same block mask, "Risultati
// Sperimentali"): with s = q.k / sqrt(d) on the kept blocks, P the row
// softmax over the kept keys and O = P V, for an output gradient dO
//   dV = P^T dO,  dP = dO V^T,  D_i = sum_c dO_ic O_ic,  dS = P * (dP - D),
//   dQ = dS K / sqrt(d),  dK = dS^T Q / sqrt(d).
// P is recomputed from the forward's row log-sum-exp: P = 2^(s log2(e) - lse2).
//
// Four launches: prep (D and lse2 into fractal order), lists (per key tile the
// q-blocks that keep it, from the keep bitmaps), the key-stationary tcgen05
// kernel (dK, dV per key tile; dQ reduced into an fp32 accumulator), and the
// dQ conversion.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

namespace {

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

// One thread per (bh, fractal position): D = dO . O over the d channels and
// lse2 = lse * log2(e), both written in fractal order.
template <int D>
__global__ void __launch_bounds__(256)
    bwd_prep_kernel(const void* __restrict__ o, const __nv_bfloat16* __restrict__ dout,
                    const float* __restrict__ lse, float* __restrict__ lse2,
                    float* __restrict__ dsum, int o_fp32, Geometry g) {
  const long p = long(blockIdx.x) * blockDim.x + threadIdx.x;
  if (p >= long(g.BH) * g.S) return;
  const int bh = int(p / g.S), pos = int(p - long(bh) * g.S);
  const size_t row = size_t(bh) * g.S + block_row_token(g, pos >> 6, pos & 63);
  const uint4* dr = reinterpret_cast<const uint4*>(dout + row * D);
  float acc = 0.f;
  if (o_fp32) {
    const float4* orow = reinterpret_cast<const float4*>(static_cast<const float*>(o) + row * D);
#pragma unroll 4
    for (int v = 0; v < D / 8; ++v) {
      const uint4 dv = __ldg(dr + v);
      const float4 oa = __ldg(orow + 2 * v), ob = __ldg(orow + 2 * v + 1);
      const float2 d0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.x));
      const float2 d1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.y));
      const float2 d2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.z));
      const float2 d3 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&dv.w));
      acc += d0.x * oa.x + d0.y * oa.y + d1.x * oa.z + d1.y * oa.w;
      acc += d2.x * ob.x + d2.y * ob.y + d3.x * ob.z + d3.y * ob.w;
    }
  } else {
    const uint4* orow =
        reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(o) + row * D);
#pragma unroll 4
    for (int v = 0; v < D / 8; ++v) {
      const uint4 dv = __ldg(dr + v), ov = __ldg(orow + v);
      const uint32_t* dw = &dv.x;
      const uint32_t* ow = &ov.x;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(dw + w));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(ow + w));
        acc += a.x * b.x + a.y * b.y;
      }
    }
  }
  dsum[p] = acc;
  lse2[p] = lse[row] * kLog2e;
}

cudaError_t launch_bwd_prep(const void* o, const void* do_, const float* lse, float* lse2,
                            float* dsum, int o_fp32, const Geometry& g, cudaStream_t stream) {
  const long n = long(g.BH) * g.S;
  const unsigned grid = unsigned((n + 255) / 256);
  const auto* dd = static_cast<const __nv_bfloat16*>(do_);
  if (g.d == 128)
    bwd_prep_kernel<128><<<grid, 256, 0, stream>>>(o, dd, lse, lse2, dsum, o_fp32, g);
  else
    bwd_prep_kernel<64><<<grid, 256, 0, stream>>>(o, dd, lse, lse2, dsum, o_fp32, g);
  return cudaGetLastError();
}

// One warp per (bh, key tile): scan every q-block's keep bitmap for the
// tile's two k-blocks (the query-tile pairing applied to keys) and compact
// the q-blocks keeping either, ascending.
__global__ void __launch_bounds__(256)
    bwd_lists_kernel(const uint32_t* __restrict__ bits, int32_t* __restrict__ kcnt,
                     int32_t* __restrict__ kidx, Geometry g) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long unit = long(blockIdx.x) * 8 + warp;
  if (unit >= long(g.BH) * g.ntile) return;
  const int bh = int(unit / g.ntile), tile = int(unit - long(bh) * g.ntile);
  int ka, kb;
  tile_blocks(g, tile, ka, kb);
  const int words = bitmap_words(g);
  const uint32_t* rows = bits + size_t(bh) * g.nb * words;
  int32_t* out = kidx + size_t(unit) * g.nb;
  int n = 0;
  for (int i0 = 0; i0 < g.nb; i0 += 32) {
    const int i = i0 + lane;
    bool a = false, b = false;
    if (i < g.nb) {
      a = (rows[size_t(i) * words + (ka >> 5)] >> (ka & 31)) & 1u;
      if (kb >= 0) b = (rows[size_t(i) * words + (kb >> 5)] >> (kb & 31)) & 1u;
    }
    const unsigned m = __ballot_sync(0xFFFFFFFFu, a || b);
    if (a || b)
      out[n + __popc(m & ((1u << lane) - 1u))] =
          i | (a ? kEntryKeepA : 0) | (b ? kEntryKeepB : 0);
    n += __popc(m);
  }
  if (lane == 0) kcnt[unit] = n;
}

cudaError_t launch_bwd_lists(const uint32_t* bits, int32_t* kcnt, int32_t* kidx, const Geometry& g,
                             cudaStream_t stream) {
  const long units = long(g.BH) * g.ntile;
  bwd_lists_kernel<<<unsigned((units + 7) / 8), 256, 0, stream>>>(bits, kcnt, kidx, g);
  return cudaGetLastError();
}

// dq = dq_acc, four values per thread.
__global__ void __launch_bounds__(256)
    dq_convert_kernel(const float4* __restrict__ acc, void* __restrict__ dq, long n4, int out_fp32) {
  const long i = long(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  const float4 v = acc[i];
  if (out_fp32) {
    static_cast<float4*>(dq)[i] = v;
  } else {
    static_cast<uint2*>(dq)[i] = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
  }
}

cudaError_t launch_dq_convert(const float* dq_acc, void* dq, int out_fp32, const Geometry& g,
                              cudaStream_t stream) {
  const long n4 = long(g.BH) * g.S * g.d / 4;
  dq_convert_kernel<<<unsigned((n4 + 255) / 256), 256, 0, stream>>>(
      reinterpret_cast<const float4*>(dq_acc), dq, n4, out_fp32);
  return cudaGetLastError();
}

namespace {

constexpr int kBThreads = 192;        // warp 0 TMA, warp 1 MMA, warps 2-5 rows
constexpr int kBChunk = 128 * 128;    // 128 rows x 128 B (64 bf16 channels)
// TMEM columns: dV and dK accumulators (fp32, one key per lane); S^T, then P
// (bf16 pairs, in place), then dQ (fp32, one query row per lane); dP^T, then
// dS (bf16 pairs, in place).
constexpr uint32_t kColDV = 0, kColDK = 128, kColS = 256, kColDP = 384;

template <int D>
struct __align__(1024) BwdSmem {
  uint8_t k[D / 64][kBChunk];     // key tile: two k-blocks, 64 keys each
  uint8_t v[D / 64][kBChunk];
  uint8_t q[D / 64][kBChunk];     // the step's query rows: two q-blocks
  uint8_t dout[D / 64][kBChunk];
  uint8_t ds[2][kBChunk];         // dS as the MN-major A of dQ = dS K: [64-query chunk][key][64 q]
  float lse2[128], dsum[128];     // per query row of the step
  uint64_t kv_full, q_full, q_empty, do_full, do_empty, st_full;
  uint64_t s_full, p_full, dq_full, tmem_free, acc_full, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail_b(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

// 32 fp32 values -> row `row` of a [.][D] output, bf16 or fp32.
template <int D>
__device__ __forceinline__ void store_row32(void* out, size_t row, int col0, const float (&x)[32],
                                            int out_fp32) {
  if (out_fp32) {
    float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row * D + col0);
#pragma unroll
    for (int v = 0; v < 8; ++v) dst[v] = make_float4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
  } else {
    uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(out) + row * D + col0);
#pragma unroll
    for (int v = 0; v < 4; ++v)
      dst[v] = make_uint4(pack_bf16x2(x[8 * v], x[8 * v + 1]), pack_bf16x2(x[8 * v + 2], x[8 * v + 3]),
                          pack_bf16x2(x[8 * v + 4], x[8 * v + 5]),
                          pack_bf16x2(x[8 * v + 6], x[8 * v + 7]));
  }
}

}  // namespace

// One CTA per (key tile, bh): the key tile's K and V stay in shared memory;
// each step takes the next two q-blocks of its list (S^T = K Q^T and
// dP^T = V dO^T with the keys as the MMA's M), the row warps form P^T and
// dS^T, then dV += P^T dO, dK += dS^T Q and dQ = dS K, whose rows are added
// to the fp32 accumulator.
template <int D>
__global__ void __launch_bounds__(kBThreads, 1)
    bwd_kernel(const __grid_constant__ BwdArgs a, const Geometry g) {
  extern __shared__ uint8_t b_raw[];
  BwdSmem<D>& sm = *reinterpret_cast<BwdSmem<D>*>(
      (reinterpret_cast<uintptr_t>(b_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, bh = blockIdx.y;
  int ka, kb;
  tile_blocks(g, tile, ka, kb);
  const size_t unit = size_t(bh) * g.ntile + tile;
  const int cnt = a.kcnt[unit];
  const int32_t* ent = a.kidx + unit * g.nb;
  const int nsteps = (cnt + 1) / 2;
  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    mbar_init(&sm.do_full, 1);
    mbar_init(&sm.do_empty, 1);
    mbar_init(&sm.st_full, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, 128);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.tmem_free, 128);
    mbar_init(&sm.acc_full, 1);
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
    if (lane == 0 && nsteps > 0) {
      prefetch_tensormap(&a.map_q);
      prefetch_tensormap(&a.map_k);
      prefetch_tensormap(&a.map_v);
      prefetch_tensormap(&a.map_do);
      mbar_arrive_expect_tx(&sm.kv_full, 2u * 2u * 64u * D * 2u);
      for (int e = 0; e < 2; ++e) {
        const int blk = (e == 0 || kb < 0) ? ka : kb;  // a lone k-block: its copy fills the rest
        int t, hp, wp;
        block_coords(g, blk, t, hp, wp);
        for (int c = 0; c < D / 64; ++c) {
          tma_load_5d(&sm.k[c][e * 8192], &a.map_k, &sm.kv_full, c * 64, wp * g.pw, hp * g.ph,
                      t * g.pt, bh);
          tma_load_5d(&sm.v[c][e * 8192], &a.map_v, &sm.kv_full, c * 64, wp * g.pw, hp * g.ph,
                      t * g.pt, bh);
        }
      }
      int last_st = -1, last_do = -1, last_q = -1;
      for (int j = 0; j < nsteps; ++j) {
        const bool two = 2 * j + 1 < cnt;
        const int nq = two ? 2 : 1;
        int blk[2];
        blk[0] = ent[2 * j] & kEntryBlockMask;
        blk[1] = two ? (ent[2 * j + 1] & kEntryBlockMask) : blk[0];
        // statistics, once the row warps are done with the previous step's
        if (j > 0 && !mbar_wait(&sm.p_full, (j - 1) & 1, abort)) {
          fail_b(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        mbar_arrive_expect_tx(&sm.st_full, uint32_t(nq) * 2u * 256u);
        for (int x = 0; x < nq; ++x) {
          const size_t off = size_t(bh) * g.S + size_t(blk[x]) * 64;
          bulk_load(&sm.lse2[64 * x], a.lse2 + off, 256u, &sm.st_full);
          bulk_load(&sm.dsum[64 * x], a.dsum + off, 256u, &sm.st_full);
        }
        last_st = j;
        if (j > 0 && !mbar_wait(&sm.do_empty, (j - 1) & 1, abort)) {
          fail_b(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        mbar_arrive_expect_tx(&sm.do_full, uint32_t(nq) * 64u * D * 2u);
        for (int x = 0; x < nq; ++x) {
          int t, hp, wp;
          block_coords(g, blk[x], t, hp, wp);
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.dout[c][x * 8192], &a.map_do, &sm.do_full, c * 64, wp * g.pw,
                        hp * g.ph, t * g.pt, bh);
        }
        last_do = j;
        if (j > 0 && !mbar_wait(&sm.q_empty, (j - 1) & 1, abort)) {
          fail_b(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        mbar_arrive_expect_tx(&sm.q_full, uint32_t(nq) * 64u * D * 2u);
        for (int x = 0; x < nq; ++x) {
          int t, hp, wp;
          block_coords(g, blk[x], t, hp, wp);
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.q[c][x * 8192], &a.map_q, &sm.q_full, c * 64, wp * g.pw, hp * g.ph,
                        t * g.pt, bh);
        }
        last_q = j;
        if (*abort) break;
      }
      if (*abort) {
        // let this thread's copies land before the CTA can exit (time-bounded,
        // ignoring the abort flag)
        int never = 0;
        mbar_wait(&sm.kv_full, 0, &never);
        if (last_st >= 0) mbar_wait(&sm.st_full, last_st & 1, &never);
        if (last_do >= 0) mbar_wait(&sm.do_full, last_do & 1, &never);
        if (last_q >= 0) mbar_wait(&sm.q_full, last_q & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && nsteps > 0) {
      const uint32_t id_s2 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_acc = idesc_bf16_f32(128, D, 0, 1);  // A from TMEM, B MN-major
      const uint32_t id_dq = idesc_bf16_f32(128, D, 1, 1);   // A and B MN-major
      const uint64_t kd = sw128_desc(smem_u32(&sm.k[0][0]), 16, 1024);
      const uint64_t vd = sw128_desc(smem_u32(&sm.v[0][0]), 16, 1024);
      const uint64_t qd = sw128_desc(smem_u32(&sm.q[0][0]), 16, 1024);
      const uint64_t dod = sw128_desc(smem_u32(&sm.dout[0][0]), 16, 1024);
      const uint64_t q_mn = sw128_desc(smem_u32(&sm.q[0][0]), kBChunk, 1024);
      const uint64_t do_mn = sw128_desc(smem_u32(&sm.dout[0][0]), kBChunk, 1024);
      const uint64_t k_mn = sw128_desc(smem_u32(&sm.k[0][0]), kBChunk, 1024);
      const uint64_t ds_mn = sw128_desc(smem_u32(&sm.ds[0][0]), kBChunk, 1024);
      bool ok = mbar_wait(&sm.kv_full, 0, abort);
      for (int j = 0; ok && j < nsteps; ++j) {
        const bool two = 2 * j + 1 < cnt;
        ok = mbar_wait(&sm.q_full, j & 1, abort) && mbar_wait(&sm.do_full, j & 1, abort) &&
             (j == 0 || mbar_wait(&sm.tmem_free, (j - 1) & 1, abort));
        if (!ok) break;
        tc_fence_after_sync();
        const uint32_t ids = two ? id_s2 : id_s1;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t(kk >> 2) * kBChunk + uint32_t(kk & 3) * 32u) >> 4;
          mma_ss(tmem + kColS, kd + off, qd + off, ids, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t(kk >> 2) * kBChunk + uint32_t(kk & 3) * 32u) >> 4;
          mma_ss(tmem + kColDP, vd + off, dod + off, ids, kk > 0);
        }
        mma_commit(&sm.s_full);
        ok = mbar_wait(&sm.p_full, j & 1, abort);
        if (!ok) break;
        tc_fence_after_sync();
        // dV += P^T dO and dK += dS^T Q over the step's query rows (K = 128
        // or 64); each commit frees the tile it was the last reader of
        if (two)
          mma_ts_k<8>(tmem + kColDV, tmem + kColS, do_mn, id_acc, j > 0 ? 1u : 0u);
        else
          mma_ts_k<4>(tmem + kColDV, tmem + kColS, do_mn, id_acc, j > 0 ? 1u : 0u);
        mma_commit(&sm.do_empty);
        if (two)
          mma_ts_k<8>(tmem + kColDK, tmem + kColDP, q_mn, id_acc, j > 0 ? 1u : 0u);
        else
          mma_ts_k<4>(tmem + kColDK, tmem + kColDP, q_mn, id_acc, j > 0 ? 1u : 0u);
        mma_commit(&sm.q_empty);
        // dQ = dS K: the 128 query rows as M, the 128 keys as K
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + kColS, ds_mn + uint64_t(kk) * 128u, k_mn + uint64_t(kk) * 128u, id_dq,
                 kk > 0);
        mma_commit(&sm.dq_full);
      }
      if (ok) {
        mma_commit(&sm.acc_full);
      } else {
        fail_b(a.status, &sm.abort, kDevErrTimeoutMma);
        mma_commit(&sm.drain);  // wait (bounded) for this thread's MMAs before exit
        int never = 0;
        mbar_wait(&sm.drain, 0, &never);
      }
    }
  } else {
    // ---------------------------------------------------------------- rows
    const int quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane: a key in S^T, dP^T, dK, dV; a query row in dQ
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const int my_keep = r < 64 ? kEntryKeepA : kEntryKeepB;  // uniform across the warp
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int j = 0; j < nsteps; ++j) {
      const bool two = 2 * j + 1 < cnt;
      const int f0 = ent[2 * j], f1 = two ? ent[2 * j + 1] : 0;
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full, j & 1, abort) &&
                                       mbar_wait(&sm.st_full, j & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      // P^T = 2^(s log2(e)/sqrt(d) - lse2) on kept (k-block, q-block) pairs,
      // dS^T = P^T * (dP^T - D); 32 query columns per chunk
      for (int c = 0; c < (two ? 4 : 2); ++c) {
        const bool keep = (((c < 2) ? f0 : f1) & my_keep) != 0;
        uint32_t pk[16], dk[16];
        if (keep) {
          uint32_t sv[32], dp[32];
          tmem_ld32(lane_base + kColS + 32u * c, sv);
          tmem_ld32(lane_base + kColDP + 32u * c, dp);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int col = 32 * c + 2 * i;
            const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * i]), sl2, -sm.lse2[col]));
            const float p1 =
                ex2_approx(fmaf(__uint_as_float(sv[2 * i + 1]), sl2, -sm.lse2[col + 1]));
            const float d0 = p0 * (__uint_as_float(dp[2 * i]) - sm.dsum[col]);
            const float d1 = p1 * (__uint_as_float(dp[2 * i + 1]) - sm.dsum[col + 1]);
            pk[i] = pack_bf16x2(p0, p1);
            dk[i] = pack_bf16x2(d0, d1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = dk[i] = 0u;
        }
        tmem_st16(lane_base + kColS + 16u * c, pk);
        tmem_st16(lane_base + kColDP + 16u * c, dk);
        // this key's row of dS in the 128-byte-swizzled MN-major layout:
        // 16-byte unit u of the row sits at unit u ^ (r & 7)
        uint8_t* row = &sm.ds[c >> 1][r * 128];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const int u = ((c & 1) << 2) + w;
          *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) << 4)) =
              make_uint4(dk[4 * w], dk[4 * w + 1], dk[4 * w + 2], dk[4 * w + 3]);
        }
      }
      if (!two) {
        // dQ's MMA reads all 128 query rows of dS: zero the absent q-block's
        uint8_t* row = &sm.ds[1][r * 128];
#pragma unroll
        for (int u = 0; u < 8; ++u) *reinterpret_cast<uint4*>(row + (u << 4)) = make_uint4(0, 0, 0, 0);
      }
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&sm.p_full);
      // dQ rows (one query row per lane) -> the fp32 accumulator
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.dq_full, j & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      const int h = r >> 6;  // uniform across the warp
      if (h == 0 || two) {
        const int blk = (h ? f1 : f0) & kEntryBlockMask;
        float* dst = a.dq_acc + (size_t(bh) * g.S + block_row_token(g, blk, r & 63)) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColS + 32u * c, o);
          tmem_wait_ld();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            red_add_f32x4(dst + 32 * c + 4 * v, __uint_as_float(o[4 * v]) * a.scale,
                          __uint_as_float(o[4 * v + 1]) * a.scale,
                          __uint_as_float(o[4 * v + 2]) * a.scale,
                          __uint_as_float(o[4 * v + 3]) * a.scale);
        }
      }
      tc_fence_before_sync();
      mbar_arrive(&sm.tmem_free);
    }
    if (!ok) {
      fail_b(a.status, &sm.abort, kDevErrTimeoutSoftmax);
    } else if (r < 64 || kb >= 0) {  // uniform across the warp
      // dK (scaled) and dV rows of this key to its natural position
      const bool acc = nsteps == 0 || __all_sync(0xFFFFFFFFu, mbar_wait(&sm.acc_full, 0, abort));
      if (!acc) {
        fail_b(a.status, &sm.abort, kDevErrTimeoutSoftmax);
      } else {
        if (nsteps > 0) tc_fence_after_sync();
        const size_t row = size_t(bh) * g.S + block_row_token(g, r < 64 ? ka : kb, r & 63);
        for (int which = 0; which < 2; ++which) {
          const float mul = which ? a.scale : 1.0f;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            float x[32];
            if (nsteps > 0) {
              uint32_t o[32];
              tmem_ld32(lane_base + (which ? kColDK : kColDV) + 32u * c, o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(o[i]) * mul;
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = 0.f;
            }
            store_row32<D>(which ? a.dk : a.dv, row, 32 * c, x, a.out_fp32);
          }
        }
      }
    }
  }
  tc_fence_before_sync();
  __syncthreads();
  tc_fence_after_sync();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

template <int D>
static cudaError_t launch_bwd_d(const BwdArgs& a, const Geometry& g, cudaStream_t stream) {
  const int smem = int(sizeof(BwdSmem<D>) + 1024);
  cudaError_t e = cudaFuncSetAttribute(bwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       smem);
  if (e != cudaSuccess) return e;
  bwd_kernel<D><<<dim3(unsigned(g.ntile), unsigned(g.BH)), kBThreads, smem, stream>>>(a, g);
  return cudaGetLastError();
}

cudaError_t launch_bwd(const BwdArgs& a, const Geometry& g, cudaStream_t stream) {
  return g.d == 128 ? launch_bwd_d<128>(a, g, stream) : launch_bwd_d<64>(a, g, stream);
}

}  // namespace sa
