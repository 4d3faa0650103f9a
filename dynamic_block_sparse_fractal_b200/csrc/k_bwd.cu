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

constexpr int kBThreads = 320;        // warp 0 TMA, warp 1 MMA, warps 2-9 rows
constexpr int kBChunk = 128 * 128;    // 128 rows x 128 B (64 bf16 channels)
// TMEM columns: dV and dK accumulators (fp32, one key per lane); S^T, then P;
// dP^T, then dS, then dQ (fp32, one query row per lane). Each row warpgroup
// owns 64 columns of S^T and of dP^T (its q-block) and packs its P / dS
// (bf16 pairs) into the first 32 of them, so the two never write columns the
// other still reads; the MMAs read P and dS as two K = 64 halves.
constexpr uint32_t kColDV = 0, kColDK = 128, kColS = 256, kColDP = 384;
// List entries staged in shared memory per key tile; longer lists (heads of
// more than 2880 blocks) read the rest from global memory (L2).
constexpr int kBMaxEntries = 2880;

template <int D>
struct __align__(1024) BwdSmem {
  uint8_t k[D / 64][kBChunk];     // key tile: two k-blocks, 64 keys each
  uint8_t v[D / 64][kBChunk];
  uint8_t q[2][D / 64][kBChunk];  // the step's query rows (two q-blocks), two slots
  uint8_t dout[D / 64][kBChunk];
  uint8_t ds[2][kBChunk];         // dS as the MN-major A of dQ = dS K: [64-query chunk][key][64 q]
  float lse2[2][128], dsum[2][128];  // per query row of the step, two slots
  int32_t ent[kBMaxEntries];      // the key tile's list (q-block | keep bits)
  uint64_t kv_full, q_full[2], q_empty[2], do_full, do_empty, st_full[2], st_empty[2];
  uint64_t s_full, dp_full, p_full, ds_full, dq_full, tmem_free, acc_full, drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void fail_b(uint32_t* status, int* abort, uint32_t bit) {
  atomicOr(status, bit);
  *reinterpret_cast<volatile int*>(abort) = 1;
}

// 32 fp32 values -> columns [col0, col0 + 32) of row `row` of a [.][D]
// output, bf16 or fp32.
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

// 64 packed bf16 pairs of this thread's key row: TMEM columns and the
// 128-byte-swizzled dS row in shared memory (unit u of the row at u ^ (r & 7)).
__device__ __forceinline__ void store_ds_row(uint8_t* row, int r, const uint32_t (&x)[32]) {
#pragma unroll
  for (int u = 0; u < 8; ++u)
    *reinterpret_cast<uint4*>(row + ((u ^ (r & 7)) << 4)) =
        make_uint4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
}

}  // namespace

// One CTA per (key tile, bh): the key tile's K and V stay in shared memory;
// each step takes the next two q-blocks of its list. Per step:
//   S^T = K Q^T        (keys as M)             -> row warps: P^T
//   dP^T = V dO^T                               -> row warps: dS^T = P^T (dP^T - D)
//   dV += P^T dO, dK += dS^T Q (A from TMEM), dQ = dS K (dS from shared
//   memory), whose rows the row warps add to the fp32 accumulator.
// The two row warpgroups take one q-block each (and half of dQ's columns);
// the next step's S^T is issued right after this step's dQ, so it overlaps
// the dQ read-out.
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
  const int nsteps = (cnt + 1) / 2;
  // the key tile's list, read once (every role walks it step by step)
  const int32_t* gent = a.kidx + unit * g.nb;
  for (int i = threadIdx.x; i < cnt && i < kBMaxEntries; i += kBThreads) sm.ent[i] = gent[i];
  auto ent_at = [&](int i) -> int {
    return i < kBMaxEntries ? sm.ent[i] : __ldg(gent + i);
  };
  if (threadIdx.x == 0) {
    sm.abort = 0;
    mbar_init(&sm.kv_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.st_full[s], 1);
      mbar_init(&sm.st_empty[s], 256);
    }
    mbar_init(&sm.do_full, 1);
    mbar_init(&sm.do_empty, 1);
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.dp_full, 1);
    mbar_init(&sm.p_full, 256);
    mbar_init(&sm.ds_full, 256);
    mbar_init(&sm.dq_full, 1);
    mbar_init(&sm.tmem_free, 256);
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
      int last_q = -1, last_do = -1, last_st = -1;
      for (int j = 0; j < nsteps; ++j) {
        const int slot = j & 1;
        const bool two = 2 * j + 1 < cnt;
        const int nq = two ? 2 : 1;
        int blk[2];
        blk[0] = ent_at(2 * j) & kEntryBlockMask;
        blk[1] = two ? (ent_at(2 * j + 1) & kEntryBlockMask) : blk[0];
        // Q (two slots: loaded a step ahead)
        if (j >= 2 && !mbar_wait(&sm.q_empty[slot], ((j >> 1) - 1) & 1, abort)) {
          fail_b(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        const bool stall = j == 0 && (a.debug_flags & SA_DEBUG_STALL_LOADER);  // test hook
        if (!stall) mbar_arrive_expect_tx(&sm.q_full[slot], uint32_t(nq) * 64u * D * 2u);
        for (int x = 0; x < nq && !stall; ++x) {
          int t, hp, wp;
          block_coords(g, blk[x], t, hp, wp);
          for (int c = 0; c < D / 64; ++c)
            tma_load_5d(&sm.q[slot][c][x * 8192], &a.map_q, &sm.q_full[slot], c * 64, wp * g.pw,
                        hp * g.ph, t * g.pt, bh);
        }
        if (!stall) last_q = j;
        // dO (one slot: free once dV's MMA of the previous step is done)
        if (j >= 1 && !mbar_wait(&sm.do_empty, (j - 1) & 1, abort)) {
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
        // row statistics (two slots)
        if (j >= 2 && !mbar_wait(&sm.st_empty[slot], ((j >> 1) - 1) & 1, abort)) {
          fail_b(a.status, &sm.abort, kDevErrTimeoutLoad);
          break;
        }
        mbar_arrive_expect_tx(&sm.st_full[slot], uint32_t(nq) * 2u * 256u);
        for (int x = 0; x < nq; ++x) {
          const size_t off = size_t(bh) * g.S + size_t(blk[x]) * 64;
          bulk_load(&sm.lse2[slot][64 * x], a.lse2 + off, 256u, &sm.st_full[slot]);
          bulk_load(&sm.dsum[slot][64 * x], a.dsum + off, 256u, &sm.st_full[slot]);
        }
        last_st = j;
        if (*abort) break;
      }
      if (*abort) {
        // let this thread's copies land before the CTA can exit (time-bounded,
        // ignoring the abort flag); at most the last use of each slot is open
        int never = 0;
        mbar_wait(&sm.kv_full, 0, &never);
        for (int jj = last_q; jj >= 0 && jj > last_q - 2; --jj)
          mbar_wait(&sm.q_full[jj & 1], (jj >> 1) & 1, &never);
        if (last_do >= 0) mbar_wait(&sm.do_full, last_do & 1, &never);
        for (int jj = last_st; jj >= 0 && jj > last_st - 2; --jj)
          mbar_wait(&sm.st_full[jj & 1], (jj >> 1) & 1, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA
    if (lane == 0 && nsteps > 0) {
      const uint32_t id_s2 = idesc_bf16_f32(128, 128, 0, 0);
      const uint32_t id_s1 = idesc_bf16_f32(128, 64, 0, 0);
      const uint32_t id_acc = idesc_bf16_f32(128, D, 0, 1);  // A from TMEM, B MN-major
      const uint32_t id_dq = idesc_bf16_f32(128, D, 1, 1);   // A and B MN-major
      constexpr uint32_t kSlot = (D / 64) * kBChunk / 16;    // a Q slot, descriptor units
      constexpr uint64_t kHalfRows = 64 * 128 / 16;          // 64 rows of an MN-major tile
      const uint64_t kd = sw128_desc(smem_u32(&sm.k[0][0]), 16, 1024);
      const uint64_t vd = sw128_desc(smem_u32(&sm.v[0][0]), 16, 1024);
      const uint64_t qd0 = sw128_desc(smem_u32(&sm.q[0][0][0]), 16, 1024);
      const uint64_t dod = sw128_desc(smem_u32(&sm.dout[0][0]), 16, 1024);
      const uint64_t q_mn0 = sw128_desc(smem_u32(&sm.q[0][0][0]), kBChunk, 1024);
      const uint64_t do_mn = sw128_desc(smem_u32(&sm.dout[0][0]), kBChunk, 1024);
      const uint64_t k_mn = sw128_desc(smem_u32(&sm.k[0][0]), kBChunk, 1024);
      const uint64_t ds_mn = sw128_desc(smem_u32(&sm.ds[0][0]), kBChunk, 1024);
      bool ok = mbar_wait(&sm.kv_full, 0, abort);
      for (int j = 0; ok && j < nsteps; ++j) {
        const int slot = j & 1;
        const bool two = 2 * j + 1 < cnt;
        const uint32_t ids = two ? id_s2 : id_s1;
        const uint64_t qd = qd0 + uint64_t(slot) * kSlot;
        // S^T = K Q^T
        ok = mbar_wait(&sm.q_full[slot], (j >> 1) & 1, abort);
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t(kk >> 2) * kBChunk + uint32_t(kk & 3) * 32u) >> 4;
          mma_ss(tmem + kColS, kd + off, qd + off, ids, kk > 0);
        }
        mma_commit(&sm.s_full);
        // dP^T = V dO^T, once the previous step's dQ has left TMEM
        ok = mbar_wait(&sm.do_full, j & 1, abort) &&
             (j == 0 || mbar_wait(&sm.tmem_free, (j - 1) & 1, abort));
        if (!ok) break;
        tc_fence_after_sync();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (uint32_t(kk >> 2) * kBChunk + uint32_t(kk & 3) * 32u) >> 4;
          mma_ss(tmem + kColDP, vd + off, dod + off, ids, kk > 0);
        }
        mma_commit(&sm.dp_full);
        // dV += P^T dO over the step's query rows (K = 128 or 64)
        ok = mbar_wait(&sm.p_full, j & 1, abort);
        if (!ok) break;
        tc_fence_after_sync();
        // (the second q-block's P sits 64 columns on; its dO rows 64 rows on)
        mma_ts_k<4>(tmem + kColDV, tmem + kColS, do_mn, id_acc, j > 0 ? 1u : 0u);
        if (two) mma_ts_k<4>(tmem + kColDV, tmem + kColS + 64u, do_mn + kHalfRows, id_acc, 1u);
        mma_commit(&sm.do_empty);
        // dK += dS^T Q, then dQ = dS K over the dS columns (read just before)
        ok = mbar_wait(&sm.ds_full, j & 1, abort);
        if (!ok) break;
        tc_fence_after_sync();
        const uint64_t q_mn = q_mn0 + uint64_t(slot) * kSlot;
        mma_ts_k<4>(tmem + kColDK, tmem + kColDP, q_mn, id_acc, j > 0 ? 1u : 0u);
        if (two) mma_ts_k<4>(tmem + kColDK, tmem + kColDP + 64u, q_mn + kHalfRows, id_acc, 1u);
        mma_commit(&sm.q_empty[slot]);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + kColDP, ds_mn + uint64_t(kk) * 128u, k_mn + uint64_t(kk) * 128u, id_dq,
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
    // warpgroup wg takes query columns [64 wg, 64 wg + 64) of S^T / dP^T (its
    // q-block of the step) and dQ / dK / dV columns [D/2 wg, D/2 (wg + 1))
    constexpr int DH = D / 2;
    const int wg = (warp - 2) >> 2, quad = warp & 3;
    const int r = quad * 32 + lane;  // TMEM lane: a key in S^T, dP^T, dK, dV; a query row in dQ
    const uint32_t lane_base = tmem + (uint32_t(quad * 32) << 16);
    const int my_keep = r < 64 ? kEntryKeepA : kEntryKeepB;  // uniform across the warp
    const float sl2 = a.scale_log2;
    bool ok = true;
    for (int j = 0; j < nsteps; ++j) {
      const int slot = j & 1;
      const bool two = 2 * j + 1 < cnt;
      const int f0 = ent_at(2 * j), f1 = two ? ent_at(2 * j + 1) : 0;
      const bool mine = wg == 0 || two;                       // this half has a q-block
      const bool keep = mine && (((wg ? f1 : f0) & my_keep) != 0);  // uniform across the warp
      const float* lse2 = &sm.lse2[slot][64 * wg];
      const float* dsum = &sm.dsum[slot][64 * wg];
      // ---- P^T = 2^(s log2(e)/sqrt(d) - lse2) on a kept (k-block, q-block) pair
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.s_full, j & 1, abort) &&
                                       mbar_wait(&sm.st_full[slot], (j >> 1) & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      float p[64];
      uint32_t pk[32];
      const uint32_t s_col = lane_base + kColS + 64u * wg;    // this half's S^T, then P
      const uint32_t dp_col = lane_base + kColDP + 64u * wg;  // this half's dP^T, then dS
      if (keep) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t sv[32];
          tmem_ld32(s_col + 32u * c, sv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i)
            p[32 * c + i] = ex2_approx(fmaf(__uint_as_float(sv[i]), sl2, -lse2[32 * c + i]));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = pack_bf16x2(p[2 * i], p[2 * i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
      }
      if (mine) tmem_st32(s_col, pk);
      tmem_wait_st();
      tc_fence_before_sync();
      // relaxed: the stores above are complete, and the previous step's dQ
      // reductions need not be
      mbar_arrive_relaxed(&sm.p_full);
      // ---- dS^T = P^T (dP^T - D)
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.dp_full, j & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      if (keep) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t dp[32];
          tmem_ld32(dp_col + 32u * c, dp);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int k2 = 32 * c + 2 * i;
            pk[16 * c + i] = pack_bf16x2(p[k2] * (__uint_as_float(dp[2 * i]) - dsum[k2]),
                                         p[k2 + 1] * (__uint_as_float(dp[2 * i + 1]) - dsum[k2 + 1]));
          }
        }
      }  // otherwise pk is still all zero
      if (mine) tmem_st32(dp_col, pk);
      // dQ's MMA reads all 128 query rows of dS: an absent q-block's are zero
      store_ds_row(&sm.ds[wg][r * 128], r, pk);
      fence_proxy_async_smem();
      tmem_wait_st();
      tc_fence_before_sync();
      mbar_arrive(&sm.ds_full);
      mbar_arrive(&sm.st_empty[slot]);
      // ---- dQ rows (one query row per lane, this half's columns) -> the fp32
      // accumulator by vector reductions. Each warp turns its 32 rows x 32
      // columns around in a 4 KB staging tile (in the dS buffer, free from
      // dQ's MMA until the next step's dP^T, which waits for every thread's
      // TMEM release below), so that one reduction instruction covers four
      // whole 128-byte row segments: full-sector L2 operations. TMEM is
      // released with a relaxed arrive once read (tcgen05.wait::ld), so the
      // reductions in flight do not hold the next step's MMAs back.
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&sm.dq_full, j & 1, abort));
      if (!ok) break;
      tc_fence_after_sync();
      const int h = r >> 6;  // uniform across the warp
      if (h == 0 || two) {
        const int blk = (h ? f1 : f0) & kEntryBlockMask;
        const unsigned long long dst = reinterpret_cast<unsigned long long>(
            a.dq_acc + (size_t(bh) * g.S + block_row_token(g, blk, r & 63)) * D + DH * wg);
        uint8_t* stage = &sm.ds[0][0] + (warp - 2) * 4096;
        for (int c = 0; c < DH / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColDP + uint32_t(DH * wg + 32 * c), o);
          tmem_wait_ld();
          // this lane's row segment, 16-byte units swizzled by row
#pragma unroll
          for (int u = 0; u < 8; ++u)
            *reinterpret_cast<float4*>(stage + lane * 128 + ((u ^ (lane & 7)) << 4)) =
                make_float4(__uint_as_float(o[4 * u]) * a.scale,
                            __uint_as_float(o[4 * u + 1]) * a.scale,
                            __uint_as_float(o[4 * u + 2]) * a.scale,
                            __uint_as_float(o[4 * u + 3]) * a.scale);
          __syncwarp();
          // 8 lanes per row segment, 4 rows per instruction
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int row = 4 * i + (lane >> 3), u = lane & 7;
            const float4 x =
                *reinterpret_cast<const float4*>(stage + row * 128 + ((u ^ (row & 7)) << 4));
            float* p = reinterpret_cast<float*>(__shfl_sync(0xFFFFFFFFu, dst, row));
            red_add_f32x4(p + 32 * c + 4 * u, x.x, x.y, x.z, x.w);
          }
          __syncwarp();  // the tile is reused by the next segment
        }
      }
      tc_fence_before_sync();
      mbar_arrive_relaxed(&sm.tmem_free);
    }
    if (!ok) {
      fail_b(a.status, &sm.abort, kDevErrTimeoutSoftmax);
    } else if (r < 64 || kb >= 0) {  // uniform across the warp
      // dK (scaled) and dV of this key, this half's columns, to its natural position
      const bool acc = nsteps == 0 || __all_sync(0xFFFFFFFFu, mbar_wait(&sm.acc_full, 0, abort));
      if (!acc) {
        fail_b(a.status, &sm.abort, kDevErrTimeoutSoftmax);
      } else {
        if (nsteps > 0) tc_fence_after_sync();
        const size_t row = size_t(bh) * g.S + block_row_token(g, r < 64 ? ka : kb, r & 63);
        for (int which = 0; which < 2; ++which) {
          const float mul = which ? a.scale : 1.0f;
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            const int col = DH * wg + 32 * c;
            float x[32];
            if (nsteps > 0) {
              uint32_t o[32];
              tmem_ld32(lane_base + (which ? kColDK : kColDV) + uint32_t(col), o);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = __uint_as_float(o[i]) * mul;
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) x[i] = 0.f;
            }
            store_row32<D>(which ? a.dk : a.dv, row, col, x, a.out_fp32);
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
