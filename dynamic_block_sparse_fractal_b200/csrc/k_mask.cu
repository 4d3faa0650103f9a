// Mask build (NABLA, Metodologia 2 "Attenzione Ridotta" + "CDF Thresholding",
// Metodologia 3 STA union). One CTA handles 16 q-block rows (8 query tiles)
// of one head, one warp per row:
//
//  1. logits L[r][j] = Qbar[r] . Kbar[j] / sqrt(d) in fp32 FFMA, Kbar streamed
//     through shared memory in chunks of 64 blocks;
//  2. row softmax (max, exp, one deterministic warp sum);
//  3. CDF threshold without sorting: k-block j is kept iff the probability
//     mass ranked before it is < 1 - thr. With masses in 2^-40 fixed point
//     (integer sums, so the result is bit-identical run to run), a 4-pass
//     8-bit radix select over the probabilities' bit patterns finds the
//     probability tau of the last kept block and the mass strictly above it;
//     blocks equal to tau are kept in ascending index order while the running
//     mass stays below the threshold (ties broken by index, as the sorted
//     definition does);
//  4. OR with the static STA window, compaction into the ascending kept list
//     and a keep bitmap per row;
//  5. per query tile (two rows), the union of the two bitmaps as a list of
//     k-blocks tagged with which q-block keeps each, temporal pairs first.
#include <cuda_runtime.h>

#include "kernels.cuh"
#include "sm100.cuh"

namespace sa {

constexpr int kMaskRows = 16;
constexpr int kMaskThreads = kMaskRows * 32;
constexpr int kKChunk = 64;
constexpr unsigned kFull = 0xFFFFFFFFu;

__device__ __forceinline__ unsigned long long mass_fx(float p) {
  return __float2ull_rn(p * 1099511627776.0f);  // p * 2^40, exact scaling
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__host__ __device__ constexpr size_t mask_region2_bytes(int D) {
  return (size_t(kKChunk) * (D + 4) * 4 > size_t(kMaskRows) * 256 * 8)
             ? size_t(kKChunk) * (D + 4) * 4
             : size_t(kMaskRows) * 256 * 8;
}

size_t mask_smem_bytes(const Geometry& g) {
  const size_t nwords = (g.nb + 31) / 32;
  return size_t(kMaskRows) * g.d * 4 + mask_region2_bytes(g.d) + size_t(kMaskRows) * g.nb * 4 +
         size_t(kMaskRows) * nwords * 4;
}

template <int D>
__global__ void __launch_bounds__(kMaskThreads, 1) mask_kernel(MaskArgs a, Geometry g) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int KP = D + 4;  // padded K-chunk row (conflict-free float4 reads)
  const int nb = g.nb;
  const int nwords = (nb + 31) / 32;
  float* qs = reinterpret_cast<float*>(smem);                      // [16][D]
  uint8_t* region2 = smem + size_t(kMaskRows) * D * 4;              // K chunk / histograms
  float* ks = reinterpret_cast<float*>(region2);                    // [64][KP]
  float* L = reinterpret_cast<float*>(region2 + mask_region2_bytes(D));  // [16][nb]
  uint32_t* bits = reinterpret_cast<uint32_t*>(L + size_t(kMaskRows) * nb);  // [16][nwords]
  __shared__ int row_blk[kMaskRows];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int tile0 = blockIdx.x * (kMaskRows / 2);

  if (threadIdx.x < kMaskRows) {
    const int tile = tile0 + threadIdx.x / 2;
    int blk = -1;
    if (tile < g.ntile) {
      int qa, qb;
      tile_blocks(g, tile, qa, qb);
      blk = (threadIdx.x & 1) ? qb : qa;
    }
    row_blk[threadIdx.x] = blk;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kMaskRows * D / 4; i += kMaskThreads) {
    const int r = i / (D / 4), c = i - r * (D / 4);
    const int blk = row_blk[r];
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (blk >= 0) v = reinterpret_cast<const float4*>(a.qbar + (size_t(bh) * nb + blk) * D)[c];
    reinterpret_cast<float4*>(qs)[i] = v;
  }

  // ---- 1. logits
  const int r = warp;
  const float* kbase = a.kbar + size_t(bh) * nb * D;
  for (int c0 = 0; c0 < nb; c0 += kKChunk) {
    __syncthreads();
    for (int i = threadIdx.x; i < kKChunk * D / 4; i += kMaskThreads) {
      const int row = i / (D / 4), c = i - row * (D / 4);
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (c0 + row < nb) v = reinterpret_cast<const float4*>(kbase + size_t(c0 + row) * D)[c];
      *reinterpret_cast<float4*>(ks + row * KP + 4 * c) = v;
    }
    __syncthreads();
    const float* qr = qs + r * D;
    const float* k0 = ks + lane * KP;
    const float* k1 = ks + (lane + 32) * KP;
    float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
    for (int dd = 0; dd < D; dd += 4) {
      const float4 qv = *reinterpret_cast<const float4*>(qr + dd);
      const float4 x0 = *reinterpret_cast<const float4*>(k0 + dd);
      const float4 x1 = *reinterpret_cast<const float4*>(k1 + dd);
      acc0 = fmaf(qv.x, x0.x, acc0);
      acc0 = fmaf(qv.y, x0.y, acc0);
      acc0 = fmaf(qv.z, x0.z, acc0);
      acc0 = fmaf(qv.w, x0.w, acc0);
      acc1 = fmaf(qv.x, x1.x, acc1);
      acc1 = fmaf(qv.y, x1.y, acc1);
      acc1 = fmaf(qv.z, x1.z, acc1);
      acc1 = fmaf(qv.w, x1.w, acc1);
    }
    if (c0 + lane < nb) L[size_t(r) * nb + c0 + lane] = acc0 * a.scale;
    if (c0 + lane + 32 < nb) L[size_t(r) * nb + c0 + lane + 32] = acc1 * a.scale;
  }
  __syncthreads();  // region2 is free from here on: histograms

  const int blk = row_blk[r];
  uint32_t* my_bits = bits + size_t(r) * nwords;
  if (blk >= 0) {
    float* Lr = L + size_t(r) * nb;
    // ---- 2. softmax
    float mx = -INFINITY;
    for (int j = lane; j < nb; j += 32) mx = fmaxf(mx, Lr[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, o));
    float sum = 0.f;
    for (int j = lane; j < nb; j += 32) {
      const float e = expf(Lr[j] - mx);
      Lr[j] = e;
      sum += e;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(kFull, sum, o);
    const float inv = 1.0f / sum;
    for (int j = lane; j < nb; j += 32) Lr[j] *= inv;
    __syncwarp();

    // ---- 3. CDF threshold by radix select
    bool keep_all = a.dense != 0;
    unsigned tau = 0;
    unsigned long long keep_ties = 0;
    if (!keep_all) {
      const unsigned long long tgt = a.target_fx;
      unsigned long long* hist = reinterpret_cast<unsigned long long*>(region2) + warp * 256;
      unsigned prefix = 0, pmask = 0;
      unsigned long long above = 0;
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) hist[i] = 0ull;
        __syncwarp();
        for (int j = lane; j < nb; j += 32) {
          const float p = Lr[j];
          const unsigned key = __float_as_uint(p);
          if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], mass_fx(p));
        }
        __syncwarp();
        // lane l owns bins 255-8l down to 248-8l
        unsigned long long h[8], s = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          h[i] = hist[255 - 8 * lane - i];
          s += h[i];
        }
        unsigned long long inc = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const unsigned long long v = __shfl_up_sync(kFull, inc, o);
          if (lane >= o) inc += v;
        }
        const unsigned long long pre = above + (inc - s);
        const bool cross = pre < tgt && tgt <= pre + s;
        const unsigned bal = __ballot_sync(kFull, cross);
        if (bal == 0u) {  // total mass below the target (rounding): keep all
          keep_all = true;
          break;
        }
        const int src = __ffs(bal) - 1;
        int digit = 0;
        unsigned long long above_new = 0;
        if (lane == src) {
          unsigned long long run = pre;
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            if (run + h[i] >= tgt) {
              digit = 255 - 8 * lane - i;
              above_new = run;
              break;
            }
            run += h[i];
          }
        }
        digit = __shfl_sync(kFull, digit, src);
        above_new = __shfl_sync(kFull, above_new, src);
        prefix |= unsigned(digit) << shift;
        pmask |= 255u << shift;
        above = above_new;
        __syncwarp();
      }
      if (!keep_all) {
        tau = prefix;
        const unsigned long long mt = mass_fx(__uint_as_float(tau));  // > 0
        keep_ties = (tgt - above + mt - 1) / mt;
      }
    }

    // ---- 4. STA union + compaction
    int tq, hq, wq;
    block_coords(g, blk, tq, hq, wq);
    int32_t* out_idx = a.idx + (size_t(bh) * nb + blk) * nb;
    int pos = 0;
    unsigned long long ties = 0;
    for (int base = 0; base < nb; base += 32) {
      const int j = base + lane;
      const bool valid = j < nb;
      bool nab = false, tie = false;
      if (valid) {
        if (keep_all) {
          nab = true;
        } else {
          const unsigned key = __float_as_uint(Lr[j]);
          nab = key > tau;
          tie = key == tau;
        }
      }
      const unsigned tb = __ballot_sync(kFull, tie);
      if (tie) nab = (ties + __popc(tb & lanemask_lt())) < keep_ties;
      ties += __popc(tb);
      bool in_sta = false;
      if (valid && a.sta_t >= 0) {
        int tk, hk, wk;
        block_coords(g, j, tk, hk, wk);
        in_sta = abs(tk - tq) <= a.sta_t && abs(hk - hq) <= a.sta_h && abs(wk - wq) <= a.sta_w;
      }
      const bool kept = valid && (nab || in_sta);
      const unsigned kb = __ballot_sync(kFull, kept);
      if (kept) out_idx[pos + __popc(kb & lanemask_lt())] = j;
      pos += __popc(kb);
      if (lane == 0) my_bits[base >> 5] = kb;
    }
    if (lane == 0) a.cnt[size_t(bh) * nb + blk] = pos;
  } else {
    for (int i = lane; i < nwords; i += 32) my_bits[i] = 0u;
  }
  __syncthreads();

  // ---- 5. per-tile union lists, ordered for the attention kernel: first the
  // steps that pair the same patch in frames t and t+1 (one two-frame TMA box
  // each), then the remaining blocks in ascending order. The probability
  // buffer L is free now and holds the pairing bitmaps.
  if (warp < kMaskRows / 2) {
    const int tile = tile0 + warp;
    if (tile < g.ntile) {
      const uint32_t* ba = bits + size_t(2 * warp) * nwords;
      const uint32_t* bb = bits + size_t(2 * warp + 1) * nwords;
      uint32_t* u = reinterpret_cast<uint32_t*>(L) + size_t(warp) * 3 * nwords;
      uint32_t* first = u + nwords;
      uint32_t* second = first + nwords;
      for (int w = lane; w < nwords; w += 32) {
        u[w] = ba[w] | bb[w];
        first[w] = 0u;
        second[w] = 0u;
      }
      __syncwarp();
      // greedy along time, one patch per lane
      const int pf = g.nh * g.nw;
      for (int p = lane; p < pf; p += 32) {
        bool pending = false;
        for (int t = 0; t < g.T; ++t) {
          const int b = t * pf + p;
          const bool in = (u[b >> 5] >> (b & 31)) & 1u;
          if (pending && in) {
            const int f = b - pf;
            atomicOr(&first[f >> 5], 1u << (f & 31));
            atomicOr(&second[b >> 5], 1u << (b & 31));
            pending = false;
          } else {
            pending = in;
          }
        }
      }
      __syncwarp();
      int32_t* out = a.tidx + (size_t(bh) * g.ntile + tile) * nb;
      auto flags = [&](int b) {
        return int(((ba[b >> 5] >> (b & 31)) & 1u) << 16) | int(((bb[b >> 5] >> (b & 31)) & 1u) << 17);
      };
      int pos = 0;
      for (int w = 0; w < nwords; ++w) {
        const uint32_t x = first[w];
        if ((x >> lane) & 1u) {
          const int b = w * 32 + lane;
          const int o = pos + 2 * __popc(x & lanemask_lt());
          out[o] = b | flags(b) | kEntryTPair;
          out[o + 1] = (b + pf) | flags(b + pf);
        }
        pos += 2 * __popc(x);
      }
      for (int w = 0; w < nwords; ++w) {
        const uint32_t x = u[w] & ~first[w] & ~second[w];
        if ((x >> lane) & 1u) {
          const int b = w * 32 + lane;
          out[pos + __popc(x & lanemask_lt())] = b | flags(b);
        }
        pos += __popc(x);
      }
      if (lane == 0) a.tcnt[size_t(bh) * g.ntile + tile] = pos;
    }
  }
}

cudaError_t launch_mask(const MaskArgs& a, const Geometry& g, cudaStream_t stream) {
  const size_t smem = mask_smem_bytes(g);
  const dim3 grid(unsigned((g.ntile + kMaskRows / 2 - 1) / (kMaskRows / 2)), unsigned(g.BH));
  cudaError_t e;
  if (g.d == 128) {
    e = cudaFuncSetAttribute(mask_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    mask_kernel<128><<<grid, kMaskThreads, smem, stream>>>(a, g);
  } else {
    e = cudaFuncSetAttribute(mask_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             int(smem));
    if (e != cudaSuccess) return e;
    mask_kernel<64><<<grid, kMaskThreads, smem, stream>>>(a, g);
  }
  return cudaGetLastError();
}

// One CTA per head: bitonic sort of the head's tiles by descending union
// length, so that the attention grid meets the heaviest tiles of a head first
// (longest-processing-time order) while concurrently running CTAs still share
// one head's K/V in L2.
__global__ void __launch_bounds__(1024) tile_order_kernel(const int32_t* __restrict__ tcnt,
                                                          int32_t* __restrict__ order, Geometry g) {
  __shared__ uint32_t key[2048];
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
          const uint32_t a = key[i], b = key[partner];
          if ((a > b) == up) {
            key[i] = b;
            key[partner] = a;
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
