// Block pooling of Q and K ("Sottocampionamento", NABLA Metodologia 2):
// Qbar[bh][b] = mean of the N = 64 tokens of block b, i.e. of the P x P
// patch (hp, wp) of frame t, or of the pt x ph x pw tile (t, hp, wp) in block
// units, read straight from the natural layout (the fractal flattening is
// only an addressing here). A block is pt * ph runs of pw consecutive tokens.
//
// One warp per (bh, block) and tensor; each lane owns d/32 channels and
// streams the 64 token rows with coalesced 8-byte (d = 128) or 4-byte loads,
// accumulating in fp32. HBM-bound: reads Q and K once, writes Qbar, Kbar and
// their split hi = tf32(x) (round to nearest, ties away), lo = x - hi (exact
// in fp32), which the logits GEMM multiplies as hi*hi + hi*lo + lo*hi on the
// TF32 tensor cores: the dropped lo*lo term and the tf32 rounding of lo are
// both ~2^-22 relative, fp32-level accuracy.
#include <cuda_bf16.h>

#include "kernels.cuh"

namespace sa {

template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   float* __restrict__ qbar,
                                                   float* __restrict__ kbar,
                                                   float* __restrict__ qsplit,
                                                   float* __restrict__ ksplit, Geometry g) {
  constexpr int kPerLane = D / 32;  // 4 or 2 channels per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long unit = long(blockIdx.x) * 8 + warp;  // (tensor, bh, b)
  const long per_tensor = long(g.BH) * g.nb;
  if (unit >= 2 * per_tensor) return;
  const int which = int(unit / per_tensor);
  const long rest = unit - which * per_tensor;
  const int bh = int(rest / g.nb), b = int(rest - long(bh) * g.nb);
  int t, hp, wp;
  block_coords(g, b, t, hp, wp);
  const __nv_bfloat16* src = (which == 0 ? q : k) + (size_t(bh) * g.S) * D + lane * kPerLane;
  float acc[kPerLane];
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) acc[i] = 0.f;
  // token r of the block: frame t*pt + (r >> (lph + lpw)), row hp*ph +
  // ((r >> lpw) & (ph - 1)), column wp*pw + (r & (pw - 1)); the 8 x 8 patch
  // of one frame (the default block) takes a loop with constant addressing
  const size_t base_tok = (size_t(t) * g.pt * g.Hh + size_t(hp) * g.ph) * g.Ww + size_t(wp) * g.pw;
  const bool patch8 = g.pt == 1 && g.ph == 8 && g.pw == 8;
#pragma unroll 2
  for (int r0 = 0; r0 < 64; r0 += 8) {
    float2 raw[8];
    const size_t run0 = patch8 ? base_tok + size_t(r0 >> 3) * g.Ww : 0;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      size_t tok;
      if (patch8) {
        tok = run0 + u;
      } else {
        const int r = r0 + u;
        const int run = r >> g.lpw, wi = r & (g.pw - 1);
        const int ti = run >> g.lph, hi = run & (g.ph - 1);
        tok = base_tok + (size_t(ti) * g.Hh + hi) * g.Ww + wi;
      }
      const __nv_bfloat16* p = src + tok * D;
      if constexpr (kPerLane == 4) {
        raw[u] = __ldg(reinterpret_cast<const float2*>(p));
      } else {
        raw[u].x = __ldg(reinterpret_cast<const float*>(p));
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
#pragma unroll
      for (int i = 0; i < kPerLane / 2; ++i) {
        const float2 f = __bfloat1622float2(h[i]);
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  }
  const size_t off = (size_t(bh) * g.nb + b) * D + lane * kPerLane;
  const size_t half = size_t(g.BH) * g.nb * D;  // lo follows hi
  float* dst = (which == 0 ? qbar : kbar) + off;
  float* hi = (which == 0 ? qsplit : ksplit) + off;
  const float inv = 1.0f / 64.0f;  // exact: N = 64
#pragma unroll
  for (int i = 0; i < kPerLane; ++i) {
    const float x = acc[i] * inv;
    uint32_t h;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
    dst[i] = x;
    hi[i] = __uint_as_float(h);
    hi[half + i] = x - __uint_as_float(h);
  }
}

cudaError_t launch_pool(const void* q, const void* k, float* qbar, float* kbar, float* qsplit,
                        float* ksplit, const Geometry& g, cudaStream_t stream) {
  const long units = 2L * g.BH * g.nb;
  const unsigned grid = unsigned((units + 7) / 8);
  const auto* qq = static_cast<const __nv_bfloat16*>(q);
  const auto* kk = static_cast<const __nv_bfloat16*>(k);
  if (g.d == 128)
    pool_kernel<128><<<grid, 256, 0, stream>>>(qq, kk, qbar, kbar, qsplit, ksplit, g);
  else
    pool_kernel<64><<<grid, 256, 0, stream>>>(qq, kk, qbar, kbar, qsplit, ksplit, g);
  return cudaGetLastError();
}

// Fractal flattening as an explicit copy: position b*64 + r of a head holds
// token r of block b (see the pooling above for r -> (t, h, w)). One warp per
// (bh, block, run of pw consecutive tokens): pw tokens x d channels,
// 16-byte vectors.
__global__ void __launch_bounds__(256) permute_kernel(const uint4* __restrict__ x,
                                                      uint4* __restrict__ y, Geometry g,
                                                      int inverse) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int runs = 64 >> g.lpw;                   // pt * ph runs per block
  const long unit = long(blockIdx.x) * 8 + warp;  // (bh, b, run)
  if (unit >= long(g.BH) * g.nb * runs) return;
  const long bb = unit / runs;
  const int run = int(unit - bb * runs);
  const int bh = int(bb / g.nb), b = int(bb - long(bh) * g.nb);
  int t, hp, wp;
  block_coords(g, b, t, hp, wp);
  const int ti = run >> g.lph, hi = run & (g.ph - 1);
  const int vec_per_row = g.d / 8;  // 16-byte vectors per token row
  const size_t nat = (size_t(t) * g.pt + ti) * g.Hh * g.Ww + size_t(hp * g.ph + hi) * g.Ww +
                     size_t(wp) * g.pw;
  const size_t frac = size_t(b) * 64 + size_t(run) * g.pw;
  const size_t head = size_t(bh) * g.S;
  const size_t src0 = (head + (inverse ? frac : nat)) * vec_per_row;
  const size_t dst0 = (head + (inverse ? nat : frac)) * vec_per_row;
  // the pw tokens of a run are contiguous in both orders
  for (int i = lane; i < g.pw * vec_per_row; i += 32) y[dst0 + i] = __ldg(x + src0 + i);
}

cudaError_t launch_permute(const void* x, void* y, const Geometry& g, int inverse,
                           cudaStream_t stream) {
  const long units = long(g.BH) * g.nb * (64 >> g.lpw);
  permute_kernel<<<unsigned((units + 7) / 8), 256, 0, stream>>>(
      static_cast<const uint4*>(x), static_cast<uint4*>(y), g, inverse);
  return cudaGetLastError();
}

}  // namespace sa
