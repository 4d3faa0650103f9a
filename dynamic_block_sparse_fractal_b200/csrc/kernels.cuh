// Launch wrappers of the library's kernels (host side). Each returns the
// launch's cudaError_t; argument validation happens before any of them.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "layout.cuh"

namespace sa {

// Qbar, Kbar (fp32 means) and their tf32 hi / lo split for the logits GEMM
// (qsplit, ksplit: [2][BH][nb][d], hi first).
cudaError_t launch_pool(const void* q, const void* k, float* qbar, float* kbar, float* qsplit,
                        float* ksplit, const Geometry& g, cudaStream_t stream);

cudaError_t launch_permute(const void* x, void* y, const Geometry& g, int inverse,
                           cudaStream_t stream);

// Reduced map + CDF threshold + STA union -> per-q-block lists and keep
// bitmaps, then per-tile union lists. target_fx = round((1 - thr) * 2^30)
// (mass threshold in the select kernel's fixed point); dense = (thr == 0).
struct MaskArgs {
  CUtensorMap map_qhi, map_qlo;  // [BH*nb][d] fp32, box 32 x 128 rows
  CUtensorMap map_khi, map_klo;  // [BH*nb][d] fp32, box 32 x 256 rows
  const float* qbar;
  const float* kbar;
  float* logits;   // [BH][nb][logits_ld(g)]
  uint32_t* bits;  // [BH][nb][bitmap_words(g)]
  int32_t* cnt;
  int32_t* idx;
  int32_t* tcnt;
  int32_t* tidx;
  uint32_t* status;  // device status word (bounded waits of the logits GEMM)
  uint32_t target_fx;
  int dense;
  int sta_t, sta_h, sta_w;  // half-widths (window / 2), -1 = no STA
  float scale;              // 1 / sqrt(d)
};
// Three launches: logits GEMM, row select, tile union.
cudaError_t launch_mask(const MaskArgs& a, const Geometry& g, cudaStream_t stream);

// Per head: tiles sorted by descending union length (ties by tile index).
cudaError_t launch_tile_order(const int32_t* tcnt, int32_t* order, const Geometry& g,
                              cudaStream_t stream);

struct AttnArgs {
  CUtensorMap map_q, map_k, map_v;  // 5-D patch maps, see tma_host.h
  CUtensorMap map_k2, map_v2;       // the same with two-frame boxes
  void* out;
  const int32_t* tcnt;
  const int32_t* tidx;
  const int32_t* order;
  uint32_t* status;
  float scale_log2;  // log2(e) / sqrt(d)
  int out_fp32;
  int debug_flags;
};
cudaError_t launch_attn(const AttnArgs& a, const Geometry& g, cudaStream_t stream);

// Exact block max-pooled attention map: heat[bh][qb][kb] = max over the
// block pair of the full softmax probability (zeroes heat, then one launch of
// a persistent grid of heat_ctas(g) CTAs, each with 256 rows of nb fp32 of
// scratch).
struct HeatArgs {
  CUtensorMap map_q, map_k;  // 5-D patch maps, one block per box
  float* heat;               // [BH][nb][nb], fractal block order
  float* scratch;            // [heat_ctas(g)][nb][256]
  uint32_t* status;
  float scale_log2;  // log2(e) / sqrt(d)
};
constexpr int kHeatCtas = 148;  // one per SM of a B200
inline int heat_ctas(const Geometry& g) {
  const long units = long(g.BH) * ((g.nb + 3) / 4);  // four q-blocks each
  return int(units < kHeatCtas ? units : kHeatCtas);
}
inline size_t heat_scratch_bytes(const Geometry& g) {
  return size_t(heat_ctas(g)) * 256 * size_t(g.nb) * sizeof(float);
}
cudaError_t launch_heat(const HeatArgs& a, const Geometry& g, cudaStream_t stream);

}  // namespace sa
