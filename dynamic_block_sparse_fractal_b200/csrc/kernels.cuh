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
// Three launches: logits GEMM, row select, tile union. marks (optional, two
// events) are recorded after the logits GEMM and after the row select.
cudaError_t launch_mask(const MaskArgs& a, const Geometry& g, cudaStream_t stream,
                        cudaEvent_t* marks = nullptr);

// Per-tile union lists from the rows' keep bitmaps (a.bits -> a.tcnt, a.tidx).
cudaError_t launch_union(const MaskArgs& a, const Geometry& g, cudaStream_t stream);

// Token Radius Attention block mask: per q-block row, the k-blocks that at
// least vote_min of its query tokens reach (keep bitmap, count, ascending
// list, as the select step writes them).
struct RadiusArgs {
  const float* entropy;  // [BH][S] natural order, nats
  uint32_t* bits;        // [BH][nb][bitmap_words(g)]
  int32_t* cnt;          // [BH][nb]
  int32_t* idx;          // [BH][nb][nb]
  float tau;             // keys per query = min(S, tau exp(H))
  float gamma;           // radius decay exp(-gamma delta) per frame of distance
  int vote_min;          // 1 .. N
};
cudaError_t launch_radius(const RadiusArgs& a, const Geometry& g, cudaStream_t stream);
// The radius kernel's limits: T <= 4096 frames, Hh, Ww <= 1024, nb <= 6144 blocks.
bool radius_supported(const Geometry& g);

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
  float* lse;  // [BH][S] natural order: each row's log-sum-exp (natural log), or null
};
cudaError_t launch_attn(const AttnArgs& a, const Geometry& g, cudaStream_t stream);

// Exact block max-pooled attention map: heat[bh][qb][kb] = max over the
// block pair of the full softmax probability (zeroes heat, then one launch of
// a persistent grid of heat_ctas(g) CTAs, each with 256 rows of nb fp32 of
// scratch).
struct HeatArgs {
  CUtensorMap map_q, map_k;  // 5-D patch maps, one block per box
  float* heat;               // [BH][nb][nb], fractal block order (null: no map)
  float* scratch;            // [heat_ctas(g)][nb][256] (map only)
  float* entropy;            // [BH][S] natural order: each query's attention entropy
                             // in nats (null: none); heat or entropy must be given
  uint32_t* status;
  float scale_log2;  // log2(e) / sqrt(d)
  int debug_flags;   // SA_DEBUG_STALL_LOADER: the first K load is never issued (test hook)
};
// Gradients of the block-sparse attention. Scratch (every region 256-byte
// aligned): dq_acc fp32 [BH][S][d] natural order (zeroed, then reduced into),
// lse2 and dsum fp32 [BH][S] in fractal order, kcnt int32 [BH][ntile] and
// kidx int32 [BH][ntile][nb]: per key tile (the query-tile pairing applied to
// k-blocks) the q-blocks keeping either of its k-blocks, ascending, as
// q-block | kEntryKeepA (keeps the first k-block) | kEntryKeepB (the second).
struct BwdLayout {
  size_t dq_acc, lse2, dsum, kcnt, kidx, total;
};
inline BwdLayout make_bwd_layout(const Geometry& g) {
  BwdLayout b;
  size_t o = 0;
  b.dq_acc = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.S * g.d);
  b.lse2 = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.S);
  b.dsum = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.S);
  b.kcnt = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.ntile);
  b.kidx = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.ntile * g.nb);
  b.total = o;
  return b;
}

struct BwdArgs {
  CUtensorMap map_q, map_k, map_v, map_do;  // 5-D patch maps, one block per box
  const float* lse2;                        // [BH][S] fractal order, log2 units
  const float* dsum;                        // [BH][S] fractal order: rowsum(dO * O)
  const int32_t* kcnt;
  const int32_t* kidx;
  float* dq_acc;  // [BH][S][d] natural order, zeroed
  void* dk;       // [BH][S][d] natural order, bf16 or fp32
  void* dv;
  uint32_t* status;
  float scale_log2;  // log2(e) / sqrt(d)
  float scale;       // 1 / sqrt(d)
  int out_fp32;
  int debug_flags;   // SA_DEBUG_STALL_LOADER: the first Q load is never issued (test hook)
};
// D = rowsum(dO * O) and lse * log2(e), both into fractal order (o: bf16 or
// fp32 per o_fp32; do_: bf16; lse: natural-log row log-sum-exp, natural order).
cudaError_t launch_bwd_prep(const void* o, const void* do_, const float* lse, float* lse2,
                            float* dsum, int o_fp32, const Geometry& g, cudaStream_t stream);
// Per key tile, the q-blocks that keep one of its k-blocks (from the keep bitmaps).
cudaError_t launch_bwd_lists(const uint32_t* bits, int32_t* kcnt, int32_t* kidx, const Geometry& g,
                             cudaStream_t stream);
// dK, dV of every key tile and dQ reduced into dq_acc.
cudaError_t launch_bwd(const BwdArgs& a, const Geometry& g, cudaStream_t stream);
// dq = dq_acc (bf16 or fp32).
cudaError_t launch_dq_convert(const float* dq_acc, void* dq, int out_fp32, const Geometry& g,
                              cudaStream_t stream);

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
