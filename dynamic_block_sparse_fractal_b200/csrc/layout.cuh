// Geometry shared by the host entry points and the kernels: block grid,
// query-tile pairing and the workspace layout.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/sparse_attn.h"

namespace sa {

#define SA_HD __host__ __device__ __forceinline__

struct Geometry {
  int BH, T, Hh, Ww, d, P, N;
  int pt, ph, pw;     // block shape (frames, rows, columns); pt*ph*pw = N
  int lph, lpw;       // log2(ph), log2(pw) (N = 64: every extent is a power of 2)
  int nt, nh, nw;     // blocks along t, h and w
  int nb;             // blocks per head = nt * nh * nw
  int ntile;    // query tiles per head
  int S;        // tokens per head
};

SA_HD Geometry make_geometry(const sa_desc& s) {
  Geometry g;
  g.BH = s.B * s.H;
  g.T = s.T;
  g.Hh = s.Hh;
  g.Ww = s.Ww;
  g.d = s.d;
  g.P = s.P;
  const bool tiled = s.pt != 0 || s.ph != 0 || s.pw != 0;
  g.pt = tiled ? s.pt : 1;
  g.ph = tiled ? s.ph : s.P;
  g.pw = tiled ? s.pw : s.P;
  g.lph = 0;
  while ((1 << g.lph) < g.ph) ++g.lph;
  g.lpw = 0;
  while ((1 << g.lpw) < g.pw) ++g.lpw;
  g.N = s.N;
  g.nt = s.T / g.pt;
  g.nh = s.Hh / g.ph;
  g.nw = s.Ww / g.pw;
  g.nb = g.nt * g.nh * g.nw;
  g.S = s.T * s.Hh * s.Ww;
  const int pairs_t = (g.nt / 2) * g.nh * g.nw;
  g.ntile = pairs_t + ((g.nt & 1) ? g.nh * ((g.nw + 1) / 2) : 0);
  return g;
}

// Block b (fractal block order) -> block coordinates (t, hp, wp) along
// (time, rows, columns), in units of the block shape.
SA_HD void block_coords(const Geometry& g, int b, int& t, int& hp, int& wp) {
  const int per_frame = g.nh * g.nw;
  t = b / per_frame;
  const int r = b - t * per_frame;
  hp = r / g.nw;
  wp = r - hp * g.nw;
}

// Natural token index (within a head) of row i (0..63) of block b: frame
// t*pt + (i >> (lph + lpw)), row hp*ph + ((i >> lpw) & (ph - 1)), column
// wp*pw + (i & (pw - 1)).
SA_HD int block_row_token(const Geometry& g, int b, int i) {
  int t, hp, wp;
  block_coords(g, b, t, hp, wp);
  const int run = i >> g.lpw;
  return (t * g.pt + (run >> g.lph)) * g.Hh * g.Ww + (hp * g.ph + (run & (g.ph - 1))) * g.Ww +
         wp * g.pw + (i & (g.pw - 1));
}

// Query tile -> the two q-blocks it holds (qb = -1 when alone). Pairs are
// the same patch in block frames (2i, 2i+1); an odd last block frame pairs
// neighbouring patch columns.
SA_HD void tile_blocks(const Geometry& g, int tile, int& qa, int& qb) {
  const int per_frame = g.nh * g.nw;
  const int pairs_t = (g.nt / 2) * per_frame;
  if (tile < pairs_t) {
    const int tp = tile / per_frame;
    qa = 2 * tp * per_frame + (tile - tp * per_frame);
    qb = qa + per_frame;
  } else {
    const int i = tile - pairs_t;
    const int half = (g.nw + 1) / 2;
    const int hp = i / half, wq = i - hp * half;
    qa = (g.nt - 1) * per_frame + hp * g.nw + 2 * wq;
    qb = (2 * wq + 1 < g.nw) ? qa + 1 : -1;
  }
}

// Workspace: every region starts on a 256-byte boundary.
struct WsLayout {
  size_t status;   // uint32 device status word (+ padding)
  size_t qbar;     // float [BH][nb][d]
  size_t kbar;     // float [BH][nb][d]
  size_t cnt;      // int32 [BH][nb]
  size_t idx;      // int32 [BH][nb][nb]
  size_t tcnt;     // int32 [BH][ntile]
  size_t tidx;     // int32 [BH][ntile][nb]
  size_t order;    // int32 [BH][ntile]: tiles of a head, heaviest union first
  size_t qsplit;   // float [2][BH][nb][d]: Qbar as tf32 hi and lo = Qbar - hi
  size_t ksplit;   // float [2][BH][nb][d]: the same for Kbar
  size_t logits;   // float [BH][nb][logits_ld]: the reduced map's scaled logits
  size_t bits;     // uint32 [BH][nb][nwords]: keep bitmap of every q-block row
  size_t total;
};

// Row pitch of the logits region (whole 256-column tiles of the logits GEMM)
// and words per keep bitmap.
SA_HD int logits_ld(const Geometry& g) { return (g.nb + 255) / 256 * 256; }
SA_HD int bitmap_words(const Geometry& g) { return (g.nb + 31) / 32; }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline WsLayout make_ws_layout(const Geometry& g) {
  WsLayout w;
  size_t o = 0;
  w.status = o; o = align256(o + 256);
  w.qbar = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.nb * g.d);
  w.kbar = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.nb * g.d);
  w.cnt = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.nb);
  w.idx = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.nb * g.nb);
  w.tcnt = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.ntile);
  w.tidx = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.ntile * g.nb);
  w.order = o; o = align256(o + sizeof(int32_t) * size_t(g.BH) * g.ntile);
  w.qsplit = o; o = align256(o + sizeof(float) * 2 * size_t(g.BH) * g.nb * g.d);
  w.ksplit = o; o = align256(o + sizeof(float) * 2 * size_t(g.BH) * g.nb * g.d);
  w.logits = o; o = align256(o + sizeof(float) * size_t(g.BH) * g.nb * logits_ld(g));
  w.bits = o; o = align256(o + sizeof(uint32_t) * size_t(g.BH) * g.nb * bitmap_words(g));
  w.total = o;
  return w;
}

// Union-list entry: k-block id | keep bit of the tile's first q-block << 16
// | keep bit of the second q-block << 17 | kEntryTPair on the first entry of
// a step whose two k-blocks are the same patch in frames t and t+1 (the next
// entry is then this block + patches per frame).
constexpr int kEntryBlockMask = 0xFFFF;
constexpr int kEntryKeepA = 1 << 16;
constexpr int kEntryKeepB = 1 << 17;
constexpr int kEntryTPair = 1 << 18;

}  // namespace sa
