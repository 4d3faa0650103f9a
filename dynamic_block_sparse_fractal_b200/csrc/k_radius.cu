// Token Radius Attention block mask (page "Token Radius Attention per la
// Generazione di Video Efficiente", gist.science/it/paper/2608.02504, section
// 2, "La Pipeline TRA"), from each query token's attention entropy H:
//
//   budget   k = min(S, tau exp(H)) keys ("Entropy-to-Budget");
//   radius   r^2 = k / (pi Z(t)), Z(t) = sum over the frames t' of
//            exp(-2 gamma |t' - t|): the discs of radius r exp(-gamma delta)
//            in the frames at distance delta hold k keys in all
//            ("Budget-to-Radius");
//   support  key (t', h', w') of query (t, h, w) iff
//            (h' - h)^2 + (w' - w)^2 <= r^2 exp(-2 gamma |t' - t|);
//   votes    query token i votes for k-block b iff its support holds a key of
//            b; block (a, b) is kept iff at least vote_min of a's N query
//            tokens vote for b ("Kernel CUDA Fusi": distance, radius test,
//            block pruning and token votes in one pass).
//
// A k-block is a box of frames x rows x columns, so the key of b nearest to a
// query lies at the box's nearest frame, row and column: the query votes iff
// dh^2 + dw^2 <= r^2 f(dt), dt, dh, dw its distances to the box along time,
// rows and columns (0 inside), f(dt) = exp(-2 gamma dt). A whole k-block is
// pruned first when even the q-block's bounding box, at the largest radius of
// its queries, misses it.
//
// One warp per q-block row; eight rows per CTA. Each lane holds two of the
// q-block's 64 queries; the k-blocks are taken 32 at a time (lane = k-block)
// for the pruning test, then the warp walks the unpruned ones and its lanes
// vote for each at once. The per-frame tables f and 1 / (pi Z) are built once
// per CTA in fp64 and kept as fp32.
#include <cuda_runtime.h>

#include "kernels.cuh"

namespace sa {

namespace {

constexpr int kRadWarps = 8;
constexpr int kRadMaxFrames = 4096;
constexpr int kRadMaxWords = 192;  // keep-bitmap words of a row (nb <= 6144)

__device__ __forceinline__ int dist_to_range(int x, int lo, int hi) {
  return x < lo ? lo - x : (x > hi ? x - hi : 0);
}

__global__ void __launch_bounds__(kRadWarps * 32) radius_kernel(RadiusArgs a, Geometry g) {
  __shared__ float f_tab[kRadMaxFrames];     // exp(-2 gamma delta)
  __shared__ float zinv_tab[kRadMaxFrames];  // 1 / (pi Z(t))
  __shared__ uint32_t rbits_all[kRadWarps][kRadMaxWords];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = g.T;
  // Per-frame tables in fp64, kept as fp32. With rho = exp(-2 gamma),
  // Z(t) = G(t) + G(T - 1 - t) - 1 where G(n) = sum_{u=0}^{n} rho^u
  // = expm1(-2 gamma (n + 1)) / expm1(-2 gamma) (n + 1 when gamma = 0).
  const double g2 = -2.0 * double(a.gamma);
  for (int t = threadIdx.x; t < T; t += blockDim.x) {
    f_tab[t] = float(exp(g2 * t));
    const double lo = g2 == 0.0 ? double(t + 1) : expm1(g2 * (t + 1)) / expm1(g2);
    const double hi = g2 == 0.0 ? double(T - t) : expm1(g2 * (T - t)) / expm1(g2);
    zinv_tab[t] = float(1.0 / (3.14159265358979323846 * (lo + hi - 1.0)));
  }
  __syncthreads();
  const long row = long(blockIdx.x) * kRadWarps + warp;
  if (row >= long(g.BH) * g.nb) return;
  const int bh = int(row / g.nb), qb = int(row - long(bh) * g.nb);
  const float S = float(g.S);

  // ---- the q-block's queries (lane holds queries lane and lane + 32):
  // position and squared base radius
  int qtt[2], qhh[2], qww[2];
  float r2q[2];
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int tok = block_row_token(g, qb, lane + 32 * u);
    qtt[u] = tok / (g.Hh * g.Ww);
    const int rem = tok - qtt[u] * g.Hh * g.Ww;
    qhh[u] = rem / g.Ww;
    qww[u] = rem - qhh[u] * g.Ww;
    const float H = a.entropy[size_t(bh) * g.S + tok];
    const float k = fminf(a.tau * expf(H), S);
    r2q[u] = k * zinv_tab[qtt[u]];
  }
  float r2max = fmaxf(r2q[0], r2q[1]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) r2max = fmaxf(r2max, __shfl_xor_sync(0xFFFFFFFFu, r2max, o));
  int qt, qh, qw;
  block_coords(g, qb, qt, qh, qw);
  const int qt0 = qt * g.pt, qt1 = qt0 + g.pt - 1;
  const int qh0 = qh * g.ph, qh1 = qh0 + g.ph - 1;
  const int qw0 = qw * g.pw, qw1 = qw0 + g.pw - 1;

  // ---- votes per k-block: 32 k-blocks per round (lane = k-block) for the
  // pruning test, then every unpruned one voted on by all 64 queries
  uint32_t* rbits = rbits_all[warp];
  const int nwords = bitmap_words(g);
  for (int base = 0; base < g.nb; base += 32) {
    const int kb = base + lane;
    bool live = false;
    uint32_t corner = 0u;  // (t0 << 20) | (h0 << 10) | w0 of the k-block's box
    if (kb < g.nb) {
      int kt, kh, kw;
      block_coords(g, kb, kt, kh, kw);
      const int kt0 = kt * g.pt, kt1 = kt0 + g.pt - 1;
      const int kh0 = kh * g.ph, kh1 = kh0 + g.ph - 1;
      const int kw0 = kw * g.pw, kw1 = kw0 + g.pw - 1;
      corner = (uint32_t(kt0) << 20) | (uint32_t(kh0) << 10) | uint32_t(kw0);
      // prune: the nearest points of the two boxes, at the largest radius
      const int bt = kt0 > qt1 ? kt0 - qt1 : (qt0 > kt1 ? qt0 - kt1 : 0);
      const int bhd = kh0 > qh1 ? kh0 - qh1 : (qh0 > kh1 ? qh0 - kh1 : 0);
      const int bwd = kw0 > qw1 ? kw0 - qw1 : (qw0 > kw1 ? qw0 - kw1 : 0);
      live = float(bhd * bhd + bwd * bwd) <= r2max * f_tab[bt];
    }
    uint32_t unp = __ballot_sync(0xFFFFFFFFu, live), keep = 0u;
    while (unp) {  // warp-uniform
      const int j = __ffs(unp) - 1;
      unp &= unp - 1u;
      const uint32_t c = __shfl_sync(0xFFFFFFFFu, corner, j);
      const int kt0 = int(c >> 20), kh0 = int((c >> 10) & 1023u), kw0 = int(c & 1023u);
      const int kt1 = kt0 + g.pt - 1, kh1 = kh0 + g.ph - 1, kw1 = kw0 + g.pw - 1;
      int votes = 0;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int dt = dist_to_range(qtt[u], kt0, kt1);
        const int dh = dist_to_range(qhh[u], kh0, kh1), dw = dist_to_range(qww[u], kw0, kw1);
        votes += __popc(__ballot_sync(0xFFFFFFFFu,
                                      float(dh * dh + dw * dw) <= r2q[u] * f_tab[dt]));
      }
      if (votes >= a.vote_min) keep |= 1u << j;
    }
    if (lane == 0) rbits[base >> 5] = keep;
  }
  __syncwarp();

  // ---- bitmap, ascending list and count to global: a lane per word
  uint32_t* bits = a.bits + size_t(row) * nwords;
  int32_t* out_idx = a.idx + size_t(row) * g.nb;
  int done = 0;
  for (int w0 = 0; w0 < nwords; w0 += 32) {
    const int wi = w0 + lane;
    uint32_t x = wi < nwords ? rbits[wi] : 0u;
    if (wi < nwords) bits[wi] = x;
    const int c = __popc(x);
    int inc = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xFFFFFFFFu, inc, o);
      if (lane >= o) inc += v;
    }
    int o = done + inc - c;
    while (x) {
      out_idx[o++] = 32 * wi + __ffs(x) - 1;
      x &= x - 1u;
    }
    done += __shfl_sync(0xFFFFFFFFu, inc, 31);
  }
  if (lane == 0) a.cnt[row] = done;
}

}  // namespace

bool radius_supported(const Geometry& g) {
  return g.T <= kRadMaxFrames && bitmap_words(g) <= kRadMaxWords && g.Hh <= 1024 &&
         g.Ww <= 1024 && g.N == 64;
}

cudaError_t launch_radius(const RadiusArgs& a, const Geometry& g, cudaStream_t stream) {
  const long rows = long(g.BH) * g.nb;
  radius_kernel<<<unsigned((rows + kRadWarps - 1) / kRadWarps), kRadWarps * 32, 0, stream>>>(a, g);
  return cudaGetLastError();
}

}  // namespace sa
