// Host side of the C ABI declared in include/sparse_attn.h: argument
// validation, workspace layout, launch sequencing and status reporting.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>

#include "kernels.cuh"
#include "layout.cuh"
#include "tma_host.h"

using namespace sa;

namespace {

// Largest block count per head: the select kernel holds a row's masses in
// shared memory up to 6144 (192 per lane), and the radius kernel's row
// bitmap has 192 words. (The attention and gradient kernels stage the first
// 2880 entries of a list in shared memory and read the rest from L2.)
constexpr int kMaxBlocks = 6144;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

sa_status validate(const sa_desc* d) {
  if (d == nullptr) return SA_ERR_INVALID_ARG;
  const bool tiled = d->pt != 0 || d->ph != 0 || d->pw != 0;
  if (d->B < 1 || d->H < 1 || d->T < 1 || d->Hh < 1 || d->Ww < 1 || d->d < 1 || d->N < 1 ||
      (!tiled && d->P < 1))
    return SA_ERR_INVALID_ARG;
  if (!(d->thr >= 0.0f && d->thr < 1.0f)) return SA_ERR_INVALID_ARG;  // also rejects NaN
  const bool no_sta = d->sta_t == 0 && d->sta_h == 0 && d->sta_w == 0;
  if (!no_sta) {
    if (d->sta_t < 1 || d->sta_h < 1 || d->sta_w < 1) return SA_ERR_INVALID_ARG;
    if (!(d->sta_t & 1) || !(d->sta_h & 1) || !(d->sta_w & 1)) return SA_ERR_INVALID_ARG;
  }
  if (d->out_fp32 != 0 && d->out_fp32 != 1) return SA_ERR_INVALID_ARG;
  if (d->debug_flags & ~SA_DEBUG_STALL_LOADER) return SA_ERR_INVALID_ARG;
  if (d->d != 64 && d->d != 128) return SA_ERR_UNSUPPORTED;
  if (d->N != 64) return SA_ERR_UNSUPPORTED;  // the attention kernel's 64-row blocks
  int pt = 1, ph = d->P, pw = d->P;
  if (tiled) {
    if (d->pt < 1 || d->ph < 1 || d->pw < 1) return SA_ERR_INVALID_ARG;
    pt = d->pt;
    ph = d->ph;
    pw = d->pw;
  }
  if ((long long)pt * ph * pw != d->N) return SA_ERR_UNSUPPORTED;  // also: powers of 2
  if (d->T % pt || d->Hh % ph || d->Ww % pw) return SA_ERR_UNSUPPORTED;
  const long long BH = (long long)d->B * d->H;
  const long long nb = (long long)(d->T / pt) * (d->Hh / ph) * (d->Ww / pw);
  if (BH > 65535 || nb > kMaxBlocks) return SA_ERR_UNSUPPORTED;
  return SA_OK;
}

sa_status check_ws(const Geometry& g, const void* ws, size_t ws_bytes) {
  if (ws == nullptr || !aligned(ws, 256)) return SA_ERR_INVALID_ARG;
  if (ws_bytes < make_ws_layout(g).total) return SA_ERR_WORKSPACE;
  return SA_OK;
}

sa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SA_OK : SA_ERR_CUDA; }

template <class T>
T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<uint8_t*>(base) + off);
}
template <class T>
const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const uint8_t*>(base) + off);
}

}  // namespace

extern "C" {

sa_status sparse_attn_workspace_size(const sa_desc* desc, size_t* bytes) {
  const sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  *bytes = make_ws_layout(make_geometry(*desc)).total;
  return SA_OK;
}

// Stages of the plan, in launch order (sparse_attn_plan_profile).
const char* const kPlanStages[] = {"pool", "logits", "select", "union", "tile_order"};
constexpr int kNumPlanStages = 5;

// The plan; when ev is given (kNumPlanStages + 1 events) ev[0] is recorded
// before the first launch and ev[i + 1] after stage i.
static sa_status plan_impl(const sa_desc* desc, const void* q, const void* k, void* workspace,
                           size_t ws_bytes, void* stream, cudaEvent_t* ev) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (q == nullptr || k == nullptr || !aligned(q, 16) || !aligned(k, 16))
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const WsLayout w = make_ws_layout(g);
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  cudaError_t e;
  if (ev != nullptr && cudaEventRecord(ev[0], s) != cudaSuccess) return SA_ERR_CUDA;
  e = cudaMemsetAsync(at<uint32_t>(workspace, w.status), 0, 256, s);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  e = launch_pool(q, k, at<float>(workspace, w.qbar), at<float>(workspace, w.kbar),
                  at<float>(workspace, w.qsplit), at<float>(workspace, w.ksplit), g, s);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  if (ev != nullptr && cudaEventRecord(ev[1], s) != cudaSuccess) return SA_ERR_CUDA;

  MaskArgs m;
  std::memset(&m, 0, sizeof(m));
  const long long rows = (long long)g.BH * g.nb;
  const float* qsplit = at<float>(workspace, w.qsplit);
  const float* ksplit = at<float>(workspace, w.ksplit);
  if (!encode_rows_f32(&m.map_qhi, qsplit, rows, g.d, 128) ||
      !encode_rows_f32(&m.map_qlo, qsplit + rows * g.d, rows, g.d, 128) ||
      !encode_rows_f32(&m.map_khi, ksplit, rows, g.d, 256) ||
      !encode_rows_f32(&m.map_klo, ksplit + rows * g.d, rows, g.d, 256))
    return SA_ERR_CUDA;
  m.status = at<uint32_t>(workspace, w.status);
  m.qbar = at<float>(workspace, w.qbar);
  m.kbar = at<float>(workspace, w.kbar);
  m.logits = at<float>(workspace, w.logits);
  m.bits = at<uint32_t>(workspace, w.bits);
  m.cnt = at<int32_t>(workspace, w.cnt);
  m.idx = at<int32_t>(workspace, w.idx);
  m.tcnt = at<int32_t>(workspace, w.tcnt);
  m.tidx = at<int32_t>(workspace, w.tidx);
  m.dense = desc->thr == 0.0f;
  // mass threshold 1 - thr in the select kernel's 2^-30 fixed point
  m.target_fx = (uint32_t)std::llround((1.0 - (double)desc->thr) * 1073741824.0);
  const bool sta = desc->sta_t > 0;
  m.sta_t = sta ? desc->sta_t / 2 : -1;
  m.sta_h = sta ? desc->sta_h / 2 : -1;
  m.sta_w = sta ? desc->sta_w / 2 : -1;
  m.scale = (float)(1.0 / std::sqrt((double)g.d));
  e = launch_mask(m, g, s, ev != nullptr ? ev + 2 : nullptr);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  if (ev != nullptr && cudaEventRecord(ev[4], s) != cudaSuccess) return SA_ERR_CUDA;
  e = launch_tile_order(m.tcnt, at<int32_t>(workspace, w.order), g, s);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  if (ev != nullptr && cudaEventRecord(ev[5], s) != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}

sa_status sparse_attn_plan(const sa_desc* desc, const void* q, const void* k, void* workspace,
                           size_t ws_bytes, void* stream) {
  return plan_impl(desc, q, k, workspace, ws_bytes, stream, nullptr);
}

sa_status sparse_attn_plan_profile(const sa_desc* desc, const void* q, const void* k,
                                   void* workspace, size_t ws_bytes, int reps, float* stage_us,
                                   int max_stages, int* n_stages, void* stream) {
  if (reps < 1 || stage_us == nullptr || n_stages == nullptr || max_stages < kNumPlanStages)
    return SA_ERR_INVALID_ARG;
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  *n_stages = kNumPlanStages;
  for (int i = 0; i < kNumPlanStages; ++i) stage_us[i] = 0.f;
  cudaEvent_t ev[kNumPlanStages + 1];
  int made = 0;
  for (; made <= kNumPlanStages; ++made)
    if (cudaEventCreate(&ev[made]) != cudaSuccess) break;
  st = made == kNumPlanStages + 1 ? SA_OK : SA_ERR_CUDA;
  for (int r = 0; r < reps && st == SA_OK; ++r) {
    st = plan_impl(desc, q, k, workspace, ws_bytes, stream, ev);
    if (st == SA_OK && cudaEventSynchronize(ev[kNumPlanStages]) != cudaSuccess) st = SA_ERR_CUDA;
    for (int i = 0; i < kNumPlanStages && st == SA_OK; ++i) {
      float ms = 0.f;
      if (cudaEventElapsedTime(&ms, ev[i], ev[i + 1]) != cudaSuccess) st = SA_ERR_CUDA;
      stage_us[i] += ms * 1000.f / float(reps);
    }
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  return st;
}

const char* sparse_attn_plan_stage_name(int i) {
  return (i >= 0 && i < kNumPlanStages) ? kPlanStages[i] : nullptr;
}

static sa_status fwd_impl(const sa_desc* desc, const void* q, const void* k, const void* v,
                          const void* workspace, size_t ws_bytes, void* out, float* lse,
                          void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || !aligned(q, 16) ||
      !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const WsLayout w = make_ws_layout(g);
  AttnArgs a;
  std::memset(&a, 0, sizeof(a));
  const int pair_frames = g.nt > 1 ? 2 : 1;  // a temporal pair = two block frames
  if (!encode_tile_map(&a.map_q, q, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_k, k, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_v, v, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_k2, k, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw, pair_frames) ||
      !encode_tile_map(&a.map_v2, v, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw, pair_frames))
    return SA_ERR_CUDA;
  a.out = out;
  a.tcnt = at<int32_t>(workspace, w.tcnt);
  a.tidx = at<int32_t>(workspace, w.tidx);
  a.order = at<int32_t>(workspace, w.order);
  a.status = const_cast<uint32_t*>(at<uint32_t>(workspace, w.status));
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  a.out_fp32 = desc->out_fp32;
  a.debug_flags = desc->debug_flags;
  a.lse = lse;
  return cuda_status(launch_attn(a, g, static_cast<cudaStream_t>(stream)));
}

sa_status sparse_attn_fwd(const sa_desc* desc, const void* q, const void* k, const void* v,
                          const void* workspace, size_t ws_bytes, void* out, void* stream) {
  return fwd_impl(desc, q, k, v, workspace, ws_bytes, out, nullptr, stream);
}

sa_status sparse_attn_fwd_lse(const sa_desc* desc, const void* q, const void* k, const void* v,
                              const void* workspace, size_t ws_bytes, void* out, float* lse,
                              void* stream) {
  if (lse == nullptr || !aligned(lse, 4)) return SA_ERR_INVALID_ARG;
  return fwd_impl(desc, q, k, v, workspace, ws_bytes, out, lse, stream);
}

sa_status sparse_attn_bwd_scratch_size(const sa_desc* desc, size_t* bytes) {
  const sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  *bytes = make_bwd_layout(make_geometry(*desc)).total;
  return SA_OK;
}

sa_status sparse_attn_bwd(const sa_desc* desc, const void* q, const void* k, const void* v,
                          const void* out, const void* dout, const float* lse,
                          const void* workspace, size_t ws_bytes, void* dq, void* dk, void* dv,
                          void* scratch, size_t scratch_bytes, void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  const void* ptrs[] = {q, k, v, out, dout, dq, dk, dv, scratch};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned(p, 16)) return SA_ERR_INVALID_ARG;
  if (lse == nullptr || !aligned(lse, 4)) return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const BwdLayout b = make_bwd_layout(g);
  if (scratch_bytes < b.total) return SA_ERR_WORKSPACE;
  if (!aligned(scratch, 256)) return SA_ERR_INVALID_ARG;
  const WsLayout w = make_ws_layout(g);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  BwdArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!encode_tile_map(&a.map_q, q, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_k, k, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_v, v, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_do, dout, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw))
    return SA_ERR_CUDA;
  a.lse2 = at<float>(scratch, b.lse2);
  a.dsum = at<float>(scratch, b.dsum);
  a.kcnt = at<int32_t>(scratch, b.kcnt);
  a.kidx = at<int32_t>(scratch, b.kidx);
  a.dq_acc = at<float>(scratch, b.dq_acc);
  a.dk = dk;
  a.dv = dv;
  a.status = const_cast<uint32_t*>(at<uint32_t>(workspace, w.status));
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  a.scale = (float)(1.0 / std::sqrt((double)g.d));
  a.out_fp32 = desc->out_fp32;
  a.debug_flags = desc->debug_flags;
  cudaError_t e = cudaMemsetAsync(a.dq_acc, 0, sizeof(float) * size_t(g.BH) * g.S * g.d, s);
  if (e == cudaSuccess)
    e = launch_bwd_prep(out, dout, lse, at<float>(scratch, b.lse2), at<float>(scratch, b.dsum),
                        desc->out_fp32, g, s);
  if (e == cudaSuccess)
    e = launch_bwd_lists(at<uint32_t>(workspace, w.bits), at<int32_t>(scratch, b.kcnt),
                         at<int32_t>(scratch, b.kidx), g, s);
  if (e == cudaSuccess) e = launch_bwd(a, g, s);
  if (e == cudaSuccess) e = launch_dq_convert(a.dq_acc, dq, desc->out_fp32, g, s);
  return cuda_status(e);
}

sa_status sparse_attn_block_heatmap_scratch_size(const sa_desc* desc, size_t* bytes) {
  const sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  *bytes = heat_scratch_bytes(make_geometry(*desc));
  return SA_OK;
}

sa_status sparse_attn_block_heatmap(const sa_desc* desc, const void* q, const void* k,
                                    void* workspace, size_t ws_bytes, float* heat,
                                    void* scratch, size_t scratch_bytes, void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (q == nullptr || k == nullptr || heat == nullptr || scratch == nullptr ||
      !aligned(q, 16) || !aligned(k, 16) || !aligned(heat, 4) || !aligned(scratch, 16))
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  if (scratch_bytes < heat_scratch_bytes(g)) return SA_ERR_WORKSPACE;
  const WsLayout w = make_ws_layout(g);
  HeatArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!encode_tile_map(&a.map_q, q, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_k, k, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw))
    return SA_ERR_CUDA;
  a.heat = heat;
  a.scratch = static_cast<float*>(scratch);
  a.status = at<uint32_t>(workspace, w.status);
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  a.debug_flags = desc->debug_flags;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a.status, 0, sizeof(uint32_t), s) != cudaSuccess) return SA_ERR_CUDA;
  return cuda_status(launch_heat(a, g, s));
}

sa_status sparse_attn_token_entropy(const sa_desc* desc, const void* q, const void* k,
                                    void* workspace, size_t ws_bytes, float* entropy,
                                    void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (q == nullptr || k == nullptr || entropy == nullptr || !aligned(q, 16) || !aligned(k, 16) ||
      !aligned(entropy, 4))
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const WsLayout w = make_ws_layout(g);
  HeatArgs a;
  std::memset(&a, 0, sizeof(a));
  if (!encode_tile_map(&a.map_q, q, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw) ||
      !encode_tile_map(&a.map_k, k, g.BH, g.T, g.Hh, g.Ww, g.d, g.pt, g.ph, g.pw))
    return SA_ERR_CUDA;
  a.entropy = entropy;
  a.status = at<uint32_t>(workspace, w.status);
  a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)g.d));
  a.debug_flags = desc->debug_flags;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(a.status, 0, sizeof(uint32_t), s) != cudaSuccess) return SA_ERR_CUDA;
  return cuda_status(launch_heat(a, g, s));
}

sa_status sparse_attn_plan_radius(const sa_desc* desc, const sa_radius* radius,
                                  const float* entropy, void* workspace, size_t ws_bytes,
                                  void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (radius == nullptr || entropy == nullptr || !aligned(entropy, 4)) return SA_ERR_INVALID_ARG;
  if (!(radius->tau > 0.0f && std::isfinite(radius->tau)) ||
      !(radius->gamma >= 0.0f && std::isfinite(radius->gamma)) || radius->vote_min < 1 ||
      radius->vote_min > desc->N)
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  if (!radius_supported(g)) return SA_ERR_UNSUPPORTED;
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const WsLayout w = make_ws_layout(g);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(at<uint32_t>(workspace, w.status), 0, 256, s) != cudaSuccess)
    return SA_ERR_CUDA;
  RadiusArgs r;
  r.entropy = entropy;
  r.bits = at<uint32_t>(workspace, w.bits);
  r.cnt = at<int32_t>(workspace, w.cnt);
  r.idx = at<int32_t>(workspace, w.idx);
  r.tau = radius->tau;
  r.gamma = radius->gamma;
  r.vote_min = radius->vote_min;
  if (launch_radius(r, g, s) != cudaSuccess) return SA_ERR_CUDA;
  MaskArgs m;
  std::memset(&m, 0, sizeof(m));
  m.bits = r.bits;
  m.cnt = r.cnt;
  m.idx = r.idx;
  m.tcnt = at<int32_t>(workspace, w.tcnt);
  m.tidx = at<int32_t>(workspace, w.tidx);
  m.status = at<uint32_t>(workspace, w.status);
  if (launch_union(m, g, s) != cudaSuccess) return SA_ERR_CUDA;
  return cuda_status(launch_tile_order(m.tcnt, at<int32_t>(workspace, w.order), g, s));
}

sa_status sparse_attn_permute(const sa_desc* desc, const void* x, void* y, int inverse,
                              void* stream) {
  const sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (x == nullptr || y == nullptr || !aligned(x, 16) || !aligned(y, 16) ||
      (inverse != 0 && inverse != 1))
    return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  const size_t bytes = size_t(g.BH) * g.S * g.d * 2;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(x), yb = reinterpret_cast<uintptr_t>(y);
  if (xb < yb + bytes && yb < xb + bytes) return SA_ERR_INVALID_ARG;  // overlap
  return cuda_status(launch_permute(x, y, g, inverse, static_cast<cudaStream_t>(stream)));
}

sa_status sparse_attn_get_mask(const sa_desc* desc, const void* workspace, size_t ws_bytes,
                               sa_mask_views* views) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  if (views == nullptr) return SA_ERR_INVALID_ARG;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  const WsLayout w = make_ws_layout(g);
  views->qbar = at<float>(workspace, w.qbar);
  views->kbar = at<float>(workspace, w.kbar);
  views->cnt = at<int32_t>(workspace, w.cnt);
  views->idx = at<int32_t>(workspace, w.idx);
  views->tile_cnt = at<int32_t>(workspace, w.tcnt);
  views->tile_idx = at<int32_t>(workspace, w.tidx);
  views->nb = g.nb;
  views->ntile = g.ntile;
  views->logits = at<float>(workspace, w.logits);
  views->logits_ld = logits_ld(g);
  return SA_OK;
}

sa_status sparse_attn_tile_blocks(const sa_desc* desc, int tile, int* qa, int* qb) {
  const sa_status st = validate(desc);
  if (st != SA_OK) return st;
  const Geometry g = make_geometry(*desc);
  if (qa == nullptr || qb == nullptr || tile < 0 || tile >= g.ntile) return SA_ERR_INVALID_ARG;
  tile_blocks(g, tile, *qa, *qb);
  return SA_OK;
}

sa_status sparse_attn_check(const sa_desc* desc, const void* workspace, size_t ws_bytes,
                            void* stream) {
  sa_status st = validate(desc);
  if (st != SA_OK) return st;
  const Geometry g = make_geometry(*desc);
  st = check_ws(g, workspace, ws_bytes);
  if (st != SA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return SA_ERR_CUDA;
  uint32_t word = 0;
  const WsLayout w = make_ws_layout(g);
  if (cudaMemcpy(&word, at<uint32_t>(workspace, w.status), sizeof(word), cudaMemcpyDeviceToHost) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  return word ? SA_ERR_DEVICE_TIMEOUT : SA_OK;
}

const char* sparse_attn_status_string(sa_status status) {
  switch (status) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SA_ERR_WORKSPACE: return "workspace too small";
    case SA_ERR_CUDA: return "CUDA runtime error";
    case SA_ERR_DEVICE_TIMEOUT: return "a kernel's bounded wait ran out (device status set)";
  }
  return "unknown status";
}

}  // extern "C"
