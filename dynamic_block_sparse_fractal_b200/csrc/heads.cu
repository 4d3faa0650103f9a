// Per-head block shapes ("Tiling Consapevole delle Teste", Veda page section
// 2.2: a tiling (pt, ph, pw) chosen for each head): the (batch, head) pairs
// are split into maximal runs of consecutive heads that share a shape. Each
// run is an ordinary problem with H = run length on the runs' own slice of
// q, k, v, out (a head's [S, d] rows are contiguous in [B, H, S, d]) and its
// own slice of the workspace, handled by the single-shape entry points.
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <cstring>

#include "../../include/sparse_attn.h"

namespace {

struct Run {
  int head0, count;
  sa_desc sub;
  size_t ws_off, ws_bytes;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Calls f(run) for each run in order; stops and returns the first non-OK
// status (from a run's validation or from f). *total receives the workspace
// bytes of all runs.
template <class F>
sa_status for_each_run(const sa_desc* desc, const int* tiles, size_t* total, F&& f) {
  if (desc == nullptr || tiles == nullptr) return SA_ERR_INVALID_ARG;
  if (desc->B < 1 || desc->H < 1) return SA_ERR_INVALID_ARG;
  const long long bh_count = (long long)desc->B * desc->H;
  size_t off = 0;
  long long i = 0;
  while (i < bh_count) {
    long long j = i + 1;
    while (j < bh_count && tiles[3 * j] == tiles[3 * i] && tiles[3 * j + 1] == tiles[3 * i + 1] &&
           tiles[3 * j + 2] == tiles[3 * i + 2])
      ++j;
    Run r;
    r.head0 = int(i);
    r.count = int(j - i);
    r.sub = *desc;
    r.sub.B = 1;
    r.sub.H = r.count;
    r.sub.pt = tiles[3 * i];
    r.sub.ph = tiles[3 * i + 1];
    r.sub.pw = tiles[3 * i + 2];
    size_t bytes = 0;
    const sa_status st = sparse_attn_workspace_size(&r.sub, &bytes);
    if (st != SA_OK) return st;
    r.ws_off = off;
    r.ws_bytes = bytes;
    off = align256(off + bytes);
    const sa_status fs = f(r);
    if (fs != SA_OK) return fs;
    i = j;
  }
  if (total != nullptr) *total = off;
  return SA_OK;
}

size_t head_bytes(const sa_desc* d, size_t elem) {
  return size_t(d->T) * d->Hh * d->Ww * d->d * elem;
}

template <class T>
T* shift(T* p, size_t bytes) {
  return reinterpret_cast<T*>(reinterpret_cast<uintptr_t>(p) + bytes);
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

}  // namespace

extern "C" {

sa_status sparse_attn_workspace_size_heads(const sa_desc* desc, const int* tiles, size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  return for_each_run(desc, tiles, bytes, [](const Run&) { return SA_OK; });
}

sa_status sparse_attn_heads_run(const sa_desc* desc, const int* tiles, int run, sa_desc* sub,
                                int* head0, size_t* ws_offset, size_t* ws_bytes) {
  if (sub == nullptr || head0 == nullptr || ws_offset == nullptr || ws_bytes == nullptr || run < 0)
    return SA_ERR_INVALID_ARG;
  int k = 0;
  bool found = false;
  const sa_status st = for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    if (k++ == run) {
      *sub = r.sub;
      *head0 = r.head0;
      *ws_offset = r.ws_off;
      *ws_bytes = r.ws_bytes;
      found = true;
    }
    return SA_OK;
  });
  if (st != SA_OK) return st;
  return found ? SA_OK : SA_ERR_INVALID_ARG;
}

sa_status sparse_attn_plan_heads(const sa_desc* desc, const int* tiles, const void* q,
                                 const void* k, void* workspace, size_t ws_bytes, void* stream) {
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  if (workspace == nullptr || !aligned256(workspace)) return SA_ERR_INVALID_ARG;
  if (ws_bytes < need) return SA_ERR_WORKSPACE;
  const size_t hb = head_bytes(desc, 2);
  return for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    return sparse_attn_plan(&r.sub, shift(q, hb * r.head0), shift(k, hb * r.head0),
                            shift(workspace, r.ws_off), r.ws_bytes, stream);
  });
}

sa_status sparse_attn_fwd_heads(const sa_desc* desc, const int* tiles, const void* q,
                                const void* k, const void* v, const void* workspace,
                                size_t ws_bytes, void* out, void* stream) {
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  if (workspace == nullptr || !aligned256(workspace)) return SA_ERR_INVALID_ARG;
  if (ws_bytes < need) return SA_ERR_WORKSPACE;
  const size_t hb = head_bytes(desc, 2);
  const size_t ob = head_bytes(desc, desc->out_fp32 ? 4 : 2);
  return for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    return sparse_attn_fwd(&r.sub, shift(q, hb * r.head0), shift(k, hb * r.head0),
                           shift(v, hb * r.head0), shift(workspace, r.ws_off), r.ws_bytes,
                           shift(out, ob * r.head0), stream);
  });
}

sa_status sparse_attn_fwd_lse_heads(const sa_desc* desc, const int* tiles, const void* q,
                                   const void* k, const void* v, const void* workspace,
                                   size_t ws_bytes, void* out, float* lse, void* stream) {
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  if (workspace == nullptr || !aligned256(workspace)) return SA_ERR_INVALID_ARG;
  if (ws_bytes < need) return SA_ERR_WORKSPACE;
  if (lse == nullptr) return SA_ERR_INVALID_ARG;
  const size_t hb = head_bytes(desc, 2);
  const size_t ob = head_bytes(desc, desc->out_fp32 ? 4 : 2);
  const size_t S = size_t(desc->T) * desc->Hh * desc->Ww;
  return for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    return sparse_attn_fwd_lse(&r.sub, shift(q, hb * r.head0), shift(k, hb * r.head0),
                               shift(v, hb * r.head0), shift(workspace, r.ws_off), r.ws_bytes,
                               shift(out, ob * r.head0), lse + S * r.head0, stream);
  });
}

// The runs execute one after another on the caller's stream, so one scratch
// buffer of the largest run's size serves them all.
sa_status sparse_attn_bwd_scratch_size_heads(const sa_desc* desc, const int* tiles,
                                             size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  size_t most = 0;
  const sa_status st = for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    size_t b = 0;
    const sa_status s = sparse_attn_bwd_scratch_size(&r.sub, &b);
    if (b > most) most = b;
    return s;
  });
  if (st == SA_OK) *bytes = most;
  return st;
}

sa_status sparse_attn_bwd_heads(const sa_desc* desc, const int* tiles, const void* q,
                               const void* k, const void* v, const void* out, const void* dout,
                               const float* lse, const void* workspace, size_t ws_bytes, void* dq,
                               void* dk, void* dv, void* scratch, size_t scratch_bytes,
                               void* stream) {
  size_t need = 0, scr = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  st = sparse_attn_bwd_scratch_size_heads(desc, tiles, &scr);
  if (st != SA_OK) return st;
  if (workspace == nullptr || !aligned256(workspace) || lse == nullptr) return SA_ERR_INVALID_ARG;
  if (ws_bytes < need || scratch_bytes < scr) return SA_ERR_WORKSPACE;
  const size_t hb = head_bytes(desc, 2);
  const size_t ob = head_bytes(desc, desc->out_fp32 ? 4 : 2);
  const size_t S = size_t(desc->T) * desc->Hh * desc->Ww;
  return for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    return sparse_attn_bwd(&r.sub, shift(q, hb * r.head0), shift(k, hb * r.head0),
                           shift(v, hb * r.head0), shift(out, ob * r.head0),
                           shift(dout, hb * r.head0), lse + S * r.head0,
                           shift(workspace, r.ws_off), r.ws_bytes, shift(dq, ob * r.head0),
                           shift(dk, ob * r.head0), shift(dv, ob * r.head0), scratch,
                           scratch_bytes, stream);
  });
}

sa_status sparse_attn_block_heatmap_scratch_size_heads(const sa_desc* desc, const int* tiles,
                                                       size_t* bytes) {
  if (bytes == nullptr) return SA_ERR_INVALID_ARG;
  size_t most = 0;
  const sa_status st = for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    size_t b = 0;
    const sa_status s = sparse_attn_block_heatmap_scratch_size(&r.sub, &b);
    if (b > most) most = b;
    return s;
  });
  if (st == SA_OK) *bytes = most;
  return st;
}

sa_status sparse_attn_block_heatmap_heads(const sa_desc* desc, const int* tiles, const void* q,
                                          const void* k, void* workspace, size_t ws_bytes,
                                          float* heat, void* scratch, size_t scratch_bytes,
                                          void* stream) {
  size_t need = 0, scr = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  st = sparse_attn_block_heatmap_scratch_size_heads(desc, tiles, &scr);
  if (st != SA_OK) return st;
  if (workspace == nullptr || !aligned256(workspace) || heat == nullptr) return SA_ERR_INVALID_ARG;
  if (ws_bytes < need || scratch_bytes < scr) return SA_ERR_WORKSPACE;
  const size_t hb = head_bytes(desc, 2);
  const size_t nb = size_t(desc->T) * desc->Hh * desc->Ww / 64;  // the same for every shape
  return for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    return sparse_attn_block_heatmap(&r.sub, shift(q, hb * r.head0), shift(k, hb * r.head0),
                                     shift(workspace, r.ws_off), r.ws_bytes,
                                     heat + nb * nb * r.head0, scratch, scratch_bytes, stream);
  });
}

sa_status sparse_attn_check_heads(const sa_desc* desc, const int* tiles, const void* workspace,
                                  size_t ws_bytes, void* stream) {
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size_heads(desc, tiles, &need);
  if (st != SA_OK) return st;
  if (workspace == nullptr || ws_bytes < need) return SA_ERR_WORKSPACE;
  sa_status worst = SA_OK;
  st = for_each_run(desc, tiles, nullptr, [&](const Run& r) {
    const sa_status s = sparse_attn_check(&r.sub, shift(workspace, r.ws_off), r.ws_bytes, stream);
    if (s == SA_ERR_CUDA) return s;
    if (s != SA_OK) worst = s;
    return SA_OK;
  });
  return st != SA_OK ? st : worst;
}

}  // extern "C"
