// Plan + forward as one CUDA graph on fixed buffers: the whole path (status
// reset, pooling, logits GEMM, select, union, tile order, attention) is
// captured once and replayed with a single launch, the plan included (one
// plan per step) or not (a plan reused across steps, e.g. denoising steps of
// slowly drifting Q/K). Replays read whatever the buffers hold at the time.
#include <cuda_runtime.h>

#include <new>

#include "../../include/sparse_attn.h"

struct sa_graph {
  cudaGraph_t graph;
  cudaGraphExec_t exec;
};

extern "C" {

sa_status sparse_attn_graph_create(const sa_desc* desc, const void* q, const void* k,
                                   const void* v, void* workspace, size_t ws_bytes, void* out,
                                   int with_plan, sa_graph** graph) {
  if (graph == nullptr || (with_plan != 0 && with_plan != 1)) return SA_ERR_INVALID_ARG;
  *graph = nullptr;
  size_t need = 0;
  sa_status st = sparse_attn_workspace_size(desc, &need);  // validates desc, launches nothing
  if (st != SA_OK) return st;
  cudaStream_t s;
  if (cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking) != cudaSuccess) return SA_ERR_CUDA;
  if (cudaStreamBeginCapture(s, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(s);
    return SA_ERR_CUDA;
  }
  if (with_plan) st = sparse_attn_plan(desc, q, k, workspace, ws_bytes, s);
  if (st == SA_OK) st = sparse_attn_fwd(desc, q, k, v, workspace, ws_bytes, out, s);
  cudaGraph_t g = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(s, &g);
  cudaStreamDestroy(s);
  if (st != SA_OK || ec != cudaSuccess || g == nullptr) {
    if (g != nullptr) cudaGraphDestroy(g);
    return st != SA_OK ? st : SA_ERR_CUDA;
  }
  cudaGraphExec_t ex;
  if (cudaGraphInstantiate(&ex, g, 0) != cudaSuccess) {
    cudaGraphDestroy(g);
    return SA_ERR_CUDA;
  }
  sa_graph* h = new (std::nothrow) sa_graph{g, ex};
  if (h == nullptr) {
    cudaGraphExecDestroy(ex);
    cudaGraphDestroy(g);
    return SA_ERR_CUDA;
  }
  *graph = h;
  return SA_OK;
}

sa_status sparse_attn_graph_launch(sa_graph* graph, void* stream) {
  if (graph == nullptr) return SA_ERR_INVALID_ARG;
  return cudaGraphLaunch(graph->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? SA_OK
             : SA_ERR_CUDA;
}

sa_status sparse_attn_graph_destroy(sa_graph* graph) {
  if (graph == nullptr) return SA_OK;
  const bool ok = cudaGraphExecDestroy(graph->exec) == cudaSuccess &&
                  cudaGraphDestroy(graph->graph) == cudaSuccess;
  delete graph;
  return ok ? SA_OK : SA_ERR_CUDA;
}

}  // extern "C"
