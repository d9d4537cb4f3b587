// eta_decode_graph_*: one decode step recorded once into a CUDA graph and
// replayed per token.
//
// The step is three dependent kernels (screen, attention, merge; plus the
// rescue counters' reset and the selection export when those are asked for)
// chained by programmatic dependent launch.  Recording them once removes the
// per-launch host work and lets the driver submit the chain as one unit; the
// programmatic edges are kept by stream capture.  Every kernel reads its
// inputs (query, caches, sequence lengths, metadata) from device memory at
// run time, so one graph serves every token of a serving loop whose buffers
// stay in place.
#include <new>

#include "eta_internal.h"

struct eta_decode_graph {
  cudaGraphExec_t exec;
};

extern "C" eta_status eta_decode_graph_create(const eta_decode_params* p, eta_decode_graph** out) {
  if (!out) return ETA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!p) return ETA_ERR_INVALID_ARG;
  for (int k = 0; k < 4; ++k)
    if (p->timing_events[k]) return ETA_ERR_INVALID_ARG;
  // Host-side validation first: a bad argument records nothing.
  size_t need = 0;
  eta_status st = eta_decode_workspace_size(p, &need);
  if (st != ETA_OK) return st;
  if (!p->workspace || p->workspace_bytes < need) return ETA_ERR_WORKSPACE;

  cudaStream_t cs = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return ETA_ERR_CUDA;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(cs);
    (void)cudaGetLastError();
    return ETA_ERR_CUDA;
  }
  st = eta_decode(p, cs);
  cudaGraph_t graph = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  if (st == ETA_OK && (ec != cudaSuccess || !graph)) st = ETA_ERR_CUDA;
  cudaGraphExec_t exec = nullptr;
  if (st == ETA_OK && cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) st = ETA_ERR_CUDA;
  if (graph) cudaGraphDestroy(graph);
  if (st != ETA_OK) {
    if (exec) cudaGraphExecDestroy(exec);
    (void)cudaGetLastError();
    return st;
  }
  eta_decode_graph* g = new (std::nothrow) eta_decode_graph{exec};
  if (!g) {
    cudaGraphExecDestroy(exec);
    return ETA_ERR_CUDA;
  }
  *out = g;
  return ETA_OK;
}

extern "C" eta_status eta_decode_graph_launch(const eta_decode_graph* g, void* stream) {
  if (!g || !g->exec) return ETA_ERR_INVALID_ARG;
  return cudaGraphLaunch(g->exec, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

extern "C" eta_status eta_decode_graph_destroy(eta_decode_graph* g) {
  if (!g) return ETA_ERR_INVALID_ARG;
  const cudaError_t e = g->exec ? cudaGraphExecDestroy(g->exec) : cudaSuccess;
  delete g;
  return e == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}
