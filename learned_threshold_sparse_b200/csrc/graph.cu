// eta_decode_graph_create / eta_step_graph_create: one decode step (or one
// whole serving-loop token: input copy, KV append, decode, output copy)
// recorded once into a CUDA graph and replayed per token.
//
// The decode step is three dependent kernels (screen, attention, merge; plus
// the rescue counters' reset and the selection export when those are asked
// for) chained by programmatic dependent launch.  Recording them once removes
// the per-launch host work and lets the driver submit the chain as one unit;
// the programmatic edges are kept by stream capture.  Every kernel reads its
// inputs (query, caches, sequence lengths, metadata) from device memory at
// run time, so one graph serves every token of a serving loop whose buffers
// stay in place.
#include <new>

#include "eta_device.cuh"
#include "eta_internal.h"

struct eta_decode_graph {
  cudaGraphExec_t exec;
};

namespace {

// The token's input and output copies of a recorded step, done by a kernel
// that reads or writes the page-locked host buffer directly (unified
// addressing) when both ends allow it: a copy of a few KB then costs one
// host-memory round trip instead of a copy-engine transfer.  Host-side data
// is loaded with .cv (fetched again, never served stale from a cache) and
// stored write-through.
constexpr int kCopyThreads = 256;

__global__ void __launch_bounds__(kCopyThreads)
    io_copy_kernel(uint8_t* dst, const uint8_t* src, size_t bytes, int src_host, unsigned long long* trace,
                   int slot) {
  if (threadIdx.x == 0) eta::dev::trace_first(trace, slot);
  const size_t n16 = (reinterpret_cast<uintptr_t>(dst) | reinterpret_cast<uintptr_t>(src)) % 16 == 0 ? bytes / 16 : 0;
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  const size_t t0 = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (size_t x = t0; x < n16; x += stride) {
    const uint4* s4 = reinterpret_cast<const uint4*>(src) + x;
    uint4* d4 = reinterpret_cast<uint4*>(dst) + x;
    if (src_host) {
      *d4 = __ldcv(s4);
    } else {
      __stwt(d4, *s4);
    }
  }
  for (size_t x = n16 * 16 + t0; x < bytes; x += stride) {
    if (src_host) {
      dst[x] = __ldcv(reinterpret_cast<const signed char*>(src) + x);
    } else {
      __stwt(reinterpret_cast<signed char*>(dst) + x, static_cast<signed char>(src[x]));
    }
  }
  if (trace) {
    __syncthreads();
    if (threadIdx.x == 0) eta::dev::trace_last(trace, slot + 1);
  }
}

// Device-side view of a page-locked host buffer, or nullptr when the buffer
// is not mapped into the device's address space.
void* host_view(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

bool is_device(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  return at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged;
}

// One input or output copy of a step: src/dst as given, the kernel's view of
// the host end resolved before recording.
struct IoCopy {
  void* dst = nullptr;
  const void* src = nullptr;
  size_t bytes = 0;
  bool h2d = true;
  void* kdst = nullptr;        // kernel path: device-visible destination
  const void* ksrc = nullptr;  // kernel path: device-visible source

  void plan() {
    if (!bytes) return;
    if (h2d) {
      void* hv = host_view(src);
      if (hv && is_device(dst)) { ksrc = hv; kdst = dst; }
    } else {
      void* hv = host_view(dst);
      if (hv && is_device(src)) { ksrc = src; kdst = hv; }
    }
  }

  // trace / slot: the step trace and this copy's first slot (see include/eta.h)
  eta_status record(cudaStream_t cs, unsigned long long* trace, int slot) const {
    if (!bytes) return ETA_OK;
    if (kdst) {
      const size_t units = (bytes + 16 * kCopyThreads - 1) / (16 * kCopyThreads);
      const int grid = static_cast<int>(units < 148 ? units : 148);
      io_copy_kernel<<<grid, kCopyThreads, 0, cs>>>(static_cast<uint8_t*>(kdst), static_cast<const uint8_t*>(ksrc),
                                                     bytes, h2d ? 1 : 0, trace, slot);
      return cudaGetLastError() == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
    }
    // the copy engine, direction taken from the unified address space
    return cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDefault, cs) == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
  }
};

eta_status check_decode(const eta_decode_params* p) {
  if (!p) return ETA_ERR_INVALID_ARG;
  for (int k = 0; k < 4; ++k)
    if (p->timing_events[k]) return ETA_ERR_INVALID_ARG;
  size_t need = 0;
  const eta_status st = eta_decode_workspace_size(p, &need);
  if (st != ETA_OK) return st;
  if (!p->workspace || p->workspace_bytes < need) return ETA_ERR_WORKSPACE;
  return ETA_OK;
}

// Records record(stream, side) on a private stream under thread-local
// capture and instantiates the result; `side` is a second private stream
// that record may fork work onto (an event recorded on `stream` and waited
// on by `side`) and must join back before it returns.  Nothing runs on the
// GPU.
template <typename F>
eta_status capture(F&& record, eta_decode_graph** out) {
  cudaStream_t cs = nullptr, side = nullptr;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return ETA_ERR_CUDA;
  if (cudaStreamCreateWithFlags(&side, cudaStreamNonBlocking) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return ETA_ERR_CUDA;
  }
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(cs);
    cudaStreamDestroy(side);
    (void)cudaGetLastError();
    return ETA_ERR_CUDA;
  }
  eta_status st = record(cs, side);
  cudaGraph_t graph = nullptr;
  const cudaError_t ec = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  cudaStreamDestroy(side);
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

}  // namespace

extern "C" eta_status eta_decode_graph_create(const eta_decode_params* p, eta_decode_graph** out) {
  if (!out) return ETA_ERR_INVALID_ARG;
  *out = nullptr;
  const eta_status st = check_decode(p);  // a bad argument records nothing
  if (st != ETA_OK) return st;
  return capture([&](cudaStream_t cs, cudaStream_t) { return eta_decode(p, cs); }, out);
}

extern "C" eta_status eta_step_graph_create(const eta_step_desc* d, eta_decode_graph** out) {
  if (!out) return ETA_ERR_INVALID_ARG;
  *out = nullptr;
  if (!d) return ETA_ERR_INVALID_ARG;
  const int nappend = (d->k_new != nullptr) + (d->v_new != nullptr) + (d->positions != nullptr);
  if (nappend != 0 && nappend != 3) return ETA_ERR_INVALID_ARG;
  if (d->q_new && nappend != 3) return ETA_ERR_INVALID_ARG;
  if (d->h2d_bytes && (!d->h2d_src || !d->h2d_dst)) return ETA_ERR_INVALID_ARG;
  if (d->d2h_bytes && (!d->d2h_src || !d->d2h_dst)) return ETA_ERR_INVALID_ARG;
  const eta_status st = check_decode(d->decode);
  if (st != ETA_OK) return st;
  const eta_decode_params* p = d->decode;
  IoCopy in, outc;
  in.dst = d->h2d_dst;
  in.src = d->h2d_src;
  in.bytes = d->h2d_bytes;
  in.h2d = true;
  outc.dst = d->d2h_dst;
  outc.src = d->d2h_src;
  outc.bytes = d->d2h_bytes;
  outc.h2d = false;
  in.plan();
  outc.plan();
  return capture(
      [&](cudaStream_t cs, cudaStream_t) -> eta_status {
        eta_status sc = in.record(cs, p->trace, ETA_TRACE_IN_FIRST);
        if (sc != ETA_OK) return sc;
        if (nappend == 3) {
          const eta_status sa = eta::append_step(&p->cache, &p->summary, d->k_new, d->v_new, d->positions, d->q_new,
                                                 d->q_new ? const_cast<void*>(p->q) : nullptr, cs, p->trace);
          if (sa != ETA_OK) return sa;
        }
        const eta_status sd = eta_decode(p, cs);
        if (sd != ETA_OK) return sd;
        return outc.record(cs, p->trace, ETA_TRACE_OUT_FIRST);
      },
      out);
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
