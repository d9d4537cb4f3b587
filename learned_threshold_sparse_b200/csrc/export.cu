// Export of the selection: the GQA-union list of every (sequence, KV head)
// with its head masks, and the integer selection counts (per-head blocks,
// union blocks) that Elastic Threshold Attention, Appendix F.4, reports for
// kernel validation.
#include <math.h>

#include "eta_device.cuh"

namespace eta {
namespace {

// One CTA per (KV head, sequence): the union list of the segment, ascending,
// with its head masks, and the per-head and union block counts.  Chunk
// offsets come from a prefix over the chunk counts in shared memory, so every
// entry is copied in parallel.
constexpr int kExportThreads = 256;

__global__ void __launch_bounds__(kExportThreads) export_kernel(ExportArgs a) {
  const Shape& s = a.s;
  const int g = blockIdx.x, i = blockIdx.y;
  const int seg = i * s.Hkv + g;
  const int t = threadIdx.x;
  if (t == 0) dev::trace_first(a.trace, ETA_TRACE_EXPORT_FIRST);
  extern __shared__ int s_off[];  // [nchunks + 1]
  __shared__ int s_head[8];
  if (t < 8) s_head[t] = 0;
  const int* counts = a.chunk_count + static_cast<size_t>(seg) * s.nchunks;
  // only the chunks that hold blocks of the sequence carry counts of this step
  int T = a.seq_lens[i];
  T = T < 0 ? 0 : (T > s.max_ctx ? s.max_ctx : T);
  const int nch = min(s.nchunks, ((T + s.b - 1) / s.b + s.chunk - 1) / s.chunk);
  if (t == 0) {
    // a count outside [0, chunk] cannot come from this step's screen: it is
    // read as 0 rather than trusted (never reads past a chunk's list)
    int run = 0;
    for (int c = 0; c < nch; ++c) {
      s_off[c] = run;
      const int n = counts[c];
      run += (n >= 0 && n <= s.chunk) ? n : 0;
    }
    s_off[nch] = run;
  }
  __syncthreads();
  const int total = s_off[nch];
  int hc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int c = 0; c < nch; ++c) {
    const int n = s_off[c + 1] - s_off[c];
    const int* list = a.chunk_list + static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(c) * s.chunk;
    for (int k = t; k < n; k += kExportThreads) {
      const int ent = list[k];
      const unsigned m = static_cast<unsigned>(ent) >> kEntryBlockBits;
      const size_t o = static_cast<size_t>(seg) * s.nbmax + s_off[c] + k;
      if (a.union_list) a.union_list[o] = ent & kMaxBlocksPerSeq;
      if (a.union_mask) a.union_mask[o] = m;
      for (int jj = 0; jj < s.G; ++jj) hc[jj] += (m >> jj) & 1u;
    }
  }
  for (int jj = 0; jj < s.G; ++jj) atomicAdd(&s_head[jj], hc[jj]);
  for (int k = total + t; k < s.nbmax; k += kExportThreads) {
    if (a.union_list) a.union_list[static_cast<size_t>(seg) * s.nbmax + k] = -1;
    if (a.union_mask) a.union_mask[static_cast<size_t>(seg) * s.nbmax + k] = 0u;
  }
  __syncthreads();
  if (t == 0 && a.union_count) a.union_count[seg] = total;
  if (t < s.G && a.admitted_count) a.admitted_count[static_cast<size_t>(i) * s.Hq + g * s.G + t] = s_head[t];
  if (t == 0) dev::trace_last(a.trace, ETA_TRACE_EXPORT_LAST);
}

}  // namespace

cudaError_t launch_export(const ExportArgs& a, cudaStream_t st) {
  const size_t smem = static_cast<size_t>(a.s.nchunks + 1) * sizeof(int);
  export_kernel<<<dim3(a.s.Hkv, a.s.B), kExportThreads, smem, st>>>(a);
  return cudaGetLastError();
}

}  // namespace eta
