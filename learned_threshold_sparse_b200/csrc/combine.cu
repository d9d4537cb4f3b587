// Merge of the split-KV partials and export of the selection.
//
// Source: Elastic Threshold Attention, section 3.2 and Appendix F.3: chunk
// partials (acc_c, m_c, l_c) merged by the associative online-softmax
// reduction  m* = max m_c,  l* = sum l_c 2^(m_c - m*),
// o = sum 2^(m_c - m*) acc_c / l*   (base-2 state; lse = (m* + log2 l*) ln 2).
// Appendix F.4: the integer selection counts (per-head blocks, GQA-union
// blocks) reported for validation.
#include <math.h>

#include "eta_device.cuh"

namespace eta {
namespace {

// One CTA per (query head, sequence), one thread per output coordinate.
// The attention CTAs that touched segment `seg` are those owning its first
// and last unit; CTA c owns units [U c / N, U (c + 1) / N), so unit u belongs
// to CTA ((u + 1) N - 1) / U.  Their partials sit at slots seg + c.
__global__ void combine_kernel(CombineArgs a) {
  dev::pdl_wait();
  const Shape& s = a.s;
  const int h = blockIdx.x, i = blockIdx.y;
  const int g = h / s.G, j = h - g * s.G;
  const int seg = i * s.Hkv + g;
  const int e = threadIdx.x;
  const int D = s.d;
  const long long U = a.seg_start[s.nseg];
  const long long N = s.attend_ctas;
  const long long us = a.seg_start[seg], ue = a.seg_start[seg + 1];
  const size_t orow = (static_cast<size_t>(i) * s.Hq + h) * D;
  float o = 0.f, lse = -INFINITY;
  if (ue > us) {
    const int c0 = static_cast<int>(((us + 1) * N - 1) / U);
    const int c1 = static_cast<int>((ue * N - 1) / U);
    float mstar = -INFINITY;
    for (int c = c0; c <= c1; ++c) {
      const float* p = a.partials + (static_cast<size_t>(seg + c) * s.G + j) * (D + 2);
      mstar = fmaxf(mstar, p[D]);
    }
    if (mstar != -INFINITY) {
      float acc = 0.f, l = 0.f;
      for (int c = c0; c <= c1; ++c) {
        const float* p = a.partials + (static_cast<size_t>(seg + c) * s.G + j) * (D + 2);
        const float m = p[D];
        if (m == -INFINITY) continue;
        const float f = dev::fast_exp2(m - mstar);
        acc = fmaf(f, p[e], acc);
        l = fmaf(f, p[D + 1], l);
      }
      if (l > 0.f) {
        o = acc / l;
        lse = (mstar + log2f(l)) * 0.6931471805599453f;
      }
    }
  }
  if (s.elt == 4) {
    static_cast<float*>(a.out)[orow + e] = o;
  } else {
    static_cast<uint16_t*>(a.out)[orow + e] = dev::f32_to_bf16_rn(o);
  }
  if (e == 0 && a.lse) a.lse[static_cast<size_t>(i) * s.Hq + h] = lse;
}

// One CTA per (KV head, sequence): the union list of the segment, ascending,
// with its head masks, and the per-head and union block counts.
__global__ void export_kernel(ExportArgs a) {
  const Shape& s = a.s;
  const int g = blockIdx.x, i = blockIdx.y;
  const int seg = i * s.Hkv + g;
  const int t = threadIdx.x;
  __shared__ int s_head[8];
  if (t < 8) s_head[t] = 0;
  __syncthreads();
  int off = 0;
  for (int c = 0; c < s.nchunks; ++c) {
    const int n = a.chunk_count[static_cast<size_t>(seg) * s.nchunks + c];
    const int* list = a.chunk_list + static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(c) * s.chunk;
    for (int k = t; k < n; k += blockDim.x) {
      const int ent = list[k];
      const unsigned m = static_cast<unsigned>(ent) >> kEntryBlockBits;
      if (a.union_list) a.union_list[static_cast<size_t>(seg) * s.nbmax + off + k] = ent & kMaxBlocksPerSeq;
      if (a.union_mask) a.union_mask[static_cast<size_t>(seg) * s.nbmax + off + k] = m;
      for (int jj = 0; jj < s.G; ++jj)
        if ((m >> jj) & 1u) atomicAdd(&s_head[jj], 1);
    }
    off += n;
  }
  for (int k = off + t; k < s.nbmax; k += blockDim.x) {
    if (a.union_list) a.union_list[static_cast<size_t>(seg) * s.nbmax + k] = -1;
    if (a.union_mask) a.union_mask[static_cast<size_t>(seg) * s.nbmax + k] = 0u;
  }
  __syncthreads();
  if (t == 0 && a.union_count) a.union_count[seg] = off;
  if (t < s.G && a.admitted_count) a.admitted_count[static_cast<size_t>(i) * s.Hq + g * s.G + t] = s_head[t];
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.s.Hq, a.s.B);
  cfg.blockDim = dim3(a.s.d);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, combine_kernel, a);
}

cudaError_t launch_export(const ExportArgs& a, cudaStream_t st) {
  export_kernel<<<dim3(a.s.Hkv, a.s.B), 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace eta
