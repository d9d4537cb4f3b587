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

// One CTA (4 warps) per (query head, sequence).  The attention CTAs that
// touched segment `seg` are those owning its first and last unit; CTA c owns
// units [U c / N, U (c + 1) / N), so unit u belongs to CTA ((u + 1) N - 1) / U.
// Their partials sit at slots seg + c (CTAs in between that own no unit at all
// wrote none).  Warps stride over the partials (loads
// independent, so they overlap), lanes over the coordinates.
constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(CombineArgs a) {
  dev::pdl_wait();
  const Shape& s = a.s;
  const int h = blockIdx.x, i = blockIdx.y;
  const int g = h / s.G, j = h - g * s.G;
  const int seg = i * s.Hkv + g;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;
  const int D = s.d;
  const int EPL = D / 32;  // 4 or 2 coordinates per lane
  const long long U = a.seg_start[s.nseg];
  const long long N = s.attend_ctas;
  const long long us = a.seg_start[seg], ue = a.seg_start[seg + 1];
  const size_t orow = (static_cast<size_t>(i) * s.Hq + h) * D;
  __shared__ float s_red[kCombineThreads / 32];
  __shared__ float s_acc[kCombineThreads / 32][128 + 1];

  int c0 = 0, c1 = -1;
  if (ue > us) {
    c0 = static_cast<int>(((us + 1) * N - 1) / U);
    c1 = static_cast<int>((ue * N - 1) / U);
  }
  const int PS = partial_stride(D);
  const size_t stride = static_cast<size_t>(s.G) * PS;
  const float* base = a.partials + (static_cast<size_t>(seg) * s.G + j) * PS;
  // CTAs with an empty range (fewer units than CTAs) wrote no partial.
  auto owns_units = [&](int c) { return U * c / N != U * (c + 1) / N; };
  float mloc = -INFINITY;
  for (int c = c0 + t; c <= c1; c += kCombineThreads)
    if (owns_units(c)) mloc = fmaxf(mloc, base[c * stride + D]);
  mloc = dev::warp_max(mloc);
  if (lane == 0) s_red[w] = mloc;
  __syncthreads();
  float mstar = s_red[0];
  for (int k = 1; k < kCombineThreads / 32; ++k) mstar = fmaxf(mstar, s_red[k]);

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  float l = 0.f;
  if (mstar != -INFINITY) {
#pragma unroll 4
    for (int c = c0 + w; c <= c1; c += kCombineThreads / 32) {
      if (!owns_units(c)) continue;
      const float* p = base + c * stride;
      const float m = p[D];
      const float f = (m == -INFINITY) ? 0.f : dev::fast_exp2(m - mstar);
      if (EPL == 4) {
        const float4 x = *reinterpret_cast<const float4*>(p + lane * 4);
        acc[0] = fmaf(f, x.x, acc[0]); acc[1] = fmaf(f, x.y, acc[1]);
        acc[2] = fmaf(f, x.z, acc[2]); acc[3] = fmaf(f, x.w, acc[3]);
      } else {
        const float2 x = *reinterpret_cast<const float2*>(p + lane * 2);
        acc[0] = fmaf(f, x.x, acc[0]); acc[1] = fmaf(f, x.y, acc[1]);
      }
      l = fmaf(f, p[D + 1], l);
    }
  }
  for (int e = 0; e < EPL; ++e) s_acc[w][lane * EPL + e] = acc[e];
  if (lane == 0) s_acc[w][128] = l;
  __syncthreads();
  if (t < D) {
    float sum = 0.f, lsum = 0.f;
    for (int k = 0; k < kCombineThreads / 32; ++k) {
      sum += s_acc[k][t];
      lsum += s_acc[k][128];
    }
    float o = 0.f, lse = -INFINITY;
    if (mstar != -INFINITY && lsum > 0.f) {
      o = sum / lsum;
      lse = (mstar + log2f(lsum)) * 0.6931471805599453f;
    }
    if (s.elt == 4) {
      static_cast<float*>(a.out)[orow + t] = o;
    } else {
      static_cast<uint16_t*>(a.out)[orow + t] = dev::f32_to_bf16_rn(o);
    }
    if (t == 0 && a.lse) a.lse[static_cast<size_t>(i) * s.Hq + h] = lse;
  }
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
  cfg.blockDim = dim3(kCombineThreads);
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
