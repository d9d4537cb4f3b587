// Merge of the split-KV partials of the segments (sequence, KV head) that
// several attention CTAs shared.
//
// Source: Elastic Threshold Attention, section 3.2 and Appendix F.3: chunk
// partials (acc_c, m_c, l_c) are merged by the associative online-softmax
// reduction  m* = max m_c,  l* = sum l_c 2^(m_c - m*),
// o = sum 2^(m_c - m*) acc_c / l*  (base-2 state; lse = (m* + log2 l*) ln 2).
//
// Grid (nseg * G, d / 32): one CTA per (segment, query head of its group,
// 32-coordinate slice); warp w folds partials w, w + 8, ... online (every load
// of a warp is issued before it is used, so the partials arrive in one round
// trip), then the eight warp states are combined in shared memory.  Segments
// owned by a single attention CTA were written by that CTA and are skipped.
// Launched with programmatic dependent launch: the CTAs become resident while
// the attention kernel runs and start as soon as it completes.
#include <math.h>

#include "attend_common.cuh"

namespace eta {
namespace {

constexpr int kMergeWarps = 8;
constexpr int kBatch = 8;  // partials in flight per lane

__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(MergeArgs a) {
  const Shape& s = a.s;
  const int seg = blockIdx.x / s.G, h = blockIdx.x - seg * s.G;
  const int slice = blockIdx.y;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;

  // The segment's unit range [us, ue) and the total U, from the screen's chunk
  // counts.  The screen (and rescue) grids completed before the attention
  // kernel passed its own dependency wait, and this grid is launched only
  // after every attention CTA passed it, so the counts are final here; they
  // are read from L2 before this grid's own wait, overlapping the attention.
  __shared__ int s_rng[3];
  if (w == 0) {
    const int n = s.nseg * s.nchunks, lo = seg * s.nchunks, hi = lo + s.nchunks;
    int before = 0, inside = 0, total = 0;
    for (int x = lane; x < n; x += 32) {
      const int c = __ldcg(a.chunk_count + x);
      total += c;
      before += x < lo ? c : 0;
      inside += (x >= lo && x < hi) ? c : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      total += __shfl_xor_sync(0xffffffffu, total, o);
      before += __shfl_xor_sync(0xffffffffu, before, o);
      inside += __shfl_xor_sync(0xffffffffu, inside, o);
    }
    if (lane == 0) {
      s_rng[0] = before;
      s_rng[1] = before + inside;
      s_rng[2] = total;
    }
  }
  __syncthreads();
  const int us = s_rng[0], ue = s_rng[1];
  if (ue <= us) return;  // empty segment
  const dev::UnitSplit split(static_cast<unsigned>(s_rng[2]), static_cast<unsigned>(s.attend_ctas));
  const int c0 = static_cast<int>(split.owner(us)), c1 = static_cast<int>(split.owner(ue - 1));
  if (c0 == c1) return;  // written by its only attention CTA
  dev::pdl_wait();  // the partials are complete from here on
  if (threadIdx.x == 0) dev::trace_first(a.trace, ETA_TRACE_MERGE_FIRST);

  const int PS = partial_stride(s.d);
  const size_t cstride = static_cast<size_t>(s.G) * PS;
  const float* col = a.partials + static_cast<size_t>(seg) * cstride + static_cast<size_t>(h) * PS;
  const int e = slice * 32 + lane;
  const int span = c1 - c0 + 1;

  float mx = -INFINITY, ls = 0.f, acc = 0.f;
  for (int k0 = w; k0 < span; k0 += kMergeWarps * kBatch) {
    float m[kBatch], l[kBatch], x[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int k = min(k0 + u * kMergeWarps, span - 1);
      const float* p = col + static_cast<size_t>(c0 + k) * cstride;
      m[u] = __ldcg(p + s.d);
      l[u] = __ldcg(p + s.d + 1);
      x[u] = __ldcg(p + e);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int k = k0 + u * kMergeWarps;
      // an unused slot may hold any bits: skip it rather than weight it by 0
      if (k >= span || !split.owns_any(c0 + k) || m[u] == -INFINITY) continue;
      if (m[u] > mx) {
        const float f = (mx == -INFINITY) ? 0.f : dev::fast_exp2(mx - m[u]);
        ls = fmaf(ls, f, l[u]);
        acc = fmaf(acc, f, x[u]);
        mx = m[u];
      } else {
        const float f = dev::fast_exp2(m[u] - mx);
        ls = fmaf(l[u], f, ls);
        acc = fmaf(x[u], f, acc);
      }
    }
  }
  __shared__ float s_m[kMergeWarps], s_l[kMergeWarps], s_acc[kMergeWarps][32];
  if (lane == 0) {
    s_m[w] = mx;
    s_l[w] = ls;
  }
  s_acc[w][lane] = acc;
  __syncthreads();
  if (w == 0) {
    float mstar = -INFINITY;
    for (int k = 0; k < kMergeWarps; ++k) mstar = fmaxf(mstar, s_m[k]);
    float lsum = 0.f, asum = 0.f;
    if (mstar != -INFINITY) {
      for (int k = 0; k < kMergeWarps; ++k) {
        if (s_m[k] == -INFINITY) continue;
        const float f = dev::fast_exp2(s_m[k] - mstar);
        lsum = fmaf(s_l[k], f, lsum);
        asum = fmaf(s_acc[k][lane], f, asum);
      }
    }
    const int i = seg / s.Hkv, g = seg - i * s.Hkv;
    const size_t orow = static_cast<size_t>(i) * s.Hq + g * s.G + h;
    dev::store_out_slot(a.out, s.elt, orow * s.d + e, lsum > 0.f ? asum / lsum : 0.f);
    if (lane == 0 && slice == 0 && a.lse) a.lse[orow] = dev::lse_of(mstar, lsum);
    if (lane == 0) dev::trace_last(a.trace, ETA_TRACE_MERGE_LAST);
  }
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.s.nseg * a.s.G, a.s.d / 32);
  cfg.blockDim = dim3(kMergeWarps * 32);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, merge_kernel, a);
}

}  // namespace eta
