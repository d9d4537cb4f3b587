// Offline per-head threshold calibration (section 4.7 and Appendix D.2 of
// Elastic Threshold Attention): a weighted histogram of every causal logit
// S_tj = scale q_t . k_j (j <= t) of each query head, each entry weighted by
// 1/(t + 1) so that every query row carries weight 1; the frozen constant of
// a head is then the logit at which the weighted fraction at or above it
// equals the head's target density (host-side solver below).
//
// Grid (query tiles of 64, query heads, sequences); each CTA stages its 64
// query rows and, in turn, every key tile up to the diagonal in shared memory
// (fp32, rows padded against bank conflicts), computes the 64 x 64 logits
// with a 4 x 4 register tile per thread on the CUDA cores, bins them into a
// shared-memory histogram and adds that to the head's global histogram (fp64)
// once at the end.  An offline tool, not on the decode path: plain SIMT.
#include <math.h>

#include "eta_device.cuh"

namespace eta {
namespace {

constexpr int kTile = 64;
constexpr int kThreads = 256;

__host__ __device__ inline size_t calib_smem_bytes(int d, int nbins) {
  return (2 * static_cast<size_t>(kTile) * (d + 1) + (nbins + 2)) * sizeof(float);
}

__global__ void __launch_bounds__(kThreads) calib_hist_kernel(CalibArgs a) {
  extern __shared__ float sm[];
  const int d = a.d, P = d + 1;
  float* sq = sm;                 // [64][d + 1] query rows
  float* sk = sq + kTile * P;     // [64][d + 1] key rows
  float* sh = sk + kTile * P;     // [nbins + 2] weights
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int g = h / a.G;
  const int q0 = qt * kTile;
  const int t = threadIdx.x;
  for (int x = t; x < a.nbins + 2; x += kThreads) sh[x] = 0.f;
  const size_t qbase = (static_cast<size_t>(b) * a.Hq + h) * a.T;
  for (int x = t; x < kTile * d; x += kThreads) {
    const int r = x / d, e = x - r * d;
    sq[r * P + e] = q0 + r < a.T ? dev::load_elt(a.q, (qbase + q0 + r) * d + e, a.elt) : 0.f;
  }
  const size_t kbase = (static_cast<size_t>(b) * a.Hkv + g) * a.kv_stride;
  const int ty = t >> 4, tx = t & 15;  // rows 4 ty .. 4 ty + 3, keys 4 tx .. 4 tx + 3
  for (int kt = 0; kt <= qt; ++kt) {
    __syncthreads();  // previous key tile consumed (and the query tile / histogram ready)
    for (int x = t; x < kTile * d; x += kThreads) {
      const int r = x / d, e = x - r * d;
      const int j = kt * kTile + r;
      sk[r * P + e] = j < a.T ? dev::load_elt(a.k, (kbase + j) * d + e, a.elt) : 0.f;
    }
    __syncthreads();
    float acc[4][4] = {};
    for (int e = 0; e < d; ++e) {
      float qv[4], kv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qv[u] = sq[(4 * ty + u) * P + e];
        kv[u] = sk[(4 * tx + u) * P + e];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(qv[u], kv[v], acc[u][v]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int tq = q0 + 4 * ty + u;
      if (tq >= a.T) continue;
      const float wgt = 1.f / static_cast<float>(tq + 1);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int j = kt * kTile + 4 * tx + v;
        if (j > tq) continue;
        const float s = acc[u][v] * a.scale;
        const float f = floorf((s - a.lo) * a.inv_width);
        const int bin = f < -1.f ? -1 : (f > static_cast<float>(a.nbins) ? a.nbins : static_cast<int>(f));
        atomicAdd(&sh[bin + 1], wgt);
      }
    }
  }
  __syncthreads();
  double* out = a.hist + static_cast<size_t>(h) * (a.nbins + 2);
  for (int x = t; x < a.nbins + 2; x += kThreads)
    if (sh[x] != 0.f) atomicAdd(&out[x], static_cast<double>(sh[x]));
}

}  // namespace

size_t calib_smem(int d, int nbins) { return calib_smem_bytes(d, nbins); }

cudaError_t launch_calib(const CalibArgs& a, cudaStream_t st) {
  const size_t smem = calib_smem_bytes(a.d, a.nbins);
  static SmemLimit lim;
  const dim3 grid((a.T + kTile - 1) / kTile, a.Hq, a.B);
  return launch_with_smem(reinterpret_cast<const void*>(calib_hist_kernel), smem, lim, [&] {
    calib_hist_kernel<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
  });
}

}  // namespace eta
