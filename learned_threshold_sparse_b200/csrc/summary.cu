// Block metadata refresh (per block, per KV head): centroid mu_B and
// coordinate standard deviation sigma_B stored in fp16, maximum norm M_B of
// the block's keys around the stored centroid in fp32, rounded up.
// Source: Elastic Threshold Attention, Appendix F.1 (compact metadata layout)
// and section 3.2; recomputed for the blocks an append touched.
#include "eta_device.cuh"

namespace eta {
namespace {

constexpr int kThreads = 128;

// One CTA per touched block.  Pass 1: mean per coordinate; pass 2: population
// variance around the fp32 mean; pass 3: max over rows of ||k - mu_hat||^2.
// All accumulation in fp32 (Appendix F.2 promotes squares and dot products to
// fp32).
__global__ void __launch_bounds__(kThreads) summary_kernel(SummaryArgs a) {
  const int i = blockIdx.z, g = blockIdx.y;
  int T = a.seq_lens[i];
  T = T < 0 ? 0 : (T > a.max_ctx ? a.max_ctx : T);
  const int nb = (T + a.b - 1) / a.b;
  int ft = a.first_token[i];
  ft = ft < 0 ? 0 : ft;
  const int j = ft / a.b + static_cast<int>(blockIdx.x);
  if (j >= nb) return;
  const int r0 = j * a.b;
  const int n = min(a.b, T - r0);
  const size_t row0 = (static_cast<size_t>(i) * a.Hkv + g) * a.max_ctx + r0;
  const int d = a.d;
  const int t = threadIdx.x;

  __shared__ float s_mu[128];
  __shared__ float s_wmax[kThreads / 32];

  if (t < d) {
    float sum = 0.f;
    for (int r = 0; r < n; ++r) sum += dev::load_elt(a.k, (row0 + r) * d + t, a.elt);
    const float mean = sum / static_cast<float>(n);
    float ss = 0.f;
    for (int r = 0; r < n; ++r) {
      const float x = dev::load_elt(a.k, (row0 + r) * d + t, a.elt) - mean;
      ss = fmaf(x, x, ss);
    }
    const float sd = sqrtf(ss / static_cast<float>(n));
    const uint16_t mu_h = dev::f32_to_fp16_rn(mean);
    const size_t mo = ((static_cast<size_t>(i) * a.Hkv + g) * a.nbmax + j) * d + t;
    a.mu[mo] = mu_h;
    a.sigma[mo] = dev::f32_to_fp16_rn(sd);
    s_mu[t] = dev::fp16_to_f32(mu_h);
  }
  __syncthreads();

  // M_B: warp w takes rows w, w+4, ...; lanes split the coordinates.
  const int w = t >> 5, lane = t & 31;
  float best = 0.f;
  for (int r = w; r < n; r += kThreads / 32) {
    float ss = 0.f;
    for (int e = lane; e < d; e += 32) {
      const float x = dev::load_elt(a.k, (row0 + r) * d + e, a.elt) - s_mu[e];
      ss = fmaf(x, x, ss);
    }
    ss = dev::warp_sum(ss);
    best = fmaxf(best, ss);
  }
  if (lane == 0) s_wmax[w] = best;
  __syncthreads();
  if (t == 0) {
    float m2 = s_wmax[0];
    for (int k = 1; k < kThreads / 32; ++k) m2 = fmaxf(m2, s_wmax[k]);
    // fp32 rounding of d squares and a 5-level tree is below 16 ulp; the
    // directed roundings and the 2^-18 inflation keep M_B >= the exact norm.
    const float m = __fmul_ru(__fsqrt_ru(m2), 1.0f + 3.814697265625e-06f);
    a.max_norm[(static_cast<size_t>(i) * a.Hkv + g) * a.nbmax + j] = m;
  }
}

}  // namespace

cudaError_t launch_summary(const SummaryArgs& a, cudaStream_t st) {
  dim3 grid(a.max_blocks, a.Hkv, a.B);
  summary_kernel<<<grid, kThreads, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace eta
