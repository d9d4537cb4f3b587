// Block metadata refresh (per block, per KV head): centroid mu_B and
// coordinate standard deviation sigma_B stored in fp16 (or as e4m3 codes with
// one fp32 scale per block and field), maximum norm M_B of the block's keys
// around the stored (dequantised) centroid in fp32, rounded up.
// Source: Elastic Threshold Attention, Appendix F.1 (compact metadata layout)
// and section 3.2; recomputed for the blocks an append touched.  The FP8
// format follows section 5's FP8 metadata extension (format: this library's).
//
// Two kernels: summary_kernel refreshes a range of blocks per sequence;
// append_kernel writes one new token per (sequence, KV head) into the cache
// and refreshes the block that holds it, in one launch.
#include "eta_device.cuh"

namespace eta {
namespace {

constexpr int kThreads = 128;

__host__ __device__ inline size_t block_stage_bytes(int b, int d, int elt) {
  return static_cast<size_t>(b) * d * elt;
}

// One e4m3 code (nearest, ties to even, saturating at +-448).
__device__ __forceinline__ uint8_t f32_to_e4m3(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.f), "f"(x));
  return static_cast<uint8_t>(r & 0xffu);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(code)));
  return dev::fp16_to_f32(static_cast<uint16_t>(h2 & 0xffffu));
}

// Largest of v over the CTA's threads (kThreads), in every thread.
__device__ __forceinline__ float cta_max(float v, float* s_w) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();  // s_w free from any earlier use
  if ((threadIdx.x & 31) == 0) s_w[w] = v;
  __syncthreads();
  float m = s_w[0];
  for (int k = 1; k < kThreads / 32; ++k) m = fmaxf(m, s_w[k]);
  return m;
}

// Summary of block j of (sequence i, KV head g) over its n present rows,
// staged once in shared memory (raw K bytes).  Pass 1: mean per coordinate;
// pass 2: population variance around the fp32 mean; pass 3: max over rows of
// ||k - mu~||^2 with mu~ the stored centroid.  All accumulation in fp32
// (Appendix F.2 promotes squares and dot products to fp32).  In the FP8
// format every step is one correctly rounded fp32 operation in row order
// (no contraction), the scale maps the largest magnitude to 448 and the code
// is the nearest e4m3 value, so the codes are reproducible exactly.
template <int FMT>
__device__ void summarize_block(const SummaryArgs& a, int i, int g, int j, int n, uint8_t* stage) {
  const int d = a.d, t = threadIdx.x;
  const KvLayout lay{a.block_table, a.Hkv, a.b, a.max_ctx, a.nbmax, a.num_pages};
  bool bad = false;
  const size_t row0 = static_cast<size_t>(lay.row(i * a.Hkv + g, j, &bad));
  if (bad) return;  // a page id outside the pool: nothing is read or written (CTA-uniform)
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.k) + row0 * d * a.elt);
  const int nvec = n * d * a.elt / 16;
  for (int x = t; x < nvec; x += kThreads) reinterpret_cast<uint4*>(stage)[x] = src[x];
  __shared__ float s_mu[128];
  __shared__ float s_wmax[kThreads / 32];
  __syncthreads();
  auto at = [&](int r, int e) -> float {
    const size_t idx = static_cast<size_t>(r) * d + e;
    if (a.elt == 4) return reinterpret_cast<const float*>(stage)[idx];
    return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(stage)[idx]) << 16);
  };
  const size_t bo = (static_cast<size_t>(i) * a.Hkv + g) * a.nbmax + j;  // block index
  if (FMT == ETA_META_BOX) {
    // per-coordinate extrema, fp16 rounded outward (the box bound stays strict)
    if (t < d) {
      float lo = at(0, t), hi = lo;
      for (int r = 1; r < n; ++r) {
        const float x = at(r, t);
        lo = fminf(lo, x);
        hi = fmaxf(hi, x);
      }
      uint16_t l16, h16;
      asm("cvt.rm.f16.f32 %0, %1;" : "=h"(l16) : "f"(lo));
      asm("cvt.rp.f16.f32 %0, %1;" : "=h"(h16) : "f"(hi));
      static_cast<uint16_t*>(a.mu)[bo * d + t] = l16;
      static_cast<uint16_t*>(a.sigma)[bo * d + t] = h16;
    }
    if (t == 0) a.max_norm[bo] = 0.f;
    return;
  }
  if (FMT == ETA_META_FP16) {
    if (t < d) {
      float sum = 0.f;
      for (int r = 0; r < n; ++r) sum += at(r, t);
      const float mean = sum / static_cast<float>(n);
      float ss = 0.f;
      for (int r = 0; r < n; ++r) {
        const float x = at(r, t) - mean;
        ss = fmaf(x, x, ss);
      }
      const float sd = sqrtf(ss / static_cast<float>(n));
      const uint16_t mu_h = dev::f32_to_fp16_rn(mean);
      static_cast<uint16_t*>(a.mu)[bo * d + t] = mu_h;
      static_cast<uint16_t*>(a.sigma)[bo * d + t] = dev::f32_to_fp16_rn(sd);
      s_mu[t] = dev::fp16_to_f32(mu_h);
    }
  } else {
    float mean = 0.f, sd = 0.f;
    if (t < d) {
      float sum = 0.f;
      for (int r = 0; r < n; ++r) sum = __fadd_rn(sum, at(r, t));
      mean = __fdiv_rn(sum, static_cast<float>(n));
      float ss = 0.f;
      for (int r = 0; r < n; ++r) {
        const float x = __fsub_rn(at(r, t), mean);
        ss = __fadd_rn(ss, __fmul_rn(x, x));
      }
      sd = __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(n)));
    }
    const float mmax = cta_max(fabsf(mean), s_wmax);
    const float smax = cta_max(sd, s_wmax);
    const float mu_scale = mmax > 0.f ? __fdiv_rn(mmax, 448.f) : 1.f;
    const float sd_scale = smax > 0.f ? __fdiv_rn(smax, 448.f) : 1.f;
    if (t < d) {
      const uint8_t mc = f32_to_e4m3(__fdiv_rn(mean, mu_scale));
      const uint8_t sc = f32_to_e4m3(__fdiv_rn(sd, sd_scale));
      static_cast<uint8_t*>(a.mu)[bo * d + t] = mc;
      static_cast<uint8_t*>(a.sigma)[bo * d + t] = sc;
      s_mu[t] = __fmul_rn(e4m3_to_f32(mc), mu_scale);
    }
    if (t == 0) {
      a.mu_scale[bo] = mu_scale;
      a.sigma_scale[bo] = sd_scale;
    }
  }
  __syncthreads();
  // M_B: warp w takes rows w, w+4, ...; lanes split the coordinates.
  const int w = t >> 5, lane = t & 31;
  float best = 0.f;
  for (int r = w; r < n; r += kThreads / 32) {
    float ss = 0.f;
    for (int e = lane; e < d; e += 32) {
      const float x = at(r, e) - s_mu[e];
      ss = fmaf(x, x, ss);
    }
    best = fmaxf(best, dev::warp_sum(ss));
  }
  if (lane == 0) s_wmax[w] = best;
  __syncthreads();
  if (t == 0) {
    float m2 = s_wmax[0];
    for (int k = 1; k < kThreads / 32; ++k) m2 = fmaxf(m2, s_wmax[k]);
    // fp32 rounding of d squares and a 5-level tree is below 16 ulp; the
    // directed roundings and the 2^-18 inflation keep M_B >= the exact norm.
    const float m = __fmul_ru(__fsqrt_ru(m2), 1.0f + 3.814697265625e-06f);
    a.max_norm[bo] = m;
  }
}

__device__ __forceinline__ int clamp_len(int T, int max_ctx) { return T < 0 ? 0 : (T > max_ctx ? max_ctx : T); }

// One CTA per touched block.
template <int FMT>
__global__ void __launch_bounds__(kThreads) summary_kernel(SummaryArgs a) {
  extern __shared__ __align__(16) uint8_t stage[];
  const int i = blockIdx.z, g = blockIdx.y;
  const int T = clamp_len(a.seq_lens[i], a.max_ctx);
  const int nb = (T + a.b - 1) / a.b;
  int ft = a.first_token[i];
  ft = ft < 0 ? 0 : ft;
  const int j = ft / a.b + static_cast<int>(blockIdx.x);
  if (j >= nb) return;
  summarize_block<FMT>(a, i, g, j, min(a.b, T - j * a.b), stage);
}

// One CTA per (KV head, sequence): write the new token's K and V rows at
// position pos[i], then refresh the block holding it over the rows present
// (seq_lens[i] already counts the new token).  A position outside
// [0, max_ctx) writes nothing.  With q_src set, the CTA also copies the
// token's G query rows of this KV head to q_dst.  The new rows are loaded
// with .cv: they may sit in page-locked host memory that the host rewrites
// between launches.
template <int FMT>
__global__ void __launch_bounds__(kThreads) append_kernel(SummaryArgs a, const void* k_new, const void* v_new,
                                                          const int* pos, void* k_cache, void* v_cache) {
  extern __shared__ __align__(16) uint8_t stage[];
  const int g = blockIdx.x, i = blockIdx.y;
  const int d = a.d, t = threadIdx.x;
  // The decode's screen may be scheduled now: it waits for this grid's
  // completion before it reads anything.
  dev::pdl_trigger();
  // Every load of the new rows is issued before the first use, so rows in
  // host memory cost one round trip: a K and a V vector per thread
  // (d * elt / 16 <= 32 vectors per row) and up to kQv query vectors
  // (G * d * elt / 16 <= 256 = kQv * kThreads).
  constexpr int kQv = 2;
  const int nvec = d * a.elt / 16;
  const size_t src = (static_cast<size_t>(i) * a.Hkv + g) * d;
  uint4 kr = make_uint4(0u, 0u, 0u, 0u), vr = kr, qr[kQv];
  if (t < nvec) {
    kr = __ldcv(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(k_new) + src * a.elt) + t);
    vr = __ldcv(reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(v_new) + src * a.elt) + t);
  }
  const size_t q0 = (static_cast<size_t>(i) * a.Hkv * a.G + static_cast<size_t>(g) * a.G) * d * a.elt / 16;
  const int qv = a.q_src ? a.G * d * a.elt / 16 : 0;
#pragma unroll
  for (int u = 0; u < kQv; ++u) {
    const int x = t + u * kThreads;
    if (x < qv) qr[u] = __ldcv(reinterpret_cast<const uint4*>(a.q_src) + q0 + x);
  }
  const int p = pos[i];
#pragma unroll
  for (int u = 0; u < kQv; ++u) {
    const int x = t + u * kThreads;
    if (x < qv) reinterpret_cast<uint4*>(a.q_dst)[q0 + x] = qr[u];
  }
  if (p < 0 || p >= a.max_ctx) return;
  const KvLayout lay{a.block_table, a.Hkv, a.b, a.max_ctx, a.nbmax, a.num_pages};
  bool bad = false;
  const long long brow = lay.row(i * a.Hkv + g, p / a.b, &bad);
  if (bad) return;  // a page id outside the pool: nothing is written
  const size_t dst = (static_cast<size_t>(brow) + p % a.b) * d;
  if (t < nvec) {
    reinterpret_cast<uint4*>(static_cast<uint8_t*>(k_cache) + dst * a.elt)[t] = kr;
    reinterpret_cast<uint4*>(static_cast<uint8_t*>(v_cache) + dst * a.elt)[t] = vr;
  }
  __syncthreads();  // the new row is read back by the block summary below
  const int T = clamp_len(a.seq_lens[i], a.max_ctx);
  const int j = p / a.b;
  if (j * a.b >= T) return;
  summarize_block<FMT>(a, i, g, j, min(a.b, T - j * a.b), stage);
}

}  // namespace

cudaError_t launch_summary(const SummaryArgs& a, cudaStream_t st) {
  const size_t smem = block_stage_bytes(a.b, a.d, a.elt);
  auto go = [&](auto kern, SmemLimit& lim) {
    return launch_with_smem(reinterpret_cast<const void*>(kern), smem, lim, [&] {
      kern<<<dim3(a.max_blocks, a.Hkv, a.B), kThreads, smem, st>>>(a);
      return cudaGetLastError();
    });
  };
  static SmemLimit lim16, lim8, limb;
  if (a.fmt == ETA_META_BOX) return go(summary_kernel<ETA_META_BOX>, limb);
  return a.fmt == ETA_META_FP8 ? go(summary_kernel<ETA_META_FP8>, lim8) : go(summary_kernel<ETA_META_FP16>, lim16);
}

cudaError_t launch_append(const SummaryArgs& a, const void* k_new, const void* v_new, const int* pos,
                          void* k_cache, void* v_cache, cudaStream_t st) {
  const size_t smem = block_stage_bytes(a.b, a.d, a.elt);
  auto go = [&](auto kern, SmemLimit& lim) {
    return launch_with_smem(reinterpret_cast<const void*>(kern), smem, lim, [&] {
      kern<<<dim3(a.Hkv, a.B), kThreads, smem, st>>>(a, k_new, v_new, pos, k_cache, v_cache);
      return cudaGetLastError();
    });
  };
  static SmemLimit lim16, lim8, limb;
  if (a.fmt == ETA_META_BOX) return go(append_kernel<ETA_META_BOX>, limb);
  return a.fmt == ETA_META_FP8 ? go(append_kernel<ETA_META_FP8>, lim8) : go(append_kernel<ETA_META_FP16>, lim16);
}

}  // namespace eta
