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

constexpr int kThreads = 256;        // summary_kernel: many blocks, many CTAs
constexpr int kAppendThreads = 256;   // append_kernel: one block per CTA (1024 measured no faster)

__host__ __device__ inline size_t block_stage_bytes(int b, int d, int elt) {
  return static_cast<size_t>(b) * d * elt;
}

// Nearest e4m3 code of a float64 value, from the format's definition (sign
// bit, 4 exponent bits with bias 7, 3 fraction bits, subnormal step 2^-9):
// ties to the even code, saturating at +-448; a negative value that rounds
// to zero keeps its sign (code 0x80).
__device__ __forceinline__ uint8_t f64_to_e4m3(double x) {
  const double a = fmin(fabs(x), 448.0);
  int code;
  if (a < 0.015625) {
    code = static_cast<int>(rint(a * 512.0));  // multiples of 2^-9; 8 is 2^-6 (code 0x08)
  } else {
    // a = m 2^e with m in [1, 2) and -6 <= e <= 8 (a normal double)
    int e = static_cast<int>((__double_as_longlong(a) >> 52) & 0x7ff) - 1023;
    const double m8 = a * __longlong_as_double(static_cast<long long>(1023 + 3 - e) << 52);  // m * 8, exact
    double q = rint(m8);  // 8..16: the mantissa to 3 fraction bits, ties to even
    if (q == 16.0) {
      q = 8.0;
      ++e;
    }
    code = (e + 7) * 8 + static_cast<int>(q) - 8;
  }
  code = min(code, 0x7E);
  return static_cast<uint8_t>(signbit(x) ? (code | 0x80) : code);
}

__device__ __forceinline__ uint16_t f64_to_fp16_rn(double x) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(x));
  return h;
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t code) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(static_cast<uint16_t>(code)));
  return dev::fp16_to_f32(static_cast<uint16_t>(h2 & 0xffffu));
}

// Largest of v over the CTA's NT threads, in every thread.
template <int NT>
__device__ __forceinline__ double cta_max(double v, double* s_w) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  const int w = threadIdx.x >> 5;
  __syncthreads();  // s_w free from any earlier use
  if ((threadIdx.x & 31) == 0) s_w[w] = v;
  __syncthreads();
  double m = s_w[0];
  for (int k = 1; k < NT / 32; ++k) m = fmax(m, s_w[k]);
  return m;
}

// Summary of block j of (sequence i, KV head g) over its n present rows,
// staged once in shared memory (raw K bytes).  Every statistic is evaluated
// in float64 from the exact inputs: pass 1 the mean per coordinate, pass 2
// the population variance around it, pass 3 the largest distance of a row
// from the stored (dequantised) centroid.  The stored values are then the
// correctly rounded statistics: fp16 (nearest) for the centroid and spread;
// in the FP8 format the fp32 scale nearest to (largest magnitude) / 448 and
// the e4m3 code nearest to statistic / scale; M rounded up to fp32 after an
// inflation that covers the float64 rounding of the distance, so that it
// never falls below the exact distance.  With sums of at most 128 bf16 rows
// (or fp32 rows of moderate range) the float64 sums are exact, so the stored
// metadata does not depend on the summation order.
//
// NT threads per CTA: the more, the shorter every thread's dependent chain
// (passes 1 and 2 split the rows into NT / d groups, pass 3 gives each row
// NT / n lanes).  DC, EC: the head dimension and element size when known at
// compile time (0: taken from the arguments), so that the index arithmetic
// of the common case folds to shifts and masks.
template <int FMT, int NT, int DC = 0, int EC = 0>
__device__ void summarize_block(const SummaryArgs& a, int i, int g, int j, int n, uint8_t* stage) {
  const int d = DC > 0 ? DC : a.d, elt = EC > 0 ? EC : a.elt, t = threadIdx.x;
  const KvLayout lay{a.block_table, a.Hkv, a.b, a.max_ctx, a.nbmax, a.num_pages};
  bool bad = false;
  const size_t row0 = static_cast<size_t>(lay.row(i * a.Hkv + g, j, &bad));
  if (bad) return;  // a page id outside the pool: nothing is read or written (CTA-uniform)
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(a.k) + row0 * d * elt);
  const int nvec = n * d * elt / 16;
  // all of a thread's loads in flight before its stores (one round trip)
  for (int x0 = t; x0 < nvec; x0 += 8 * NT) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (x0 + u * NT < nvec) v[u] = src[x0 + u * NT];
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (x0 + u * NT < nvec) reinterpret_cast<uint4*>(stage)[x0 + u * NT] = v[u];
  }
  __shared__ double s_mu[128];
  __shared__ double s_part[NT];
  __shared__ double s_wmax[NT / 32];
  __syncthreads();
  auto at = [&](int r, int e) -> float {
    const size_t idx = static_cast<size_t>(r) * d + e;
    if (elt == 4) return reinterpret_cast<const float*>(stage)[idx];
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
  // Passes 1 and 2: the threads split into NT / d row groups, each
  // thread one coordinate over its group's rows (four interleaved partial
  // sums), the groups' partials added in shared memory.  The pass-1 sums of
  // bf16 (or moderate fp32) rows are exact in float64, so the mean does not
  // depend on how the rows are split.
  const int ngroups = NT / d > 0 ? NT / d : 1;
  const int e_own = t % d, grp = t / d;
  const bool active = grp < ngroups && e_own < d;
  // sum over the thread's rows grp, grp + ngroups, ...: four interleaved
  // partial sums, the rows past the last full group of four into the first
  auto group_sum = [&](auto&& term) -> double {  // term(r): row r's term
    double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
    if (active) {
      int r = grp;
      for (; r + 3 * ngroups < n; r += 4 * ngroups) {
        s0 += term(r);
        s1 += term(r + ngroups);
        s2 += term(r + 2 * ngroups);
        s3 += term(r + 3 * ngroups);
      }
      for (; r < n; r += ngroups) s0 += term(r);
    }
    return (s0 + s1) + (s2 + s3);
  };
  auto val = [&](int r) -> float { return at(r, e_own); };
  double mean = 0.0, sd = 0.0;
  {
    const double part = group_sum([&](int r) { return static_cast<double>(val(r)); });
    if (active) s_part[t] = part;
    __syncthreads();
    if (t < d) {
      double tot = 0.0;
      for (int g2 = 0; g2 < ngroups; ++g2) tot += s_part[g2 * d + t];
      s_mu[t] = tot / static_cast<double>(n);  // the exact mean, for pass 2
    }
    __syncthreads();
    const double m_own = active ? s_mu[e_own] : 0.0;
    const double sq = group_sum([&](int r) {
      const double x = static_cast<double>(val(r)) - m_own;
      return x * x;
    });
    __syncthreads();  // every thread has read s_mu and s_part
    if (active) s_part[t] = sq;
    __syncthreads();
    if (t < d) {
      double tot = 0.0;
      for (int g2 = 0; g2 < ngroups; ++g2) tot += s_part[g2 * d + t];
      mean = s_mu[t];
      sd = sqrt(tot / static_cast<double>(n));
    }
    __syncthreads();  // s_mu is rewritten with the stored centroid below
  }
  if (FMT == ETA_META_FP16) {
    if (t < d) {
      const uint16_t mu_h = f64_to_fp16_rn(mean);
      static_cast<uint16_t*>(a.mu)[bo * d + t] = mu_h;
      static_cast<uint16_t*>(a.sigma)[bo * d + t] = f64_to_fp16_rn(sd);
      s_mu[t] = static_cast<double>(dev::fp16_to_f32(mu_h));
    }
  } else {
    const double mmax = cta_max<NT>(fabs(mean), s_wmax);
    const double smax = cta_max<NT>(sd, s_wmax);
    const float mu_scale = mmax > 0.0 ? __double2float_rn(mmax / 448.0) : 1.f;
    const float sd_scale = smax > 0.0 ? __double2float_rn(smax / 448.0) : 1.f;
    if (t < d) {
      const uint8_t mc = f64_to_e4m3(mean / static_cast<double>(mu_scale));
      const uint8_t sc = f64_to_e4m3(sd / static_cast<double>(sd_scale));
      static_cast<uint8_t*>(a.mu)[bo * d + t] = mc;
      static_cast<uint8_t*>(a.sigma)[bo * d + t] = sc;
      s_mu[t] = static_cast<double>(e4m3_to_f32(mc)) * static_cast<double>(mu_scale);  // exact
    }
    if (t == 0) {
      a.mu_scale[bo] = mu_scale;
      a.sigma_scale[bo] = sd_scale;
    }
  }
  __syncthreads();
  // Pass 3, M_B: tpr consecutive lanes per row (the most that fit the CTA,
  // up to a warp), each summing a share of the coordinates, visited in an
  // order skewed by the row so that the lanes of different rows read
  // different shared-memory banks; the row's partial sums are added by
  // shuffles and the largest row is taken over the CTA.  The differences
  // k - mu~ are exact in float64 and the sum of d squares has a relative
  // error below 2^-48, which the 2^-47 inflation (rounded up) covers before
  // the upward rounding to fp32.
  const int w = t >> 5, lane = t & 31;
  constexpr int kW = NT / 32;
  int tpr = 1;
  while (tpr < 32 && 2 * tpr * n <= NT) tpr *= 2;
  const int sub = t % tpr, per = d / tpr;
  double best = 0.0;
  for (int r0 = 0; r0 < n; r0 += NT / tpr) {  // the same trip count in every lane
    const int r = r0 + t / tpr;
    double rs = 0.0;
    if (r < n) {
      auto sq = [&](int k) {
        const int e = (sub + tpr * k + 2 * r) % d;
        const double x = static_cast<double>(at(r, e)) - s_mu[e];
        return x * x;
      };
      double q0 = 0.0, q1 = 0.0, q2 = 0.0, q3 = 0.0;
      int k = 0;
      for (; k + 4 <= per; k += 4) {
        q0 += sq(k);
        q1 += sq(k + 1);
        q2 += sq(k + 2);
        q3 += sq(k + 3);
      }
      for (; k < per; ++k) q0 += sq(k);
      rs = (q0 + q1) + (q2 + q3);
    }
    for (int o = 1; o < tpr; o <<= 1) rs += __shfl_xor_sync(0xffffffffu, rs, o);
    if (r < n) best = fmax(best, rs);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) best = fmax(best, __shfl_xor_sync(0xffffffffu, best, o));
  if (lane == 0) s_wmax[w] = best;
  __syncthreads();
  if (t == 0) {
    double m2 = s_wmax[0];
    for (int k = 1; k < kW; ++k) m2 = fmax(m2, s_wmax[k]);
    const double m = __dmul_ru(sqrt(m2), 1.0 + 0x1p-47);
    float mf;
    asm("cvt.rp.f32.f64 %0, %1;" : "=f"(mf) : "d"(m));
    a.max_norm[bo] = mf;
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
  const int n = min(a.b, T - j * a.b);
  if (a.d == 128 && a.elt == 2) summarize_block<FMT, kThreads, 128, 2>(a, i, g, j, n, stage);
  else summarize_block<FMT, kThreads>(a, i, g, j, n, stage);
}

// One CTA per (KV head, sequence): write the new token's K and V rows at
// position pos[i], then refresh the block holding it over the rows present
// (seq_lens[i] already counts the new token).  A position outside
// [0, max_ctx) writes nothing.  With q_src set, the CTA also copies the
// token's G query rows of this KV head to q_dst.  The new rows are loaded
// with .cv: they may sit in page-locked host memory that the host rewrites
// between launches.
template <int FMT>
__global__ void __launch_bounds__(kAppendThreads) append_kernel(SummaryArgs a, const void* k_new, const void* v_new,
                                                          const int* pos, void* k_cache, void* v_cache) {
  extern __shared__ __align__(16) uint8_t stage[];
  const int g = blockIdx.x, i = blockIdx.y;
  const int d = a.d, t = threadIdx.x;
  if (t == 0) dev::trace_first(a.trace, ETA_TRACE_APPEND_FIRST);
  // Every load of the new rows is issued before the first use, so rows in
  // host memory cost one round trip: a K and a V vector per thread
  // (d * elt / 16 <= 32 vectors per row) and up to kQv query vectors
  // (G * d * elt / 16 <= 256 <= kQv * kAppendThreads).
  constexpr int kQv = 1;
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
    const int x = t + u * kAppendThreads;
    if (x < qv) qr[u] = __ldcv(reinterpret_cast<const uint4*>(a.q_src) + q0 + x);
  }
  const int p = pos[i];
#pragma unroll
  for (int u = 0; u < kQv; ++u) {
    const int x = t + u * kAppendThreads;
    if (x < qv) reinterpret_cast<uint4*>(a.q_dst)[q0 + x] = qr[u];
  }
  if (p < 0 || p >= a.max_ctx) {
    if (t == 0) dev::trace_last(a.trace, ETA_TRACE_APPEND_LAST);
    return;
  }
  const KvLayout lay{a.block_table, a.Hkv, a.b, a.max_ctx, a.nbmax, a.num_pages};
  bool bad = false;
  const long long brow = lay.row(i * a.Hkv + g, p / a.b, &bad);
  if (bad) {  // a page id outside the pool: nothing is written
    if (t == 0) dev::trace_last(a.trace, ETA_TRACE_APPEND_LAST);
    return;
  }
  const size_t dst = (static_cast<size_t>(brow) + p % a.b) * d;
  if (t < nvec) {
    reinterpret_cast<uint4*>(static_cast<uint8_t*>(k_cache) + dst * a.elt)[t] = kr;
    reinterpret_cast<uint4*>(static_cast<uint8_t*>(v_cache) + dst * a.elt)[t] = vr;
  }
  __syncthreads();  // the new row is read back by the block summary below
  const int T = clamp_len(a.seq_lens[i], a.max_ctx);
  const int j = p / a.b;
  if (j * a.b < T) {
    const int n = min(a.b, T - j * a.b);
    if (a.d == 128 && a.elt == 2) summarize_block<FMT, kAppendThreads, 128, 2>(a, i, g, j, n, stage);
    else summarize_block<FMT, kAppendThreads>(a, i, g, j, n, stage);
  }
  if (t == 0) dev::trace_last(a.trace, ETA_TRACE_APPEND_LAST);
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
      kern<<<dim3(a.Hkv, a.B), kAppendThreads, smem, st>>>(a, k_new, v_new, pos, k_cache, v_cache);
      return cudaGetLastError();
    });
  };
  static SmemLimit lim16, lim8, limb;
  if (a.fmt == ETA_META_BOX) return go(append_kernel<ETA_META_BOX>, limb);
  return a.fmt == ETA_META_FP8 ? go(append_kernel<ETA_META_FP8>, lim8) : go(append_kernel<ETA_META_FP16>, lim16);
}

}  // namespace eta
