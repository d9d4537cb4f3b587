// Fused threshold projection + block screen + per-chunk compaction.
//
// Source: Elastic Threshold Attention,
//   section 1 / Appendix D.1   tau = w_tau . q + b_tau (learned mode),
//   section 4.7 / Appendix D.2 frozen per-head constants (calibrated mode),
//   Appendix G.1               tau~ = tau - a,
//   section 3.1 / 4.3, App. F.1 per-block bound from (mu_B, sigma_B, M_B)
//                              compared with tau~ for the G heads of a KV head,
//   section 4.8                always-loaded window (lwb blocks + tail block),
//   Appendix F.1 step 2        GQA union: a block is listed once with the
//                              G-bit mask of the heads that admitted it,
//   Appendix F.2               fp32 for squares, <q, mu> and scales.
//
// The bound (its printed form is lost from the pages) is read as
//   Score = scale * (<q, mu> + min(||q|| M, z sqrt(sum_i q_i^2 sigma_i^2))),
// the geometric half alone when z = +inf.
//
// Grid (nchunks, Hkv, B): each CTA screens `chunk` consecutive blocks of one
// (sequence, KV head) -- one warp per block, lanes split the head dimension --
// and writes the admitted blocks of its chunk, ascending, as list entries
// (block id | head mask << 24) plus the chunk's entry count.
#include <math.h>

#include "eta_device.cuh"

namespace eta {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxChunk = 1024;

// Reduce N values held by every lane across all 32 lanes, exchanging half of
// the remaining values per butterfly stage.  Afterwards lane l holds the
// total of value index l / (32 / N) (N a power of two, N <= 32).
template <int N>
__device__ __forceinline__ float transpose_reduce32(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (lane & o) != 0;
      const int half = n >> 1;
#pragma unroll
      for (int j = 0; j < N / 2; ++j) {
        if (j < half) {
          const float send = upper ? v[j] : v[j + half];
          const float keep = upper ? v[j + half] : v[j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
    }
  }
  return v[0];
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads) screen_kernel(ScreenArgs a) {
  constexpr int CPL = D / 32;  // coordinates per lane
  const Shape& s = a.s;
  const int c = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
  const int seg = i * s.Hkv + g;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;

  __shared__ float s_q[G][D];
  __shared__ float s_tau[G];
  __shared__ float s_qn[G];
  __shared__ uint8_t s_mask[kMaxChunk];
  __shared__ int s_wsum[kWarps];
  __shared__ int s_cnt[G];
  __shared__ unsigned long long s_best[G];

  // The attention kernel may be scheduled now; it waits for this grid's
  // completion before reading anything written here.
  dev::pdl_trigger();

  int T = a.seq_lens[i];
  if (T < 0 || T > s.max_ctx) {
    if (t == 0 && c == 0 && g == 0) atomicOr(a.status, kStatusRange);
    T = T < 0 ? 0 : s.max_ctx;
  }
  const int nb = (T + s.b - 1) / s.b;
  const int blk0 = c * s.chunk;
  const int nloc = max(0, min(s.chunk, nb - blk0));

  for (int x = t; x < G * D; x += kThreads) {
    const int h = x / D, e = x - h * D;
    s_q[h][e] = dev::load_elt(a.q, (static_cast<size_t>(i) * s.Hq + g * G + h) * D + e, s.elt);
  }
  if (t < G) {
    s_cnt[t] = 0;
    s_best[t] = 0ull;
  }
  __syncthreads();
  if (w < G) {
    const int hq = g * G + w;
    float tw = 0.f, qq = 0.f;
    for (int e = lane; e < D; e += 32) {
      const float qe = s_q[w][e];
      qq = fmaf(qe, qe, qq);
      if (a.tau_mode == ETA_TAU_LEARNED) tw = fmaf(a.w_tau[static_cast<size_t>(hq) * D + e], qe, tw);
    }
    tw = dev::warp_sum(tw);
    qq = dev::warp_sum(qq);
    const float tau = (a.tau_mode == ETA_TAU_LEARNED ? tw + a.b_tau[hq] : a.c_tau[hq]) - a.offset_a;
    if (lane == 0) {
      s_tau[w] = tau;
      s_qn[w] = sqrtf(qq);
      if (c == 0) a.tau[static_cast<size_t>(i) * s.Hq + hq] = tau;
    }
  }
  __syncthreads();
  if (nloc == 0) {
    if (t == 0) a.chunk_count[static_cast<size_t>(seg) * s.nchunks + c] = 0;
    return;
  }

  float qr[G][CPL], q2[G][CPL];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int k = 0; k < CPL; ++k) {
      qr[h][k] = s_q[h][lane * CPL + k];
      q2[h][k] = qr[h][k] * qr[h][k];
    }
  const float scale = a.scale, z = a.z;
  const bool strict = isinf(z);
  const int first_forced = (!a.screen_enabled) ? 0 : (a.lwb >= 0 ? max(0, nb - 1 - a.lwb) : nb);
  const size_t mbase = (static_cast<size_t>(seg) * s.nbmax) * D;
  const size_t nbase = static_cast<size_t>(seg) * s.nbmax;
  constexpr unsigned kAll = (1u << G) - 1u;

  for (int lb0 = w; lb0 < nloc; lb0 += 4 * kWarps) {
    // four blocks per warp in flight
    uint32_t mu_raw[4][CPL / 2], sg_raw[4][CPL / 2];
    float mn[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int lb = lb0 + u * kWarps;
      const int blk = blk0 + lb;
      if (lb < nloc && blk < first_forced) {
        const uint32_t* pm = reinterpret_cast<const uint32_t*>(a.mu + mbase + static_cast<size_t>(blk) * D + lane * CPL);
        const uint32_t* ps = reinterpret_cast<const uint32_t*>(a.sigma + mbase + static_cast<size_t>(blk) * D + lane * CPL);
        if constexpr (CPL == 4) {
          const uint2 x = *reinterpret_cast<const uint2*>(pm);
          const uint2 y = *reinterpret_cast<const uint2*>(ps);
          mu_raw[u][0] = x.x; mu_raw[u][1] = x.y;
          sg_raw[u][0] = y.x; sg_raw[u][1] = y.y;
        } else {
          mu_raw[u][0] = pm[0];
          sg_raw[u][0] = ps[0];
        }
        mn[u] = a.max_norm[nbase + blk];
      } else {
#pragma unroll
        for (int k = 0; k < CPL / 2; ++k) mu_raw[u][k] = sg_raw[u][k] = 0u;
        mn[u] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int lb = lb0 + u * kWarps;
      if (lb >= nloc) break;
      const int blk = blk0 + lb;
      unsigned m;
      if (blk >= first_forced) {
        m = kAll;
      } else {
        float mu[CPL], s2[CPL];
#pragma unroll
        for (int k = 0; k < CPL / 2; ++k) {
          mu[2 * k] = dev::fp16_to_f32(static_cast<uint16_t>(mu_raw[u][k] & 0xffffu));
          mu[2 * k + 1] = dev::fp16_to_f32(static_cast<uint16_t>(mu_raw[u][k] >> 16));
          const float a0 = dev::fp16_to_f32(static_cast<uint16_t>(sg_raw[u][k] & 0xffffu));
          const float a1 = dev::fp16_to_f32(static_cast<uint16_t>(sg_raw[u][k] >> 16));
          s2[2 * k] = a0 * a0;
          s2[2 * k + 1] = a1 * a1;
        }
        float v[2 * G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float dot = 0.f, sq = 0.f;
#pragma unroll
          for (int k = 0; k < CPL; ++k) {
            dot = fmaf(qr[h][k], mu[k], dot);
            sq = fmaf(q2[h][k], s2[k], sq);
          }
          v[h] = dot;
          v[G + h] = sq;
        }
        const float red = transpose_reduce32<2 * G>(v, lane);
        // lanes [0, 16) hold <q_h, mu> for h = lane / (16 / G); lanes
        // [16, 32) hold the matching sum of q^2 sigma^2.
        const float sq = __shfl_xor_sync(0xffffffffu, red, 16);
        const int hh = (lane & 15) / (16 / G);
        const float geo = s_qn[hh] * mn[u];
        const float spread = strict ? geo : fminf(geo, z * sqrtf(sq));
        const float score = scale * (red + spread);
        const bool pass = (lane < 16) && (lane % (16 / G) == 0) && (score >= s_tau[hh]);
        const unsigned bal = __ballot_sync(0xffffffffu, pass);
        m = 0u;
#pragma unroll
        for (int h = 0; h < G; ++h) m |= ((bal >> (h * (16 / G))) & 1u) << h;
        if (s.rescue && lane < 16 && (lane % (16 / G) == 0)) {
          const unsigned long long key =
              (static_cast<unsigned long long>(dev::float_order_key(score)) << 32) |
              static_cast<unsigned long long>(0xffffffffu - static_cast<unsigned>(blk));
          atomicMax(&s_best[hh], key);
          if (pass) atomicAdd(&s_cnt[hh], 1);
        }
      }
      if (lane == 0) s_mask[lb] = static_cast<uint8_t>(m);
    }
  }
  __syncthreads();

  // Ascending compaction of the chunk's admitted blocks.
  int base = 0;
  int* list = a.chunk_list + static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(c) * s.chunk;
  for (int r0 = 0; r0 < nloc; r0 += kThreads) {
    const int lb = r0 + t;
    const unsigned m = lb < nloc ? s_mask[lb] : 0u;
    const unsigned bal = __ballot_sync(0xffffffffu, m != 0u);
    if (lane == 0) s_wsum[w] = __popc(bal);
    __syncthreads();
    int off = base;
    int tot = 0;
    for (int k = 0; k < kWarps; ++k) {
      if (k < w) off += s_wsum[k];
      tot += s_wsum[k];
    }
    if (m != 0u) {
      off += __popc(bal & ((1u << lane) - 1u));
      list[off] = (blk0 + lb) | static_cast<int>(m << kEntryBlockBits);
    }
    base += tot;
    __syncthreads();
  }
  if (t == 0) a.chunk_count[static_cast<size_t>(seg) * s.nchunks + c] = base;
  if (s.rescue && t < G) {
    const size_t hq = static_cast<size_t>(i) * s.Hq + g * G + t;
    atomicAdd(&a.head_count[hq], s_cnt[t]);
    atomicMax(&a.head_best[hq], s_best[t]);
  }
}

// Top-1 rescue (Appendix F.4), read row-wise: a query head that admitted no
// block at all admits its highest-scoring block (lowest id on ties).  One
// thread per (sequence, KV head) patches the chunk list: the block is either
// already listed (its head bit is added) or inserted in ascending position.
__global__ void rescue_kernel(ScreenArgs a) {
  const Shape& s = a.s;
  const int g = blockIdx.x, i = blockIdx.y;
  if (threadIdx.x != 0) return;
  const int seg = i * s.Hkv + g;
  for (int j = 0; j < s.G; ++j) {
    const size_t hq = static_cast<size_t>(i) * s.Hq + g * s.G + j;
    if (a.head_count[hq] != 0 || a.head_best[hq] == 0ull) continue;
    const int blk = static_cast<int>(0xffffffffu - static_cast<unsigned>(a.head_best[hq] & 0xffffffffull));
    const int c = blk / s.chunk;
    int* list = a.chunk_list + static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(c) * s.chunk;
    int* cnt = a.chunk_count + static_cast<size_t>(seg) * s.nchunks + c;
    const int n = *cnt;
    int pos = 0;
    while (pos < n && (list[pos] & kMaxBlocksPerSeq) < blk) ++pos;
    if (pos < n && (list[pos] & kMaxBlocksPerSeq) == blk) {
      list[pos] |= (1 << j) << kEntryBlockBits;
    } else {
      for (int k = n; k > pos; --k) list[k] = list[k - 1];
      list[pos] = blk | ((1 << j) << kEntryBlockBits);
      *cnt = n + 1;
    }
  }
}

template <int D>
cudaError_t launch_screen_d(const ScreenArgs& a, cudaStream_t st) {
  dim3 grid(a.s.nchunks, a.s.Hkv, a.s.B);
  switch (a.s.G) {
    case 1: screen_kernel<D, 1><<<grid, kThreads, 0, st>>>(a); break;
    case 2: screen_kernel<D, 2><<<grid, kThreads, 0, st>>>(a); break;
    case 4: screen_kernel<D, 4><<<grid, kThreads, 0, st>>>(a); break;
    case 8: screen_kernel<D, 8><<<grid, kThreads, 0, st>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_screen(const ScreenArgs& a, cudaStream_t st) {
  if (a.s.chunk > kMaxChunk) return cudaErrorInvalidValue;
  return a.s.d == 64 ? launch_screen_d<64>(a, st) : launch_screen_d<128>(a, st);
}

cudaError_t launch_rescue(const ScreenArgs& a, cudaStream_t st) {
  dim3 grid(a.s.Hkv, a.s.B);
  rescue_kernel<<<grid, 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace eta
