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
// (sequence, KV head).  The metadata rows are staged in shared memory with
// 1-D bulk copies (rounds of 64 blocks; the first round overlaps the threshold
// computation); lanes split the head dimension, and the 2G partial sums of
// 32 / (2G) blocks are reduced together by one transposing butterfly.  The
// admitted blocks of the chunk are written, ascending, as list entries
// (block id | head mask << 24) plus the chunk's entry count.
#include <math.h>

#include "eta_device.cuh"

namespace eta {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kMaxChunk = 1024;

constexpr int kRound = 64;  // blocks of metadata staged in shared memory per round

// Staging buffers of mu and sigma rows (ESZ bytes per coordinate: 2 for fp16,
// 1 for e4m3 codes): the second one is used only when a chunk needs more than
// one round.
template <int D, int ESZ>
constexpr size_t screen_smem_bytes(int chunk) {
  return (chunk > kRound ? 2ull : 1ull) * 2 * kRound * D * ESZ;
}

// Two e4m3 codes (low byte first) as floats.
__device__ __forceinline__ float2 e4m3x2_to_f32(uint16_t codes) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(codes));
  return make_float2(dev::fp16_to_f32(static_cast<uint16_t>(h2 & 0xffffu)), dev::fp16_to_f32(static_cast<uint16_t>(h2 >> 16)));
}

// FMT: ETA_META_FP16 or ETA_META_FP8 (then mu~ = code * mu_scale per block,
// and <q, mu~> = mu_scale <q, code>, sum q^2 sigma~^2 = sigma_scale^2 sum q^2 code^2:
// the scales are applied after the reduction over d).
template <int D, int G, int FMT>
__global__ void __launch_bounds__(kThreads) screen_kernel(ScreenArgs a) {
  constexpr int ESZ = FMT == ETA_META_FP8 ? 1 : 2;
  constexpr int CPL = D / 32;        // coordinates per lane
  constexpr int NV = 2 * G;          // values per block: <q_h, mu>, sum q_h^2 sigma^2
  constexpr int NB = 32 / NV;        // blocks reduced together (32 values per lane)
  const Shape& s = a.s;
  const int c = blockIdx.x, g = blockIdx.y, i = blockIdx.z;
  const int seg = i * s.Hkv + g;
  const int t = threadIdx.x, w = t >> 5, lane = t & 31;

  extern __shared__ __align__(128) uint8_t dsm[];
  uint8_t* stage = dsm;  // [2 buffers][mu, sigma][kRound][D] elements of ESZ bytes
  __shared__ float s_q[G][D];
  __shared__ float s_tau[G];
  __shared__ float s_qn[G];
  __shared__ float s_mn[kMaxChunk];
  __shared__ float s_ms[FMT == ETA_META_FP8 ? kMaxChunk : 1];
  __shared__ float s_ss[FMT == ETA_META_FP8 ? kMaxChunk : 1];
  __shared__ uint8_t s_mask[kMaxChunk];
  __shared__ int s_wsum[kWarps];
  __shared__ int s_cnt[G];
  __shared__ unsigned long long s_best[G];
  __shared__ __align__(8) uint64_t s_bar[2];

  // The attention kernel may be scheduled now; it waits for this grid's
  // completion before reading anything written here.  This grid is itself
  // launched as a dependent of the stream's previous kernel (the token's
  // append, or the previous step's merge, which reads the chunk counts this
  // grid rewrites): nothing is read or written before that kernel is done.
  dev::pdl_trigger();
  dev::pdl_wait();
  if (threadIdx.x == 0) dev::trace_first(a.trace, ETA_TRACE_SCREEN_FIRST);

  const int blk0 = c * s.chunk;
  const int avail = min(s.chunk, s.nbmax - blk0);  // rows of this chunk inside the arrays
  const size_t mbase = (static_cast<size_t>(seg) * s.nbmax) * D;
  const size_t nbase = static_cast<size_t>(seg) * s.nbmax;
  auto issue_round = [&](int r0, int rows) {
    const int buf = (r0 / kRound) & 1;
    uint8_t* mu_b = stage + static_cast<size_t>(buf) * 2 * kRound * D * ESZ;
    const uint32_t bytes = static_cast<uint32_t>(rows) * D * ESZ;
    const size_t src = (mbase + static_cast<size_t>(blk0 + r0) * D) * ESZ;
    dev::mbar_arrive_expect_tx(&s_bar[buf], 2 * bytes);
    dev::bulk_g2s(mu_b, static_cast<const uint8_t*>(a.mu) + src, bytes, &s_bar[buf]);
    dev::bulk_g2s(mu_b + kRound * D * ESZ, static_cast<const uint8_t*>(a.sigma) + src, bytes, &s_bar[buf]);
  };
  // Stage the first round of metadata before the sequence length is known
  // (rows past it are in bounds and simply not used), together with the
  // block norms (and scales), while the threshold is computed.  With the
  // screen off no metadata is read at all.
  const bool meta = a.screen_enabled && avail > 0;
  if (t == 0) {
    dev::mbar_init(&s_bar[0], 1);
    dev::mbar_init(&s_bar[1], 1);
    dev::fence_barrier_init();
    if (meta) issue_round(0, min(kRound, avail));
  }
  if (meta) {
    for (int x = t; x < avail; x += kThreads) {
      s_mn[x] = a.max_norm[nbase + blk0 + x];
      if (FMT == ETA_META_FP8) {
        s_ms[x] = a.mu_scale[nbase + blk0 + x];
        s_ss[x] = a.sigma_scale[nbase + blk0 + x];
      }
    }
  }

  // Threshold inputs of this warp's head, loaded now so that they share the
  // first round trip with the metadata copies and the query rows.
  float w_reg[D / 32], q_reg[D / 32];
  float b_or_c = 0.f;
  if (w < G) {
    const int hq = g * G + w;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      const int e = lane + 32 * k;
      q_reg[k] = dev::load_elt(a.q, (static_cast<size_t>(i) * s.Hq + hq) * D + e, s.elt);
      w_reg[k] = a.tau_mode == ETA_TAU_LEARNED ? a.w_tau[static_cast<size_t>(hq) * D + e] : 0.f;
    }
    b_or_c = a.tau_mode == ETA_TAU_LEARNED ? a.b_tau[hq] : a.c_tau[hq];
  }
  int T = a.seq_lens[i];
  if (T < 0 || T > s.max_ctx) {
    if (t == 0 && c == 0 && g == 0) atomicOr(a.status, kStatusRange);
    T = T < 0 ? 0 : s.max_ctx;
  }
  const int nb = (T + s.b - 1) / s.b;
  const int nloc = max(0, min(s.chunk, nb - blk0));
  const int first_forced = (!a.screen_enabled) ? 0 : (a.lwb >= 0 ? max(0, nb - 1 - a.lwb) : nb);
  const int nscreen = max(0, min(nloc, first_forced - blk0));  // leading blocks of the chunk that are screened
  if (t == 0 && nscreen > kRound) issue_round(kRound, min(kRound, nscreen - kRound));

  for (int x = t; x < G * D; x += kThreads) {
    const int h = x / D, e = x - h * D;
    s_q[h][e] = dev::load_elt(a.q, (static_cast<size_t>(i) * s.Hq + g * G + h) * D + e, s.elt);
  }
  if (t < G) {
    s_cnt[t] = 0;
    s_best[t] = 0ull;
  }
  if (c == 0 && nb == 0) {
    // an empty sequence has no unit to attend: its outputs are 0, lse -inf
    for (int x = t; x < G * D; x += kThreads) {
      const size_t o = (static_cast<size_t>(i) * s.Hq + g * G) * D + x;
      if (s.elt == 4) static_cast<float*>(a.out)[o] = 0.f; else static_cast<uint16_t*>(a.out)[o] = 0;
    }
    if (t < G && a.lse) a.lse[static_cast<size_t>(i) * s.Hq + g * G + t] = -INFINITY;
  }
  if (w < G) {
    const int hq = g * G + w;
    float tw = 0.f, qq = 0.f;
#pragma unroll
    for (int k = 0; k < D / 32; ++k) {
      qq = fmaf(q_reg[k], q_reg[k], qq);
      tw = fmaf(w_reg[k], q_reg[k], tw);
    }
    tw = dev::warp_sum(tw);
    qq = dev::warp_sum(qq);
    const float tau = (a.tau_mode == ETA_TAU_LEARNED ? tw + b_or_c : b_or_c) - a.offset_a;
    if (lane == 0) {
      s_tau[w] = tau;
      s_qn[w] = sqrtf(qq);
      if (c == 0) a.tau[static_cast<size_t>(i) * s.Hq + hq] = tau;
    }
  }
  for (int lb = nscreen + t; lb < nloc; lb += kThreads) s_mask[lb] = static_cast<uint8_t>((1u << G) - 1u);
  __syncthreads();

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
  // after the reduction lane l holds value l % NV of block l / NV of the group
  const int vb = lane / NV, vq = lane % NV;
  const float my_tau = s_tau[vq % G], my_qn = s_qn[vq % G];

  bool staged_ok = true;
  for (int r0 = 0; r0 < nscreen && staged_ok; r0 += kRound) {
    const int r = min(kRound, nscreen - r0);
    const int buf = (r0 / kRound) & 1;
    const uint8_t* mu_s = stage + static_cast<size_t>(buf) * 2 * kRound * D * ESZ;
    const uint8_t* sg_s = mu_s + kRound * D * ESZ;
    if (!dev::mbar_wait(&s_bar[buf], (r0 / (2 * kRound)) & 1, a.status)) { staged_ok = false; break; }
    for (int gb = w * NB; gb < r; gb += kWarps * NB) {
      float v[32];
#pragma unroll
      for (int u = 0; u < NB; ++u) {
        const int lb = min(gb + u, r - 1);  // a short last group repeats a valid row
        float mu[CPL], s2[CPL], mx[CPL];
#pragma unroll
        for (int k = 0; k < CPL / 2; ++k) {
          float2 m, g2;
          if (FMT == ETA_META_FP8) {
            m = e4m3x2_to_f32(*reinterpret_cast<const uint16_t*>(mu_s + lb * D + lane * CPL + 2 * k));
            g2 = e4m3x2_to_f32(*reinterpret_cast<const uint16_t*>(sg_s + lb * D + lane * CPL + 2 * k));
          } else {
            const uint32_t mm = *reinterpret_cast<const uint32_t*>(mu_s + (lb * D + lane * CPL + 2 * k) * 2);
            const uint32_t gg = *reinterpret_cast<const uint32_t*>(sg_s + (lb * D + lane * CPL + 2 * k) * 2);
            m = make_float2(dev::fp16_to_f32(static_cast<uint16_t>(mm & 0xffffu)),
                            dev::fp16_to_f32(static_cast<uint16_t>(mm >> 16)));
            g2 = make_float2(dev::fp16_to_f32(static_cast<uint16_t>(gg & 0xffffu)),
                             dev::fp16_to_f32(static_cast<uint16_t>(gg >> 16)));
          }
          mu[2 * k] = m.x;
          mu[2 * k + 1] = m.y;
          mx[2 * k] = g2.x;
          mx[2 * k + 1] = g2.y;
          s2[2 * k] = g2.x * g2.x;
          s2[2 * k + 1] = g2.y * g2.y;
        }
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float dot = 0.f, sq = 0.f;
          if (FMT == ETA_META_BOX) {
            // mu holds the per-coordinate minima, mx the maxima
#pragma unroll
            for (int k = 0; k < CPL; ++k) dot += fmaxf(qr[h][k] * mu[k], qr[h][k] * mx[k]);
          } else {
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
              dot = fmaf(qr[h][k], mu[k], dot);
              sq = fmaf(q2[h][k], s2[k], sq);
            }
          }
          v[u * NV + h] = dot;
          v[u * NV + G + h] = sq;
        }
      }
      float red = dev::transpose_reduce32<32>(v, lane);
      float sq = __shfl_down_sync(0xffffffffu, red, G);  // sum q^2 sigma^2 of the same (block, head)
      const int lb = gb + vb;
      const bool head_lane = vq < G && lb < r;
      float score = 0.f;
      bool pass = false;
      if (head_lane) {
        if (FMT == ETA_META_FP8) {
          const float ss = s_ss[r0 + lb];
          red *= s_ms[r0 + lb];
          sq *= ss * ss;
        }
        if (FMT == ETA_META_BOX) {
          score = scale * red;
        } else {
          const float geo = my_qn * s_mn[r0 + lb];
          const float spread = strict ? geo : fminf(geo, z * sqrtf(sq));
          score = scale * (red + spread);
        }
        pass = score >= my_tau;
      }
      const unsigned bal = __ballot_sync(0xffffffffu, pass);
      if (vq == 0 && lb < r) s_mask[r0 + lb] = static_cast<uint8_t>((bal >> (vb * NV)) & ((1u << G) - 1u));
      if (s.rescue && head_lane) {
        const int blk = blk0 + r0 + lb;
        const unsigned long long key =
            (static_cast<unsigned long long>(dev::float_order_key(score)) << 32) |
            static_cast<unsigned long long>(0xffffffffu - static_cast<unsigned>(blk));
        atomicMax(&s_best[vq], key);
        if (pass) atomicAdd(&s_cnt[vq], 1);
      }
    }
    __syncthreads();  // this buffer's rows are consumed
    if (t == 0 && r0 + 2 * kRound < nscreen) issue_round(r0 + 2 * kRound, min(kRound, nscreen - r0 - 2 * kRound));
  }
  if (!staged_ok) {
    // a staging wait ran out (recorded in the status word): admit the rest
    for (int lb = t; lb < nscreen; lb += kThreads) s_mask[lb] = static_cast<uint8_t>((1u << G) - 1u);
  }
  // The speculative first copy lands before exit even when nothing here
  // was screened.
  if (t == 0 && nscreen == 0 && meta) dev::mbar_wait(&s_bar[0], 0, a.status);
  __syncthreads();
  if (nloc == 0) {
    if (t == 0) {
      a.chunk_count[static_cast<size_t>(seg) * s.nchunks + c] = 0;
      dev::trace_last(a.trace, ETA_TRACE_SCREEN_LAST);
    }
    return;
  }

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
  if (t == 0) {
    a.chunk_count[static_cast<size_t>(seg) * s.nchunks + c] = base;
    dev::trace_last(a.trace, ETA_TRACE_SCREEN_LAST);
  }
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

template <int D, int G, int FMT>
cudaError_t launch_screen_typed(const ScreenArgs& a, cudaStream_t st) {
  constexpr int ESZ = FMT == ETA_META_FP8 ? 1 : 2;  // the box format stores fp16
  const size_t smem = screen_smem_bytes<D, ESZ>(a.s.chunk);
  auto kern = screen_kernel<D, G, FMT>;
  static SmemLimit lim;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.s.nchunks, a.s.Hkv, a.s.B);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_with_smem(reinterpret_cast<const void*>(kern), screen_smem_bytes<D, ESZ>(2 * kRound), lim,
                          [&] { return cudaLaunchKernelEx(&cfg, kern, a); });
}

template <int D, int FMT>
cudaError_t launch_screen_d(const ScreenArgs& a, cudaStream_t st) {
  switch (a.s.G) {
    case 1: return launch_screen_typed<D, 1, FMT>(a, st);
    case 2: return launch_screen_typed<D, 2, FMT>(a, st);
    case 4: return launch_screen_typed<D, 4, FMT>(a, st);
    case 8: return launch_screen_typed<D, 8, FMT>(a, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_screen(const ScreenArgs& a, cudaStream_t st) {
  if (a.s.chunk > kMaxChunk) return cudaErrorInvalidValue;
  // with the screen off no metadata is read: the fp16 instance serves
  if (a.screen_enabled && a.meta_fmt == ETA_META_FP8)
    return a.s.d == 64 ? launch_screen_d<64, ETA_META_FP8>(a, st) : launch_screen_d<128, ETA_META_FP8>(a, st);
  if (a.screen_enabled && a.meta_fmt == ETA_META_BOX)
    return a.s.d == 64 ? launch_screen_d<64, ETA_META_BOX>(a, st) : launch_screen_d<128, ETA_META_BOX>(a, st);
  return a.s.d == 64 ? launch_screen_d<64, ETA_META_FP16>(a, st) : launch_screen_d<128, ETA_META_FP16>(a, st);
}

cudaError_t launch_rescue(const ScreenArgs& a, cudaStream_t st) {
  dim3 grid(a.s.Hkv, a.s.B);
  rescue_kernel<<<grid, 32, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace eta
