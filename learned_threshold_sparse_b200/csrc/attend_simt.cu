// Split-KV attention over the admitted (GQA-union) blocks, CUDA-core version.
//
// Source: Elastic Threshold Attention,
//   Appendix F.1 step 2   a listed block is fetched once for the G query heads
//                         of its KV head; each head accumulates only the
//                         blocks it admitted (head-mask bit),
//   Appendix G.1          S = q k / sqrt(d), S~ = S sigmoid(beta (S - tau~)),
//                         weights exp(S~) (online softmax in base 2),
//   Appendix F.2          fp32 accumulation and softmax state,
//   section 3.2, F.3      split-KV partials (acc, m, l) merged later,
//   Appendix F.4          tail block: rows >= seq_len are masked.
//
// Persistent grid, one CTA per SM.  The global list of admitted units
// (segment, block, head mask), ordered by (sequence, KV head, block), is cut
// into equal contiguous ranges, one per CTA, so every CTA streams the same
// number of K/V blocks whatever the per-sequence densities.  Warp 8 is the
// producer: it walks the CTA's range and issues 1-D bulk copies (TMA) of the
// contiguous K and V tiles of each unit into a ring of shared-memory stages
// guarded by mbarriers.  Warps 0-7 consume: each keeps its own online-softmax
// state for the G heads; at a segment boundary the eight states are merged
// and written as one partial per (segment, CTA).
#include <math.h>

#include "attend_common.cuh"

namespace eta {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kMaxStages = 8;

using dev::UnitInfo;
using dev::wait_or_abort;

template <int ELT, int D, int G>
struct Cfg {
  static constexpr int LPR = D * ELT / 16;  // lanes per K/V row (8, 16, 32)
  static constexpr int RPW = 32 / LPR;      // rows per warp per step
  static constexpr int EPL = 16 / ELT;      // elements per lane
  static constexpr int ROWS = kConsumerWarps * RPW;  // rows per step
  static constexpr int MAX_STEPS = (128 + ROWS - 1) / ROWS;
  static constexpr int REP = LPR / G;       // lanes holding the same head
  static_assert(G <= LPR, "group size larger than lanes per row");
};

struct Smem {
  size_t kv, bars, info, scratch, prefix, flags, total;
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

__host__ __device__ inline Smem smem_layout(int stages, int b, int d, int elt, int G, int nprefix) {
  Smem L;
  L.kv = 0;
  size_t off = static_cast<size_t>(stages) * 2 * b * d * elt;
  L.bars = off = align_up(off, 16);
  off += (2 * stages + 1) * sizeof(uint64_t);
  L.info = off = align_up(off, 16);
  off += stages * sizeof(UnitInfo);
  L.scratch = off = align_up(off, 16);
  off += static_cast<size_t>(kConsumerWarps) * G * (d + 2) * sizeof(float);
  L.prefix = off = align_up(off, 16);
  off += static_cast<size_t>(nprefix + 1) * sizeof(int);
  L.flags = off = align_up(off, 16);
  off += 16 + kMaxStages * sizeof(int);
  L.total = align_up(off, 128);
  return L;
}

// Reduce G values across the LPR lanes of one row, halving the values held
// per stage; afterwards lane sub holds head sub / (LPR / G).
template <int G, int LPR>
__device__ __forceinline__ float row_transpose_reduce(float (&v)[G], int sub) {
  int n = G;
#pragma unroll
  for (int o = LPR / 2; o >= 1; o >>= 1) {
    if (n > 1) {
      const bool upper = (sub & o) != 0;
      const int half = n >> 1;
#pragma unroll
      for (int j = 0; j < (G > 1 ? G / 2 : 1); ++j) {
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

template <int ELT, int D, int G>
__global__ void __launch_bounds__(kThreads, 1) attend_simt_kernel(AttendArgs a, int stages) {
  using C = Cfg<ELT, D, G>;
  extern __shared__ __align__(1024) uint8_t smem[];
  const Shape& s = a.s;
  const int nprefix = s.nseg * s.nchunks;
  const Smem L = smem_layout(stages, s.b, D, ELT, G, nprefix);
  uint8_t* kv = smem + L.kv;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + stages;
  uint64_t* flush_bar = empty + stages;  // consumer-warp rendezvous (count 8)
  UnitInfo* info = reinterpret_cast<UnitInfo*>(smem + L.info);
  float* scratch = reinterpret_cast<float*>(smem + L.scratch);
  int* prefix = reinterpret_cast<int*>(smem + L.prefix);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.flags);
  int* issued_parity = reinterpret_cast<int*>(smem + L.flags + 16);  // per stage, -1 = never
  const size_t tile_bytes = static_cast<size_t>(s.b) * D * ELT;

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int k = 0; k < stages; ++k) {
      dev::mbar_init(&full[k], 1);
      dev::mbar_init(&empty[k], kConsumerWarps);
      issued_parity[k] = -1;
    }
    dev::mbar_init(flush_bar, kConsumerWarps);
    *abort_flag = 0;
    dev::fence_barrier_init();
  }

  // Everything below reads what the screen wrote.
  dev::pdl_wait();
  dev::pdl_trigger();
  if (threadIdx.x == 0) dev::trace_first(a.trace, ETA_TRACE_ATTEND_FIRST);

  // Exclusive prefix of the per-chunk entry counts, in (segment, chunk) order.
  dev::chunk_prefix<kThreads>(a.chunk_count, nprefix, prefix);

  const dev::UnitSplit split(static_cast<unsigned>(prefix[nprefix]), gridDim.x);
  const int u0 = static_cast<int>(split.start(blockIdx.x));
  const int u1 = static_cast<int>(split.start(blockIdx.x + 1));
  const int nunits = u1 - u0;
  if (nunits == 0) return;

  if (warp == kConsumerWarps) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0;
    const bool ok = dev::walk_units(a, prefix, nprefix, u0, nunits, nullptr, [&](const UnitInfo& in) -> bool {
      if (!wait_or_abort(&empty[stage], phase ^ 1u, a.status, abort_flag)) return false;
      info[stage] = in;
      const uint32_t bytes = static_cast<uint32_t>(in.nrows) * D * ELT;
      dev::mbar_arrive_expect_tx(&full[stage], 2u * bytes);
      const size_t off = static_cast<size_t>(in.row) * D * ELT;
      uint8_t* dst = kv + static_cast<size_t>(stage) * 2 * tile_bytes;
      dev::bulk_g2s(dst, static_cast<const uint8_t*>(a.k) + off, bytes, &full[stage]);
      dev::bulk_g2s(dst + tile_bytes, static_cast<const uint8_t*>(a.v) + off, bytes, &full[stage]);
      issued_parity[stage] = static_cast<int>(phase);
      if (++stage == stages) { stage = 0; phase ^= 1u; }
      return true;
    });
    if (!ok && lane == 0) *abort_flag = 1;
    if (!ok && lane == 0) {
      // Let the copies already issued land before the CTA exits.
      for (int k = 0; k < stages; ++k) {
        if (issued_parity[k] < 0) continue;
        const long long t0 = clock64();
        while (!dev::mbar_try_wait(&full[k], static_cast<uint32_t>(issued_parity[k])) &&
               clock64() - t0 < dev::kWaitCycles) {
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ consumers
  const int rg = lane / C::LPR;        // row within the warp's step
  const int sub = lane - rg * C::LPR;  // 16-byte column slot of the row
  const int hh = sub / C::REP;         // head this lane reduces to
  const float scale = a.scale, beta = a.beta;

  float q[G][C::EPL], acc[G][C::EPL];
  float m_run = -INFINITY, l_run = 0.f, tau_h = 0.f;
  int cur_seg = -1;
  int stage = 0;
  uint32_t phase = 0;

  // Rendezvous of the 8 consumer warps on flush_bar (bounded: on a timeout
  // the flush is abandoned and the kernel winds down).  Consecutive
  // rendezvous complete consecutive phases.
  uint32_t rv_phase = 0;
  auto rendezvous = [&]() -> bool {
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(flush_bar);
    const bool r = wait_or_abort(flush_bar, rv_phase, a.status, abort_flag);
    rv_phase ^= 1u;
    return r;
  };

  // Segment done in this CTA: the eight warp states are merged; the result is
  // written straight to the output when no other CTA touches the segment,
  // else kept as this CTA's partial for the merge kernel.
  auto flush = [&](int seg) -> bool {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < C::EPL; ++e)
#pragma unroll
        for (int o = C::LPR; o < 32; o <<= 1) acc[h][e] += __shfl_xor_sync(0xffffffffu, acc[h][e], o);
#pragma unroll
    for (int o = C::LPR; o < 32; o <<= 1) l_run += __shfl_xor_sync(0xffffffffu, l_run, o);
    float* my = scratch + static_cast<size_t>(warp) * G * (D + 2);
    if (rg == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) my[h * (D + 2) + sub * C::EPL + e] = acc[h][e];
      if (sub % C::REP == 0) {
        my[hh * (D + 2) + D] = m_run;
        my[hh * (D + 2) + D + 1] = l_run;
      }
    }
    if (!rendezvous()) return false;
    // no other CTA touches the segment when all its units are in this range
    const bool sole = prefix[seg * s.nchunks] >= u0 && prefix[(seg + 1) * s.nchunks] <= u1;
    const int si = seg / s.Hkv, sg = seg - si * s.Hkv;
    float* part = a.partials + static_cast<size_t>(seg + blockIdx.x) * G * partial_stride(D);
    for (int x = t; x < G * D; x += kConsumerWarps * 32) {
      const int h = x / D, e = x - h * D;
      float mstar = -INFINITY;
      for (int w = 0; w < kConsumerWarps; ++w) mstar = fmaxf(mstar, scratch[(w * G + h) * (D + 2) + D]);
      float sum = 0.f, lsum = 0.f;
      if (mstar != -INFINITY) {
        for (int w = 0; w < kConsumerWarps; ++w) {
          const float* ws = scratch + (w * G + h) * (D + 2);
          const float f = ws[D] == -INFINITY ? 0.f : dev::fast_exp2(ws[D] - mstar);
          sum = fmaf(f, ws[e], sum);
          lsum = fmaf(f, ws[D + 1], lsum);
        }
      }
      if (sole) {
        const size_t orow = static_cast<size_t>(si) * s.Hq + sg * G + h;
        dev::store_out(a, orow * D + e, lsum > 0.f ? sum / lsum : 0.f);
        if (e == 0 && a.lse) a.lse[orow] = dev::lse_of(mstar, lsum);
      } else {
        part[h * partial_stride(D) + e] = sum;
        if (e == 0) {
          part[h * partial_stride(D) + D] = mstar;
          part[h * partial_stride(D) + D + 1] = lsum;
        }
      }
    }
    return rendezvous();  // the warp states may be overwritten after this
  };

  for (int u = 0; u < nunits; ++u) {
    if (!wait_or_abort(&full[stage], phase, a.status, abort_flag)) break;
    const UnitInfo in = info[stage];
    if (in.seg != cur_seg) {
      if (cur_seg >= 0 && !flush(cur_seg)) break;
      cur_seg = in.seg;
      const int i = in.seg / s.Hkv, g = in.seg - i * s.Hkv;
      const size_t qrow = static_cast<size_t>(i) * s.Hq + g * G;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float tmp[C::EPL];
        dev::Row16<ELT>::load(static_cast<const uint8_t*>(a.q) + ((qrow + h) * D + sub * C::EPL) * ELT, tmp);
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) {
          q[h][e] = tmp[e];
          acc[h][e] = 0.f;
        }
      }
      tau_h = a.tau[qrow + hh];
      m_run = -INFINITY;
      l_run = 0.f;
    }
    const uint8_t* Kt = kv + static_cast<size_t>(stage) * 2 * tile_bytes;
    const uint8_t* Vt = Kt + tile_bytes;
    const int nrows = in.nrows;
    const bool head_on = (in.mask >> hh) & 1;
    const int nsteps = (nrows + C::ROWS - 1) / C::ROWS;

    float st[C::MAX_STEPS];
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < C::MAX_STEPS; ++k) {
      st[k] = -INFINITY;
      if (k < nsteps) {
        const int r = k * C::ROWS + warp * C::RPW + rg;
        const bool valid = r < nrows;
        float kx[C::EPL];
        dev::Row16<ELT>::load(Kt + (static_cast<size_t>(valid ? r : 0) * D + sub * C::EPL) * ELT, kx);
        float part[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float acc_d = 0.f;
#pragma unroll
          for (int e = 0; e < C::EPL; ++e) acc_d = fmaf(q[h][e], kx[e], acc_d);
          part[h] = acc_d;
        }
        const float dot = row_transpose_reduce<G, C::LPR>(part, sub);
        const float S = dot * scale;
        const float St = S * dev::logistic(beta * (S - tau_h));
        st[k] = (valid && head_on) ? St * kLog2e : -INFINITY;
        mx = fmaxf(mx, st[k]);
      }
    }
#pragma unroll
    for (int o = C::LPR; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float m_new = fmaxf(m_run, mx);
    const float alpha = (m_new == -INFINITY || m_run == -INFINITY) ? (m_run == -INFINITY ? 0.f : 1.f)
                                                                  : dev::fast_exp2(m_run - m_new);
    float p[C::MAX_STEPS];
    float psum = 0.f;
#pragma unroll
    for (int k = 0; k < C::MAX_STEPS; ++k) {
      p[k] = (st[k] == -INFINITY) ? 0.f : dev::fast_exp2(st[k] - m_new);
      psum += p[k];
    }
    l_run = l_run * alpha + psum;
    m_run = m_new;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float ah = __shfl_sync(0xffffffffu, alpha, h * C::REP);
#pragma unroll
      for (int e = 0; e < C::EPL; ++e) acc[h][e] *= ah;
    }
#pragma unroll
    for (int k = 0; k < C::MAX_STEPS; ++k) {
      if (k < nsteps) {
        const int r = k * C::ROWS + warp * C::RPW + rg;
        const bool valid = r < nrows;
        float vx[C::EPL];
        dev::Row16<ELT>::load(Vt + (static_cast<size_t>(valid ? r : 0) * D + sub * C::EPL) * ELT, vx);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float ph = __shfl_sync(0xffffffffu, p[k], rg * C::LPR + h * C::REP);
          if (valid) {
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) acc[h][e] = fmaf(ph, vx[e], acc[h][e]);
          }
        }
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[stage]);
    if (++stage == stages) { stage = 0; phase ^= 1u; }
  }
  if (cur_seg >= 0 && !*abort_flag) flush(cur_seg);
  if (lane == 0) dev::trace_last(a.trace, ETA_TRACE_ATTEND_LAST);
}

template <int ELT, int D, int G>
cudaError_t launch_typed(const AttendArgs& a, cudaStream_t st, int stages, size_t smem) {
  auto kern = attend_simt_kernel<ELT, D, G>;
  static SmemLimit lim;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.s.attend_ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return launch_with_smem(reinterpret_cast<const void*>(kern), smem, lim,
                          [&] { return cudaLaunchKernelEx(&cfg, kern, a, stages); });
}

template <int ELT, int D>
cudaError_t launch_g(const AttendArgs& a, cudaStream_t st, int stages, size_t smem) {
  switch (a.s.G) {
    case 1: return launch_typed<ELT, D, 1>(a, st, stages, smem);
    case 2: return launch_typed<ELT, D, 2>(a, st, stages, smem);
    case 4: return launch_typed<ELT, D, 4>(a, st, stages, smem);
    case 8: return launch_typed<ELT, D, 8>(a, st, stages, smem);
  }
  return cudaErrorInvalidValue;
}

constexpr size_t kSmemBudget = 224 * 1024;  // leaves room for static shared memory

int pick_stages(const Shape& s) {
  for (int st = kMaxStages; st >= 2; --st) {
    if (smem_layout(st, s.b, s.d, s.elt, s.G, s.nseg * s.nchunks).total <= kSmemBudget) return st;
  }
  return 0;
}

}  // namespace

size_t attend_simt_smem(const Shape& s) {
  const int st = pick_stages(s);
  if (st == 0) return 0;
  return smem_layout(st, s.b, s.d, s.elt, s.G, s.nseg * s.nchunks).total;
}

int attend_simt_ctas_per_sm(const Shape&) { return 1; }

cudaError_t launch_attend_simt(const AttendArgs& a, cudaStream_t st) {
  const int stages = pick_stages(a.s);
  if (stages == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = smem_layout(stages, a.s.b, a.s.d, a.s.elt, a.s.G, a.s.nseg * a.s.nchunks).total;
  if (a.s.elt == 2) {
    return a.s.d == 64 ? launch_g<2, 64>(a, st, stages, smem) : launch_g<2, 128>(a, st, stages, smem);
  }
  return a.s.d == 64 ? launch_g<4, 64>(a, st, stages, smem) : launch_g<4, 128>(a, st, stages, smem);
}

}  // namespace eta
