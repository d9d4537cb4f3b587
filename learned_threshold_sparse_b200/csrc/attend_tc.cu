// Split-KV attention over the admitted (GQA-union) blocks on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory), bf16 K/V, d = 128.
//
// Source: Elastic Threshold Attention,
//   Appendix F.1 step 2   a listed block is fetched once for the G query heads
//                         of its KV head; each head accumulates only the
//                         blocks it admitted (head-mask bit),
//   Appendix F.2          bf16 operands on the tensor cores; fp32 scores,
//                         scales and softmax state,
//   Appendix G.1          S = q k / sqrt(d), S~ = S sigmoid(beta (S - tau~)),
//                         weights exp(S~) (online softmax, base 2),
//   section 3.2, F.3      split-KV partials (acc, m, l) merged later,
//   Appendix F.4          tail block: rows >= seq_len are masked.
//
// Per tile (128 key rows: one admitted 128-token block, or two consecutive
// admitted 64-token blocks of the same (sequence, KV head)):
//   S^T [128 x 16] = K [128 x 128] . Q^T [128 x 16]   (M = 128 rows, N = 16 query
//                                                      rows: the G heads, rest unused)
//   O^T [128 x 16] = V^T [128 x 128] . P^T [128 x 16] (M = d, N = 16)
// K, V and the group's 16 query rows arrive by TMA (128-byte swizzle) into a
// ring of shared-memory stages; one thread issues the MMAs; four warps read S
// from tensor memory (thread = token), apply the tempering and the online
// softmax, write P (bf16, swizzled) for the second MMA, and fold each O^T
// (thread = output coordinate) into fp32 register accumulators.
//
// Roles: warp 0 TMA producer, warp 1 tensor-memory owner and MMA issuer,
// warps 2-5 softmax/correction.  Same persistent work split as the CUDA-core
// kernel (equal ranges of the global admitted-unit list per CTA).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attend_common.cuh"
#include "tc_common.cuh"

namespace eta {
namespace {

using dev::UnitInfo;
using dev::wait_or_abort;
using namespace tc;

constexpr int D = 128;
constexpr int NQ = 16;              // N of both MMAs
constexpr int kWarps = 6;
constexpr int kThreads = kWarps * 32;
constexpr int kTmemCols = 64;       // S buffers at columns 0, 16; O buffers at 32, 48
constexpr int kMaxStages = 8;
constexpr float kLog2e = 1.4426950408889634f;

constexpr int TR = 128;  // key rows per tile
constexpr int kSmemSeqs = 256;
constexpr int kPrefixBar = 1;   // named barrier: producer publishes the prefix table  // sequence lengths staged in shared memory up to this batch

struct Tile {
  static constexpr int PANEL = TR * 128;  // one 64-column (128-byte) panel of a 128-row tile
  static constexpr int K0 = 0, K1 = PANEL, V0 = 2 * PANEL, V1 = 3 * PANEL, Q0 = 4 * PANEL, Q1 = 4 * PANEL + 2048;
  static constexpr int STAGE = 4 * PANEL + 4096;
  static constexpr int P_BYTES = NQ * TR * 2;
};

// What the producer tells the consumers about a tile: its segment and, per
// block of the tile, the admitting heads and the rows present (0 = absent).
struct TileInfo {
  int seg, mask0, mask1, nrows0, nrows1;
};

struct Layout {
  size_t stages, pbuf, bars, info, red, prefix, seqs, misc, total;
};

__host__ __device__ inline size_t align_to(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Offsets relative to a 1024-byte aligned base.
__host__ __device__ inline int smem_seqs(int B) { return B <= kSmemSeqs ? B : 0; }

__host__ __device__ inline Layout tc_layout(int nstages, int nprefix, int nseqs) {
  Layout L;
  const size_t stage = static_cast<size_t>(Tile::STAGE);
  const size_t pbytes = static_cast<size_t>(Tile::P_BYTES);
  size_t off = 0;
  L.stages = off;
  off += nstages * stage;
  L.pbuf = off;
  off += 2 * pbytes;
  L.bars = off = align_to(off, 16);
  off += (2 * kMaxStages + 12) * sizeof(uint64_t);
  L.info = off = align_to(off, 16);
  off += kMaxStages * sizeof(TileInfo);
  L.red = off = align_to(off, 16);
  off += 2 * 4 * 8 * sizeof(float) + 4 * 8 * sizeof(float);
  L.prefix = off = align_to(off, 16);
  off += static_cast<size_t>(nprefix + 1) * sizeof(int);
  L.seqs = off = align_to(off, 16);
  off += static_cast<size_t>(nseqs) * sizeof(int);
  L.misc = off = align_to(off, 16);
  off += 16 + kMaxStages * sizeof(int) + 16;
  L.total = align_to(off, 128) + 1024;  // + slack to align the dynamic base to 1024
  return L;
}

// Barrier indices inside the barrier block.
struct Bars {
  uint64_t* kv_full;   // [stages]   producer -> MMA, softmax   (tx bytes)
  uint64_t* kv_empty;  // [stages]   MMA commit -> producer
  uint64_t* s_full;    // [2]        MMA commit -> softmax
  uint64_t* s_free;    // [2]        softmax (4 warps) -> MMA
  uint64_t* p_full;    // [2]        softmax (4 warps) -> MMA
  uint64_t* o_full;    // [2]        MMA commit -> softmax
  uint64_t* o_free;    // [2]        softmax (4 warps) -> MMA
  uint64_t* rv;        // [1]        softmax-warp rendezvous (4 warps)
  uint64_t* done;      // [1]        final MMA commit
};

template <int BR, int G>
__global__ void __launch_bounds__(kThreads, 1)
    attend_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     const __grid_constant__ CUtensorMap tq, AttendArgs a, int nstages) {
  using TL = Tile;
  constexpr int BPT = TR / BR;  // blocks per tile
  extern __shared__ uint8_t smem_raw[];
  const Shape& s = a.s;
  const int nprefix = s.nseg * s.nchunks;
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw);
  const int nseqs = smem_seqs(s.B);
  const Layout L = tc_layout(nstages, nprefix, nseqs);

  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bars);
  Bars B;
  B.kv_full = bars;
  B.kv_empty = bars + kMaxStages;
  B.s_full = bars + 2 * kMaxStages;
  B.s_free = B.s_full + 2;
  B.p_full = B.s_free + 2;
  B.o_full = B.p_full + 2;
  B.o_free = B.o_full + 2;
  B.rv = B.o_free + 2;
  B.done = B.rv + 1;
  TileInfo* info = reinterpret_cast<TileInfo*>(base + L.info);
  float* red = reinterpret_cast<float*>(base + L.red);  // [2][4][8] tile maxima, then [4][8] flush sums
  int* prefix = reinterpret_cast<int*>(base + L.prefix);
  int* seq_T = reinterpret_cast<int*>(base + L.seqs);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.misc + 4);
  int* issued_parity = reinterpret_cast<int*>(base + L.misc + 32);

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int k = 0; k < nstages; ++k) {
      dev::mbar_init(&B.kv_full[k], 1);
      dev::mbar_init(&B.kv_empty[k], 1);
      issued_parity[k] = -1;
    }
    for (int k = 0; k < 2; ++k) {
      dev::mbar_init(&B.s_full[k], 1);
      dev::mbar_init(&B.s_free[k], 4);
      dev::mbar_init(&B.p_full[k], 4);
      dev::mbar_init(&B.o_full[k], 1);
      dev::mbar_init(&B.o_free[k], 4);
    }
    dev::mbar_init(B.rv, 4);
    dev::mbar_init(B.done, 1);
    *abort_flag = 0;
    dev::fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  // P rows >= G stay zero for the whole kernel.
  for (int x = t; x < 2 * TL::P_BYTES / 16; x += kThreads)
    reinterpret_cast<uint4*>(base + L.pbuf)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();  // the zero rows are read by the tensor cores
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tq)) : "memory");
  }
  // Inputs the screen does not write are read while it still runs.
  for (int x = t; x < nseqs; x += kThreads) {
    const int tt = a.seq_lens[x];
    seq_T[x] = tt < 0 ? 0 : (tt > s.max_ctx ? s.max_ctx : tt);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  dev::pdl_wait();  // screen results visible from here on
  dev::pdl_trigger();
  if (t == 0) dev::trace_first(a.trace, ETA_TRACE_ATTEND_FIRST);
  // The producer scans the chunk counts itself and publishes the table on a
  // named barrier, so its first copies do not wait on CTA-wide barriers; the
  // other warps pick the table up there (large tables: all warps scan).
  const bool warp_scan = nprefix <= dev::kWarpPrefixMax;
  if (warp_scan) {
    if (warp == 0) {
      dev::warp_prefix(a.chunk_count, nprefix, prefix);
      __threadfence_block();
      dev::named_bar_arrive(kPrefixBar, kThreads);
    } else {
      dev::named_bar_sync(kPrefixBar, kThreads);
    }
  } else {
    dev::chunk_prefix<kThreads>(a.chunk_count, nprefix, prefix);
  }

  const dev::UnitSplit split(static_cast<unsigned>(prefix[nprefix]), gridDim.x);
  const int u0 = static_cast<int>(split.start(blockIdx.x));
  const int u1 = static_cast<int>(split.start(blockIdx.x + 1));
  const int nunits = u1 - u0;

  const int ntiles = warp == 0 ? 0 : dev::count_tiles<BPT>(prefix, s, u0, u1);

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    // Consecutive units of one segment are packed BPT to a tile; block i of a
    // tile fills rows [i BR, (i + 1) BR) of every 128-row panel.
    if (nunits > 0) {
      int stage = 0;
      uint32_t phase = 0;
      TileInfo pend{-1, 0, 0, 0, 0};
      int prow[2] = {0, 0};
      int npend = 0;
      auto emit = [&]() -> bool {
        if (!wait_or_abort(&B.kv_empty[stage], phase ^ 1u, a.status, abort_flag)) return false;
        info[stage] = pend;
        const uint32_t st = base_u32 + static_cast<uint32_t>(L.stages + stage * TL::STAGE);
        dev::mbar_arrive_expect_tx(&B.kv_full[stage], static_cast<uint32_t>(npend * 4 * BR * 128 + 4096));
        for (int i = 0; i < npend; ++i) {
          const int krow = prow[i];
          const uint32_t ro = static_cast<uint32_t>(i * BR * 128);
          tma_load_2d(st + TL::K0 + ro, &tk, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::K1 + ro, &tk, 64, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V0 + ro, &tv, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V1 + ro, &tv, 64, krow, &B.kv_full[stage]);
        }
        const int qrow = pend.seg * s.G;
        tma_load_2d(st + TL::Q0, &tq, 0, qrow, &B.kv_full[stage]);
        tma_load_2d(st + TL::Q1, &tq, 64, qrow, &B.kv_full[stage]);
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == nstages) { stage = 0; phase ^= 1u; }
        npend = 0;
        return true;
      };
      bool ok = dev::walk_units(a, prefix, nprefix, u0, nunits, nseqs ? seq_T : nullptr,
                                [&](const UnitInfo& in) -> bool {
        if (npend > 0 && in.seg != pend.seg && !emit()) return false;
        if (npend == 0) pend = TileInfo{in.seg, 0, 0, 0, 0};
        prow[npend] = static_cast<int>(in.row);
        if (npend == 0) { pend.mask0 = in.mask; pend.nrows0 = in.nrows; }
        else { pend.mask1 = in.mask; pend.nrows1 = in.nrows; }
        ++npend;
        return npend < BPT || emit();  // a full tile goes out at once
      });
      if (ok && lane == 0 && npend > 0) ok = emit();
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok && lane == 0) {
        *abort_flag = 1;
        for (int k = 0; k < nstages; ++k) {  // let issued copies land
          if (issued_parity[k] < 0) continue;
          const long long t0 = clock64();
          while (!dev::mbar_try_wait(&B.kv_full[k], static_cast<uint32_t>(issued_parity[k])) &&
                 clock64() - t0 < dev::kWaitCycles) {
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(TR, NQ, 0);
    constexpr uint32_t idesc_pv = idesc_bf16(D, NQ, 1);
    bool ok = true;
    auto issue_pv = [&](int i) -> bool {
      const int pb = i & 1;
      const int st_i = i % nstages;
      if (!wait_or_abort(&B.p_full[pb], (i >> 1) & 1, a.status, abort_flag)) return false;
      if (!wait_or_abort(&B.o_free[pb], ((i >> 1) & 1) ^ 1, a.status, abort_flag)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t vbase = base_u32 + static_cast<uint32_t>(L.stages + st_i * TL::STAGE) + TL::V0;
        const uint32_t pbase = base_u32 + static_cast<uint32_t>(L.pbuf + pb * TL::P_BYTES);
#pragma unroll
        for (int kk = 0; kk < TR / 16; ++kk) {
          const uint64_t ad = sw128_desc(vbase + kk * 2048, TL::PANEL, 1024);
          const uint64_t bd = sw128_desc(pbase + (kk >> 2) * 2048 + (kk & 3) * 32, 16, 1024);
          mma_bf16(tmem + 32 + pb * 16, ad, bd, idesc_pv, kk > 0 ? 1u : 0u);
        }
        mma_commit(&B.o_full[pb]);
        mma_commit(&B.kv_empty[st_i]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < ntiles && ok; ++j) {
      const int st_j = j % nstages;
      const int sb = j & 1;
      if (!wait_or_abort(&B.kv_full[st_j], (j / nstages) & 1, a.status, abort_flag)) { ok = false; break; }
      if (!wait_or_abort(&B.s_free[sb], ((j >> 1) & 1) ^ 1, a.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t sbase = base_u32 + static_cast<uint32_t>(L.stages + st_j * TL::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * TL::PANEL + (kk & 3) * 32;
          const uint32_t qoff = (kk >> 2) * 2048 + (kk & 3) * 32;
          const uint64_t ad = sw128_desc(sbase + TL::K0 + koff, 16, 1024);
          const uint64_t bd = sw128_desc(sbase + TL::Q0 + qoff, 16, 1024);
          mma_bf16(tmem + sb * 16, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&B.s_full[sb]);
      }
      __syncwarp();
      if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok && ntiles > 0) issue_pv(ntiles - 1);
    // every MMA issued so far has completed once `done` flips
    if (lane == 0) mma_commit(B.done);
    __syncwarp();
    {
      const long long t0 = clock64();
      while (!dev::mbar_try_wait(B.done, 0) && clock64() - t0 < dev::kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ softmax / correction
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t tlane = static_cast<uint32_t>(32 * q4) << 16;
    const int row = 32 * q4 + lane;  // key row of the tile this thread owns in S^T
    const int rblk = row / BR, rrow = row - rblk * BR;
    const int dcol = 32 * q4 + lane;  // output coordinate of this thread in O^T
    const float scale = a.scale, beta = a.beta;
    float m_run[G], l_thr[G], acc[G], alpha_prev[G], tau_h[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_thr[h] = 0.f;
      acc[h] = 0.f;
      alpha_prev[h] = 1.f;
      tau_h[h] = 0.f;
    }
    int cur_seg = -1;
    uint32_t rv_phase = 0;
    bool ok = true;

    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(B.rv);
      const bool r = wait_or_abort(B.rv, rv_phase, a.status, abort_flag);
      rv_phase ^= 1u;
      return r;
    };
    auto correction = [&](int i) -> bool {
      const int ob = i & 1;
      if (!dev::warp_wait_or_abort(&B.o_full[ob], (i >> 1) & 1, a.status, abort_flag)) return false;
      tc_fence_after();
      float o[8];
      tmem_ld8(tmem + tlane + 32 + ob * 16, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.o_free[ob]);
#pragma unroll
      for (int h = 0; h < G; ++h) acc[h] = fmaf(acc[h], alpha_prev[h], o[h]);
      return true;
    };
    // Segment done in this CTA: written straight to the output when no other
    // CTA touches it, else kept as this CTA's partial for the merge kernel.
    auto flush = [&](int seg) -> bool {
      float* sums = red + 2 * 4 * 8;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float lw = dev::warp_sum(l_thr[h]);
        if (lane == 0) sums[q4 * 8 + h] = lw;
      }
      if (!rendezvous()) return false;
      // no other CTA touches the segment when all its units are in this range
      if (prefix[seg * s.nchunks] >= u0 && prefix[(seg + 1) * s.nchunks] <= u1) {
        const int i = seg / s.Hkv, g = seg - i * s.Hkv;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float l = sums[h] + sums[8 + h] + sums[16 + h] + sums[24 + h];
          const size_t orow = static_cast<size_t>(i) * s.Hq + g * G + h;
          dev::store_out(a, orow * D + dcol, l > 0.f ? acc[h] / l : 0.f);
          if (dcol == h && a.lse) a.lse[orow] = dev::lse_of(m_run[h], l);
        }
      } else {
        float* part = a.partials + static_cast<size_t>(seg + blockIdx.x) * G * partial_stride(D);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          part[h * partial_stride(D) + dcol] = acc[h];
          if (dcol == h) {
            part[h * partial_stride(D) + D] = m_run[h];
            part[h * partial_stride(D) + D + 1] = sums[h] + sums[8 + h] + sums[16 + h] + sums[24 + h];
          }
        }
      }
      return true;
    };

    int pending = -1;  // unit whose O^T is not folded in yet
    for (int j = 0; j < ntiles && ok; ++j) {
      const int st_j = j % nstages;
      if (!wait_or_abort(&B.kv_full[st_j], (j / nstages) & 1, a.status, abort_flag)) { ok = false; break; }
      const TileInfo in = info[st_j];
      if (j == 0 && warp == 2 && lane == 0) dev::trace_first(a.trace, ETA_TRACE_TILE_FIRST);
      if (in.seg != cur_seg) {
        if (pending >= 0) {
          if (!correction(pending) || !flush(cur_seg)) { ok = false; break; }
          pending = -1;
        }
        cur_seg = in.seg;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_run[h] = -INFINITY;
          l_thr[h] = 0.f;
          acc[h] = 0.f;
          tau_h[h] = a.tau[static_cast<size_t>(in.seg) * G + h];
        }
      }
      const int sb = j & 1;
      if (!dev::warp_wait_or_abort(&B.s_full[sb], (j >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      float sv[8];
      tmem_ld8(tmem + tlane + sb * 16, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.s_free[sb]);

      const int rmask = rblk == 0 ? in.mask0 : in.mask1;
      const bool valid = rrow < (rblk == 0 ? in.nrows0 : in.nrows1);
      float x[G];
      float* wmax = red + (j & 1) * 32;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float S = sv[h] * scale;
        const float St = S * dev::logistic(beta * (S - tau_h[h]));
        x[h] = (valid && ((rmask >> h) & 1)) ? St * kLog2e : -INFINITY;
        const float mw = dev::warp_max(x[h]);
        if (lane == 0) wmax[q4 * 8 + h] = mw;
      }
      if (!rendezvous()) { ok = false; break; }
      float alpha[G];
      const int pb = j & 1;
      uint8_t* pbuf = base + L.pbuf + pb * TL::P_BYTES;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = fmaxf(fmaxf(wmax[h], wmax[8 + h]), fmaxf(wmax[16 + h], wmax[24 + h]));
        const float m_new = fmaxf(m_run[h], mt);
        alpha[h] = (m_run[h] == -INFINITY) ? 0.f : dev::fast_exp2(m_run[h] - m_new);
        const float p = (x[h] == -INFINITY) ? 0.f : dev::fast_exp2(x[h] - m_new);
        const uint16_t pbits = dev::f32_to_bf16_rn(p);
        {
          const int kp = row >> 6, tc = row & 63;
          const int off = kp * 2048 + h * 128 + (((tc >> 3) ^ (h & 7)) << 4) + (tc & 7) * 2;
          *reinterpret_cast<uint16_t*>(pbuf + off) = pbits;
        }
        l_thr[h] = fmaf(l_thr[h], alpha[h], __uint_as_float(static_cast<uint32_t>(pbits) << 16));
        m_run[h] = m_new;
      }
      if (in.nrows0 < BR || (BPT == 2 && in.nrows1 < BR)) {
        // rows of a tile that hold no key (past a sequence end, or an absent
        // second block) are zeroed in V so that stale or non-finite bytes
        // there cannot reach the accumulator (0 * inf)
        uint8_t* vb = base + L.stages + st_j * TL::STAGE + TL::V0;
        for (int bi = 0; bi < BPT; ++bi) {
          const int nr = bi == 0 ? in.nrows0 : in.nrows1;
          const int nz = (BR - nr) * 8;  // 16-byte chunks per panel
          for (int c = t - 64; c < 2 * nz; c += 128) {
            const int pnl = c / nz, r = c - pnl * nz;
            *reinterpret_cast<uint4*>(vb + pnl * TL::PANEL + (bi * BR + nr) * 128 + r * 16) =
                make_uint4(0u, 0u, 0u, 0u);
          }
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.p_full[pb]);
      if (pending >= 0 && !correction(pending)) { ok = false; break; }
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
      pending = j;
    }
    if (ok && pending >= 0) ok = correction(pending) && flush(cur_seg);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (t == 0) dev::trace_last(a.trace, ETA_TRACE_ATTEND_LAST);
}

// ------------------------------------------------------------ host side

constexpr size_t kSmemBudget = 224 * 1024;

int pick_stages(const Shape& s) {
  for (int st = kMaxStages; st >= 2; --st)
    if (tc_layout(st, s.nseg * s.nchunks, smem_seqs(s.B)).total <= kSmemBudget) return st;
  return 0;
}

template <int BR, int G>
cudaError_t launch_typed(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const AttendArgs& a,
                         cudaStream_t st, int stages, size_t smem) {
  auto kern = attend_tc_kernel<BR, G>;
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
                          [&] { return cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, a, stages); });
}

template <int BR>
cudaError_t launch_g(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const AttendArgs& a,
                     cudaStream_t st, int stages, size_t smem) {
  switch (a.s.G) {
    case 2: return launch_typed<BR, 2>(tk, tv, tq, a, st, stages, smem);
    case 4: return launch_typed<BR, 4>(tk, tv, tq, a, st, stages, smem);
    case 8: return launch_typed<BR, 8>(tk, tv, tq, a, st, stages, smem);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool attend_tc_supported(const Shape& s) {
  const long long rows = s.num_pages ? static_cast<long long>(s.num_pages) * s.Hkv * s.b
                                     : static_cast<long long>(s.nseg) * s.max_ctx;
  return s.elt == 2 && s.d == 128 && (s.b == 64 || s.b == 128) && (s.G == 2 || s.G == 4 || s.G == 8) &&
         rows < (1ll << 31) && static_cast<long long>(s.B) * s.Hq < (1ll << 31);
}

size_t attend_tc_smem(const Shape& s) {
  const int st = pick_stages(s);
  return st ? tc_layout(st, s.nseg * s.nchunks, smem_seqs(s.B)).total : 0;
}

cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t st) {
  const int stages = pick_stages(a.s);
  if (stages == 0) return cudaErrorInvalidConfiguration;
  const size_t smem = tc_layout(stages, a.s.nseg * a.s.nchunks, smem_seqs(a.s.B)).total;
  CUtensorMap tk, tv, tq;
  const uint64_t rows = a.s.num_pages ? static_cast<uint64_t>(a.s.num_pages) * a.s.Hkv * a.s.b
                                      : static_cast<uint64_t>(a.s.nseg) * a.s.max_ctx;
  if (!make_map(&tk, a.k, rows, a.s.b) || !make_map(&tv, a.v, rows, a.s.b) ||
      !make_map(&tq, a.q, static_cast<uint64_t>(a.s.B) * a.s.Hq, NQ))
    return cudaErrorInvalidValue;
  return a.s.b == 64 ? launch_g<64>(tk, tv, tq, a, st, stages, smem) : launch_g<128>(tk, tv, tq, a, st, stages, smem);
}

}  // namespace eta
