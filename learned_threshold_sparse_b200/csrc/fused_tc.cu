// The whole decode step in one persistent kernel on the 5th-generation tensor
// cores: threshold, block screen, split-KV attention over the admitted
// GQA-union blocks, and the merge of the split partials.  bf16 K/V, d = 128,
// fp16 block metadata, the always-loaded window on (or the screen off).
//
// Source: Elastic Threshold Attention,
//   section 1 / App. D.1, 4.7 / D.2, G.1   tau~ = w_tau . q + b_tau - a, or c - a,
//   section 3.1-3.2, 4.3, App. F.1        O(1) bound per (block, head) from
//                                          (mu_B, sigma_B, M_B), compared with tau~,
//   section 4.8                            the tail block and the lwb blocks before it
//                                          always loaded,
//   App. F.1 step 2                        GQA union: a block is fetched once for the
//                                          heads that admitted it (head mask),
//   App. F.2                               fp32 bound, scores and softmax state, bf16
//                                          operands on the tensor cores,
//   App. G.1                               S~ = S sigmoid(beta (S - tau~)), weights e^S~,
//   section 3.2, App. F.3                  split-KV partials merged associatively,
//   App. F.4                               the tail block's rows >= seq_len masked.
//
// Work unit: a positional chunk of C consecutive blocks of one (sequence, KV
// head) segment; the chunks that exist (blocks below the sequence length) are
// numbered in (sequence, KV head, block) order and cut into one contiguous
// slice per CTA (one CTA per SM, all resident together).  Every CTA runs:
//   1. screen    the slice's block metadata is staged in the (still idle)
//                K/V ring by asynchronous copies from all threads, then all
//                six warps screen it, a warp per chunk: the G heads'
//                thresholds, the bound of every block for each head,
//                and the chunk's admitted blocks, ascending, with head masks
//                (list and count written to the workspace, where the
//                selection export and the other CTAs read them); then the
//                slice's admitted total is published (then one release
//                increment of an arrival counter);
//   2. exchange  the producer warp waits (bounded) for the counter to reach
//                the grid size and reads all slice totals.  The admitted
//                units of all lists, in list order, form one sequence of U
//                units; this CTA takes the equal range [U c / N, U (c + 1) / N);
//   3. attention as in the split kernel: warp 0 walks the range through the
//                lists of the slices it covers and copies each tile's K, V
//                and query rows (TMA, 128-byte swizzle) into a 3-stage ring,
//                warp 1 issues S^T = K Q^T and O^T = V^T P^T into tensor
//                memory, warps 2-5 gate, run the online softmax, write P and
//                fold O^T; an END entry in the ring closes the range;
//   4. merge     a segment whose units all lie in this range is written out
//                directly; a segment spread over CTAs c_first..c_last leaves
//                one partial per CTA, each announced by one atomic on the
//                segment's counter, and the CTA whose announcement completes
//                the set (every CTA of the span with a non-empty range) merges
//                the pieces in CTA order, at its end, with the pieces copied
//                into the then idle K/V ring.
// The pages screen and attend in one pass over positional chunks (section
// 3.2); here the screen of a slice runs before its streaming so that no
// memory round trip of the screen sits behind the K/V stream.  Ranges, tile
// order and merge order follow from the admitted sets alone, so results do
// not depend on timing.  The only cross-CTA wait is the exchange, and it is
// bounded: if some CTA of the grid is not resident the step ends with the
// timeout status instead of hanging.
//
// Counters live in the workspace's control region and are back at zero when
// a step completes: the last CTA to finish clears the slice totals and the
// arrival counter, and the merger of a segment clears that segment's
// counter.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "attend_common.cuh"
#include "tc_common.cuh"

namespace eta {
namespace {

using dev::wait_or_abort;
using namespace tc;

constexpr int D = 128;
constexpr int NQ = 16;              // N of both MMAs
constexpr int kWarps = 6;
constexpr int kThreads = kWarps * 32;
constexpr int kTmemCols = 64;       // S buffers at columns 0, 16; O buffers at 32, 48
constexpr int kStages = 3;
constexpr int TR = 128;             // key rows per tile
constexpr float kLog2e = 1.4426950408889634f;

struct Tile {
  static constexpr int PANEL = TR * 128;
  static constexpr int K0 = 0, K1 = PANEL, V0 = 2 * PANEL, V1 = 3 * PANEL, Q0 = 4 * PANEL, Q1 = 4 * PANEL + 2048;
  static constexpr int STAGE = 4 * PANEL + 4096;
  static constexpr int P_BYTES = NQ * TR * 2;
};

// Pieces of a segment spread over several CTAs (compiled for the host as
// well).  A CTA's range [u0, u1) splits into runs of consecutive units of one
// segment.  A run is shared when the segment has units before u0 (then the
// run starts at u0) or at or after u1 (then it ends at u1); a shared run
// leaves a partial in slot 0 of its CTA if it holds u0, else in slot 1, and
// announces it with one atomic add to the segment's 64-bit counter:
//   bits 0-15 arrivals, bit 16 the first piece is in, bit 17 the last piece
//   is in, bit 18 the first piece's slot, bits 32-47 the first piece's CTA,
//   bits 48-63 the last piece's CTA.
// Every CTA between the first and the last piece's with a non-empty range
// holds exactly one piece, in its slot 0 (its range starts inside the
// segment), so the announcement that completes the set is recognised from
// the counter alone.
// ETA_PIECES_BEGIN
constexpr int kModeShared = 1;  // other CTAs hold units of the segment: write a partial
constexpr int kModeSlot1 = 2;   // partial slot 1 (the run did not contain the range's first unit)
constexpr int kModeFirst = 4;   // the run holds the segment's first unit
constexpr int kModeLast = 8;    // the run holds the segment's last unit

__host__ __device__ inline int run_mode(bool holds_u0, bool shared_start, bool shared_end) {
  int mode = (shared_start ? 0 : kModeFirst) | (shared_end ? 0 : kModeLast);
  if (shared_start || shared_end) mode |= kModeShared | (holds_u0 ? 0 : kModeSlot1);
  return mode;
}

__host__ __device__ inline unsigned long long piece_announcement(int mode, int cta) {
  const unsigned long long c64 = static_cast<unsigned long long>(cta);
  unsigned long long add = 1ull;
  if (mode & kModeFirst) add += (1ull << 16) + ((mode & kModeSlot1) ? (1ull << 18) : 0ull) + (c64 << 32);
  if (mode & kModeLast) add += (1ull << 17) + (c64 << 48);
  return add;
}

// Fields of a counter value: are both end pieces in, and which CTAs / slot.
struct PieceSet {
  bool ends_in;
  int c_first, c_last, slot_first, arrivals;
};
__host__ __device__ inline PieceSet piece_set(unsigned long long v) {
  PieceSet p;
  p.ends_in = (v & (1ull << 16)) && (v & (1ull << 17));
  p.c_first = static_cast<int>((v >> 32) & 0xffffull);
  p.c_last = static_cast<int>(v >> 48);
  p.slot_first = static_cast<int>((v >> 18) & 1ull);
  p.arrivals = static_cast<int>(v & 0xffffull);
  return p;
}

// Is the set complete: both end pieces in, and one arrival per CTA of the
// span with a non-empty range (us: the step's unit split over nctas CTAs).
// A counter naming CTAs outside the grid (left by a step that did not
// finish) never completes, and *stale says so.
template <class Split>
__host__ __device__ inline bool piece_set_complete(const PieceSet& p, const Split& us, int nctas, bool* stale) {
  *stale = false;
  if (!p.ends_in) return false;
  if (p.c_last < p.c_first || p.c_last >= nctas) {
    *stale = true;
    return false;
  }
  int expect = 0;
  for (int c = p.c_first; c <= p.c_last; ++c) expect += us.owns_any(static_cast<unsigned>(c)) ? 1 : 0;
  return p.arrivals == expect;
}
// ETA_PIECES_END

// A ring entry: the tile's segment (-1: END), per block of the tile the
// admitting heads and the rows present, and the mode of the run this entry
// closes (a new segment's first tile, or END).
struct FInfo {
  int seg, mask0, mask1, nrows0, nrows1, prev_mode;
};

constexpr int kEntStage = 256;  // list entries the producer stages per round trip

struct Layout {
  size_t stages, pbuf, bars, info, red, seqs, cseq, prefix, own, ent, spre, sseg, scid, misc, total;
};

__host__ __device__ inline size_t align_to(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Offsets relative to a 1024-byte aligned base; nctas = grid size.
__host__ __device__ inline Layout fused_layout(int nctas) {
  Layout L;
  size_t off = 0;
  L.stages = off;
  off += static_cast<size_t>(kStages) * Tile::STAGE;
  L.pbuf = off;
  off += 2 * static_cast<size_t>(Tile::P_BYTES);
  L.bars = off = align_to(off, 16);
  off += (2 * kStages + 12) * sizeof(uint64_t);
  L.info = off = align_to(off, 16);
  off += kStages * sizeof(FInfo);
  L.red = off = align_to(off, 16);
  off += (2 * 4 * 8 + 4 * 8) * sizeof(float);
  L.seqs = off = align_to(off, 16);
  off += kFusedMaxSeqs * sizeof(int);
  L.cseq = off = align_to(off, 16);
  off += (kFusedMaxSeqs + 1) * sizeof(int);
  L.prefix = off = align_to(off, 16);
  off += static_cast<size_t>(nctas + 1) * sizeof(int);
  L.own = off = align_to(off, 16);
  off += kFusedMaxSlice * sizeof(int);
  L.ent = off = align_to(off, 16);
  off += kEntStage * sizeof(int);
  L.spre = off = align_to(off, 16);
  off += (kFusedMaxSlice + 1) * sizeof(int);
  L.sseg = off = align_to(off, 16);
  off += kFusedMaxSlice * sizeof(int);
  L.scid = off = align_to(off, 16);
  off += kFusedMaxSlice * sizeof(int);
  L.misc = off = align_to(off, 16);
  off += 128;
  L.total = align_to(off, 128) + 1024;  // + slack to align the dynamic base to 1024
  return L;
}

struct Bars {
  uint64_t* kv_full;   // [kStages]  producer -> MMA, softmax   (tx bytes; END: plain arrive)
  uint64_t* kv_empty;  // [kStages]  MMA commit -> producer
  uint64_t* s_full;    // [2]        MMA commit -> softmax
  uint64_t* s_free;    // [2]        softmax (4 warps) -> MMA
  uint64_t* p_full;    // [2]        softmax (4 warps) -> MMA
  uint64_t* o_full;    // [2]        MMA commit -> softmax
  uint64_t* o_free;    // [2]        softmax (4 warps) -> MMA
  uint64_t* rv;        // [1]        softmax-warp rendezvous (4 warps)
  uint64_t* done;      // [1]        final MMA commit
};

__device__ __forceinline__ unsigned ld_acquire(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(unsigned* p, unsigned v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ unsigned long long atom_add_acq_rel64(unsigned long long* p, unsigned long long v) {
  unsigned long long old;
  asm volatile("atom.add.acq_rel.gpu.global.u64 %0, [%1], %2;" : "=l"(old) : "l"(p), "l"(v) : "memory");
  return old;
}

__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// Chunks that exist, numbered in (sequence, KV head, block) order: sequence
// i owns Hkv nch(i) consecutive numbers from cseq[i] on.
struct Chunks {
  const int* seqT;  // clamped lengths [B]
  const int* cseq;  // [B + 1]
  int B, Hkv, b, C;
  __device__ __forceinline__ int nch(int i) const {
    const int nb = (seqT[i] + b - 1) / b;
    return (nb + C - 1) / C;
  }
  // chunk number r (< cseq[B]) -> segment and chunk index inside it
  __device__ __forceinline__ void locate(int r, int& seg, int& cidx) const {
    int lo = 0, hi = B;  // largest i with cseq[i] <= r; it has chunks since cseq[i + 1] > r
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (cseq[mid] <= r) lo = mid; else hi = mid;
    }
    const int n = nch(lo), w = r - cseq[lo];
    const int g = w / n;
    seg = lo * Hkv + g;
    cidx = w - g * n;
  }
  __device__ __forceinline__ int first(int seg) const {
    const int i = seg / Hkv;
    return cseq[i] + (seg - i * Hkv) * nch(i);
  }
};

template <int BR, int G>
__global__ void __launch_bounds__(kThreads, 1)
    fused_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tq, FusedArgs a) {
  using TL = Tile;
  constexpr int BPT = TR / BR;  // blocks per tile
  constexpr int CPL = D / 32;   // coordinates per lane in the screen
  constexpr int NV = 2 * G;     // values per block: <q_h, mu>, sum q_h^2 sigma^2
  constexpr int NB = 32 / NV;   // blocks reduced together
  constexpr unsigned kFullMask = (1u << G) - 1u;
  extern __shared__ uint8_t smem_raw[];
  const Shape& s = a.s;
  const int N = gridDim.x, cta = blockIdx.x;
  const int C = s.chunk;
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw);
  const Layout L = fused_layout(N);

  uint64_t* bars = reinterpret_cast<uint64_t*>(base + L.bars);
  Bars B;
  B.kv_full = bars;
  B.kv_empty = bars + kStages;
  B.s_full = bars + 2 * kStages;
  B.s_free = B.s_full + 2;
  B.p_full = B.s_free + 2;
  B.o_full = B.p_full + 2;
  B.o_free = B.o_full + 2;
  B.rv = B.o_free + 2;
  B.done = B.rv + 1;
  FInfo* info = reinterpret_cast<FInfo*>(base + L.info);
  float* red = reinterpret_cast<float*>(base + L.red);  // [2][4][8] tile maxima, then [4][8] flush sums
  int* seqT = reinterpret_cast<int*>(base + L.seqs);
  int* cseq = reinterpret_cast<int*>(base + L.cseq);
  int* P = reinterpret_cast<int*>(base + L.prefix);     // [N + 1] admitted units before slice c
  int* own = reinterpret_cast<int*>(base + L.own);      // admitted units of this slice's chunks
  int* ent_s = reinterpret_cast<int*>(base + L.ent);    // producer: staged list entries
  int* spre = reinterpret_cast<int*>(base + L.spre);    // producer: units before chunk k of the current slice
  int* sseg = reinterpret_cast<int*>(base + L.sseg);    // producer: segment of chunk k of the current slice
  int* scid = reinterpret_cast<int*>(base + L.scid);    // producer: chunk index (in its segment) of chunk k
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.misc + 4);
  int* pm = reinterpret_cast<int*>(base + L.misc + 64);     // merges to run at the end: [count, (seg, c_first, c_last, slot) x 2]
  int* mbatch = reinterpret_cast<int*>(base + L.misc + 100);  // merge batch: [pieces, next CTA]
  int* issued_parity = reinterpret_cast<int*>(base + L.misc + 32);
  int* units_total = reinterpret_cast<int*>(base + L.misc + 48);  // U, set by the producer before its first tile

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  if (t == 0) {
    for (int k = 0; k < kStages; ++k) {
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
    *reinterpret_cast<int*>(base + L.misc + 64) = 0;
    dev::fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  // P rows >= G stay zero for the whole kernel.
  for (int x = t; x < 2 * TL::P_BYTES / 16; x += kThreads)
    reinterpret_cast<uint4*>(base + L.pbuf)[x] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tq)) : "memory");
  }
  // Nothing written by the stream's previous kernel is read before this
  // point.  The next kernel may be scheduled now: its CTAs start only once
  // every CTA of this grid has passed here, so they never keep one of ours
  // from becoming resident, and it reads nothing of ours before this grid
  // has completed.
  dev::pdl_trigger();
  dev::pdl_wait();
  if (t == 0) dev::trace_first(a.trace, ETA_TRACE_FUSED_FIRST);

  for (int x = t; x < s.B; x += kThreads) {
    int tt = a.seq_lens[x];
    if (tt < 0 || tt > s.max_ctx) {
      if (cta == 0) atomicOr(a.status, kStatusRange);
      tt = tt < 0 ? 0 : s.max_ctx;
    }
    seqT[x] = tt;
  }
  __syncthreads();
  if (warp == 0) {  // chunk numbers: cseq[i] = sum over i' < i of Hkv nch(i')
    const int per = (s.B + 31) / 32;
    const int lo = min(s.B, lane * per), hi = min(s.B, lo + per);
    int sum = 0;
    for (int x = lo; x < hi; ++x) {
      const int nb = (seqT[x] + s.b - 1) / s.b;
      sum += s.Hkv * ((nb + C - 1) / C);
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int run = incl - sum;
    for (int x = lo; x < hi; ++x) {
      cseq[x] = run;
      const int nb = (seqT[x] + s.b - 1) / s.b;
      run += s.Hkv * ((nb + C - 1) / C);
    }
    if (lane == 31) cseq[s.B] = incl;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Chunks ch{seqT, cseq, s.B, s.Hkv, s.b, C};
  const int NC = cseq[s.B];
  const dev::UnitSplit slices(static_cast<unsigned>(NC), static_cast<unsigned>(N));
  const int r_lo = static_cast<int>(slices.start(cta));
  const int nslice = static_cast<int>(slices.start(cta + 1)) - r_lo;  // <= kFusedMaxSlice (host)

  // ============================================================ 1. screen
  {
    // empty sequences have no chunk: their outputs are 0, lse -inf
    if (warp == 0) {
      for (int i = cta; i < s.B; i += N) {
        if (seqT[i] != 0) continue;
        for (int x = lane; x < s.Hq * D; x += 32) dev::store_out_slot(a.out, s.elt, static_cast<size_t>(i) * s.Hq * D + x, 0.f);
        for (int x = lane; x < s.Hq; x += 32)
          if (a.lse) a.lse[static_cast<size_t>(i) * s.Hq + x] = -INFINITY;
      }
    }
    float qr[G][CPL], q2[G][CPL], tau_h[G], qn_h[G];
    int cseg = -1;
    const bool learned = a.tau_mode == ETA_TAU_LEARNED;
    const float scale = a.scale, z = a.z;
    const bool strict = isinf(z);
    const int vb = lane / NV, vq = lane % NV;
    // The K/V ring is idle until the exchange.  A round of up to R chunks of
    // the slice has its metadata staged there: mu and sigma rows and the
    // block norms, by asynchronous copies spread over all threads (16 bytes
    // per row piece, 4 per norm), all in flight together.
    uint8_t* scr = base + L.stages;
    const int mstride = C * D * 2;  // bytes of one chunk's mu (or sigma) rows
    const int R = static_cast<int>(static_cast<size_t>(kStages) * TL::STAGE / (2 * mstride + C * sizeof(float)));
    float* mn_s = reinterpret_cast<float*>(scr + static_cast<size_t>(R) * 2 * mstride);
    const int lc = __ffs(C) - 1;  // C is a power of two
    // rows of chunk number r: its segment, first block, blocks present and screened ones
    auto chunk_rows = [&](int r, int& seg, int& cidx, int& nloc, int& nscreen) {
      ch.locate(r, seg, cidx);
      const int nb = (seqT[seg / s.Hkv] + s.b - 1) / s.b;
      const int blk0 = cidx * C;
      nloc = min(C, nb - blk0);
      const int first_forced = a.screen_enabled ? max(0, nb - 1 - a.lwb) : 0;
      nscreen = max(0, min(nloc, first_forced - blk0));
    };
    // the heads' queries, thresholds and norms of segment seg (all loads
    // issued first); tau~ also goes to the workspace for the softmax of
    // whichever CTA streams this segment's units
    auto compute_tau = [&](int i, int g, int seg) {
      uint2 qu[G];
      float wv[G][CPL], bc[G];  // w_tau is only 4-byte aligned: scalar loads
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const int hq = g * G + h;
        const size_t qo = (static_cast<size_t>(i) * s.Hq + hq) * D + lane * CPL;
        qu[h] = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.q) + qo);
#pragma unroll
        for (int c = 0; c < CPL; ++c) wv[h][c] = learned ? __ldg(a.w_tau + static_cast<size_t>(hq) * D + lane * CPL + c) : 0.f;
        bc[h] = learned ? a.b_tau[hq] : a.c_tau[hq];
      }
#pragma unroll
      for (int h = 0; h < G; ++h) {
        qr[h][0] = dev::bf16_lo(qu[h].x);
        qr[h][1] = dev::bf16_hi(qu[h].x);
        qr[h][2] = dev::bf16_lo(qu[h].y);
        qr[h][3] = dev::bf16_hi(qu[h].y);
        float tw = 0.f, qq = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
          q2[h][c] = qr[h][c] * qr[h][c];
          qq = fmaf(qr[h][c], qr[h][c], qq);
          tw = fmaf(wv[h][c], qr[h][c], tw);
        }
        tw = dev::warp_sum(tw);
        qq = dev::warp_sum(qq);
        tau_h[h] = (learned ? tw + bc[h] : bc[h]) - a.offset_a;
        qn_h[h] = sqrtf(qq);
      }
      if (lane < G) {
        float tv_ = tau_h[0];
#pragma unroll
        for (int h = 1; h < G; ++h)
          if (lane == h) tv_ = tau_h[h];
        a.tau[static_cast<size_t>(seg) * G + lane] = tv_;
      }
    };
    int* r_nsc = sseg;  // per chunk of the round: blocks screened, first metadata row (the
    int* r_row = scid;  // producer's slice tables are not in use yet)
    for (int r0 = 0; r0 < nslice; r0 += R) {
      const int nr = min(R, nslice - r0);
      if (a.screen_enabled) {
        if (warp == 0) {
          for (int k = lane; k < nr; k += 32) {
            int seg, cidx, nloc, nsc;
            chunk_rows(r_lo + r0 + k, seg, cidx, nloc, nsc);
            r_nsc[k] = nsc;
            r_row[k] = seg * s.nbmax + cidx * C;  // < 2^31: the cache holds fewer rows
          }
        }
        __syncthreads();
        const int per_chunk = 32 << lc;  // 16-byte pieces of mu and sigma rows of a full chunk
        for (int x = t; x < nr * per_chunk; x += kThreads) {
          const int k = x >> (5 + lc), r = x & (per_chunk - 1);
          const int arr = r >> (4 + lc), j = (r >> 4) & (C - 1), pc = r & 15;
          if (j < r_nsc[k]) {
            const uint8_t* src = static_cast<const uint8_t*>(arr ? a.sigma : a.mu) +
                                 (static_cast<size_t>(r_row[k]) + j) * D * 2 + pc * 16;
            dev::cp_async16(scr + static_cast<size_t>(k) * 2 * mstride + arr * mstride + j * D * 2 + pc * 16, src);
          }
        }
        for (int x = t; x < nr * C; x += kThreads) {
          const int k = x >> lc, j = x & (C - 1);
          if (j < r_nsc[k]) dev::cp_async4(&mn_s[x], a.max_norm + r_row[k] + j);
        }
        dev::cp_async_commit();
      }
      // the threshold of each warp's first chunk while the copies fly
      if (r0 + warp < r0 + nr) {
        int seg, cidx, nloc, nsc;
        chunk_rows(r_lo + r0 + warp, seg, cidx, nloc, nsc);
        if (seg != cseg) {
          cseg = seg;
          const int i = seg / s.Hkv, g = seg - i * s.Hkv;
          compute_tau(i, g, seg);
        }
      }
      if (a.screen_enabled) dev::cp_async_wait<0>();
      __syncthreads();  // every thread's copies have landed
      for (int k = r0 + warp; k < r0 + nr; k += kWarps) {
        int seg, cidx, nloc, nscreen;
        chunk_rows(r_lo + k, seg, cidx, nloc, nscreen);
        const int i = seg / s.Hkv, g = seg - i * s.Hkv;
        const int blk0 = cidx * C;
        if (seg != cseg) {
          cseg = seg;
          compute_tau(i, g, seg);
        }
        // head masks of the chunk's blocks: lane l <-> block blk0 + l
        unsigned mymask = lane < nloc ? kFullMask : 0u;  // forced window / screen off
        if (nscreen > 0) {
          {
            const uint8_t* mu_s = scr + static_cast<size_t>(k - r0) * 2 * mstride;
            const uint8_t* sg_s = mu_s + mstride;
            const float* mn = mn_s + (k - r0) * C;
            for (int gb = 0; gb < nscreen; gb += NB) {
              float v[32];
#pragma unroll
              for (int u = 0; u < NB; ++u) {
                const int lb = min(gb + u, nscreen - 1);
                const uint2 m2 = *reinterpret_cast<const uint2*>(mu_s + (lb * D + lane * CPL) * 2);
                const uint2 s2b = *reinterpret_cast<const uint2*>(sg_s + (lb * D + lane * CPL) * 2);
                float mu[CPL], s2[CPL];
                mu[0] = dev::fp16_to_f32(static_cast<uint16_t>(m2.x & 0xffffu));
                mu[1] = dev::fp16_to_f32(static_cast<uint16_t>(m2.x >> 16));
                mu[2] = dev::fp16_to_f32(static_cast<uint16_t>(m2.y & 0xffffu));
                mu[3] = dev::fp16_to_f32(static_cast<uint16_t>(m2.y >> 16));
                const float g0 = dev::fp16_to_f32(static_cast<uint16_t>(s2b.x & 0xffffu));
                const float g1 = dev::fp16_to_f32(static_cast<uint16_t>(s2b.x >> 16));
                const float g2 = dev::fp16_to_f32(static_cast<uint16_t>(s2b.y & 0xffffu));
                const float g3 = dev::fp16_to_f32(static_cast<uint16_t>(s2b.y >> 16));
                s2[0] = g0 * g0;
                s2[1] = g1 * g1;
                s2[2] = g2 * g2;
                s2[3] = g3 * g3;
#pragma unroll
                for (int h = 0; h < G; ++h) {
                  float dot = 0.f, sq = 0.f;
#pragma unroll
                  for (int c = 0; c < CPL; ++c) {
                    dot = fmaf(qr[h][c], mu[c], dot);
                    sq = fmaf(q2[h][c], s2[c], sq);
                  }
                  v[u * NV + h] = dot;
                  v[u * NV + G + h] = sq;
                }
              }
              const float redv = dev::transpose_reduce32<32>(v, lane);
              const float sqv = __shfl_down_sync(0xffffffffu, redv, G);  // sum q^2 sigma^2 of the same (block, head)
              const int lb = gb + vb;
              bool pass = false;
              if (vq < G && lb < nscreen) {
                float tq = tau_h[0], qn = qn_h[0];
#pragma unroll
                for (int h = 1; h < G; ++h)
                  if (vq == h) { tq = tau_h[h]; qn = qn_h[h]; }
                const float geo = qn * mn[lb];
                const float spread = strict ? geo : fminf(geo, z * sqrtf(sqv));
                pass = scale * (redv + spread) >= tq;
              }
              const unsigned bal = __ballot_sync(0xffffffffu, pass);
              // block gb + u's head bits sit at lanes u NV .. u NV + G - 1
#pragma unroll
              for (int u = 0; u < NB; ++u) {
                const int blk = gb + u;
                if (lane == blk && blk < nscreen) mymask = (bal >> (u * NV)) & kFullMask;
              }
            }
          }
        }
        // ascending admitted list of the chunk and its count
        const unsigned adm = __ballot_sync(0xffffffffu, mymask != 0u);
        if (mymask != 0u)
          a.chunk_list[static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(cidx) * C +
                       __popc(adm & ((1u << lane) - 1u))] = (blk0 + lane) | static_cast<int>(mymask << kEntryBlockBits);
        if (lane == 0) {
          a.chunk_count[static_cast<size_t>(seg) * s.nchunks + cidx] = __popc(adm);
          own[k] = __popc(adm);
        }
      }
      fence_proxy_async();  // generic reads of the staging area come before any later copy into it
      __syncthreads();
    }
    __threadfence();
    __syncthreads();
    if (t == 0) {
      int total = 0;
      for (int k = 0; k < nslice; ++k) total += own[k];
      a.flags[cta] = static_cast<unsigned>(total) + 1u;
      __threadfence();
      red_release_add(a.arrived, 1u);
    }
  }

  if (warp == 0) {
    // ============================================================ 2. exchange, 3. producer
    bool ok = true;
    {
      // wait (bounded) until every CTA has published its slice total: the
      // warp polls one counter, then reads all totals, eight loads in
      // flight per lane (acquire: the lists published with them are visible)
      const long long t0 = clock64();
      for (;;) {
        const unsigned n = ld_acquire(a.arrived);
        if (__all_sync(0xffffffffu, n >= static_cast<unsigned>(N))) break;
        if (clock64() - t0 > dev::kWaitCycles) {
          ok = false;
          break;
        }
        __nanosleep(100);
      }
      const int per = (N + 31) / 32;
      const int lo = min(N, lane * per), hi = min(N, lo + per);
      int sum = 0;
      for (int x0 = lo; x0 < hi && ok; x0 += 8) {
        unsigned v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = x0 + u < hi ? __ldcg(a.flags + x0 + u) : 1u;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (x0 + u < hi) {
            if (v[u] == 0u) ok = false;  // published (the counter says so) yet zero: a stale control region
            P[x0 + u] = static_cast<int>(v[u]) - 1;
            sum += static_cast<int>(v[u]) - 1;
          }
        }
      }
      ok = __all_sync(0xffffffffu, ok ? 1 : 0) != 0;
      int incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - sum;
      for (int x = lo; x < hi; ++x) {
        const int c = P[x];
        P[x] = run;
        run += c;
      }
      if (lane == 31) P[N] = incl;
      __syncwarp();
    }
    if (!ok) {
      if (lane == 0) {
        atomicOr(a.status, kStatusTimeout);
        *abort_flag = 1;
      }
    } else {
      const int U = P[N];
      if (lane == 0) *units_total = U;  // read by the softmax warps after the ring's first entry
      const dev::UnitSplit us(static_cast<unsigned>(U), static_cast<unsigned>(N));
      const int u0 = static_cast<int>(us.start(cta)), u1 = static_cast<int>(us.start(cta + 1));
      const KvLayout lay{a.block_table, s.Hkv, s.b, s.max_ctx, s.nbmax, s.num_pages};
      // admitted count of chunk number r, read by one lane
      auto chunk_count = [&](int r, int sl) -> int {
        if (sl == cta) return own[r - r_lo];
        int sg, ci;
        ch.locate(r, sg, ci);
        return __ldcg(a.chunk_count + static_cast<size_t>(sg) * s.nchunks + ci);
      };
      // units in the chunks numbered below r (warp-wide)
      auto units_before = [&](int r) -> int {
        if (r >= NC) return U;
        const int sl = static_cast<int>(slices.owner(static_cast<unsigned>(r)));
        const int lo = static_cast<int>(slices.start(sl));
        int sum = 0;
        for (int x = lo + lane; x < r; x += 32) sum += chunk_count(x, sl);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        return P[sl] + sum;
      };

      int stage = 0;
      uint32_t phase = 0;
      FInfo pend{-1, 0, 0, 0, 0, 0};
      int prow[2] = {0, 0};
      int npend = 0;
      int carry = 0;  // mode of the run closed by the next ring entry
      // (lane 0) put the pending tile into the ring
      auto emit = [&]() -> bool {
        if (!wait_or_abort(&B.kv_empty[stage], phase ^ 1u, a.status, abort_flag)) return false;
        pend.prev_mode = carry;
        carry = 0;
        info[stage] = pend;
        const uint32_t st = base_u32 + static_cast<uint32_t>(L.stages + stage * TL::STAGE);
        dev::mbar_arrive_expect_tx(&B.kv_full[stage], static_cast<uint32_t>(npend * 4 * BR * 128 + 4096));
        for (int x = 0; x < npend; ++x) {
          const int krow = prow[x];
          const uint32_t ro = static_cast<uint32_t>(x * BR * 128);
          tma_load_2d(st + TL::K0 + ro, &tk, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::K1 + ro, &tk, 64, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V0 + ro, &tv, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V1 + ro, &tv, 64, krow, &B.kv_full[stage]);
        }
        const int qrow = pend.seg * s.G;
        tma_load_2d(st + TL::Q0, &tq, 0, qrow, &B.kv_full[stage]);
        tma_load_2d(st + TL::Q1, &tq, 64, qrow, &B.kv_full[stage]);
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
        npend = 0;
        return true;
      };
      // (warp) flush the pending tile
      auto emit_pending = [&]() -> bool {
        int r = 1;
        if (lane == 0 && npend > 0) r = emit() ? 1 : 0;
        return __shfl_sync(0xffffffffu, r, 0) != 0;
      };
      // (warp) the mode of the run of segment rseg that ends here
      auto close_run = [&](int rseg, bool first_run, bool at_u1) -> int {
        const int f = ch.first(rseg);
        const bool shared_start = first_run && units_before(f) < u0;
        const bool shared_end = at_u1 && units_before(f + ch.nch(rseg / s.Hkv)) > u1;
        return run_mode(first_run, shared_start, shared_end);
      };

      int run_seg = -1;
      bool first_run = true;
      if (u0 < u1) {
        int sl = 0, hi = N;  // slice holding unit u0: the last with P[sl] <= u0
        while (hi - sl > 1) {
          const int mid = (sl + hi) >> 1;
          if (P[mid] <= u0) sl = mid; else hi = mid;
        }
        int u = u0;
        for (; ok && u < u1 && sl < N; ++sl) {
          const int rlo = static_cast<int>(slices.start(sl));
          const int n = static_cast<int>(slices.start(sl + 1)) - rlo;
          // the slice's chunk counts (lane l: chunks l and l + 32), their
          // segments and chunk indices, and the running count before each
          int cnt0 = 0, cnt1 = 0;
          if (lane < n) {
            cnt0 = chunk_count(rlo + lane, sl);
            ch.locate(rlo + lane, sseg[lane], scid[lane]);
          }
          if (lane + 32 < n) {
            cnt1 = chunk_count(rlo + lane + 32, sl);
            ch.locate(rlo + lane + 32, sseg[lane + 32], scid[lane + 32]);
          }
          if (dev::chunk_count_faults(C, cnt0) | dev::chunk_count_faults(C, cnt1)) cnt0 = -1;
          if (__any_sync(0xffffffffu, cnt0 < 0)) {
            if (lane == 0) atomicOr(a.status, kStatusList);
            ok = false;
            break;
          }
          int i0 = cnt0, i1 = cnt1;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int y0 = __shfl_up_sync(0xffffffffu, i0, o);
            const int y1 = __shfl_up_sync(0xffffffffu, i1, o);
            if (lane >= o) { i0 += y0; i1 += y1; }
          }
          const int tot0 = __shfl_sync(0xffffffffu, i0, 31);
          const int tot = tot0 + __shfl_sync(0xffffffffu, i1, 31);
          if (lane < n) spre[lane] = i0 - cnt0;
          if (lane + 32 < n) spre[lane + 32] = tot0 + i1 - cnt1;
          if (lane == 0) spre[n] = tot;
          __syncwarp();
          if (tot != P[sl + 1] - P[sl]) {  // totals and lists disagree
            if (lane == 0) atomicOr(a.status, kStatusList);
            ok = false;
            break;
          }
          // chunk k of the slice holding position pos (the last with spre[k] <= pos)
          auto chunk_of = [&](int pos) -> int {
            int lo = 0, hi = n;
            while (hi - lo > 1) {
              const int mid = (lo + hi) >> 1;
              if (spre[mid] <= pos) lo = mid; else hi = mid;
            }
            return lo;
          };
          const int pa = u - P[sl], pb = min(u1, P[sl + 1]) - P[sl];  // this range's positions in the slice
          for (int bb = pa; bb < pb && ok; bb += kEntStage) {
            // stage up to kEntStage entries with independent loads (one round trip)
            const int m = min(kEntStage, pb - bb);
            for (int x = lane; x < m; x += 32) {
              const int k = chunk_of(bb + x);
              ent_s[x] = __ldcg(a.chunk_list + static_cast<size_t>(sseg[k]) * s.list_stride +
                                static_cast<size_t>(scid[k]) * C + (bb + x - spre[k]));
            }
            __syncwarp();
            for (int k = chunk_of(bb); k < n && spre[k] < bb + m && ok; ++k) {
              const int xa = max(spre[k], bb) - bb, xb = min(spre[k + 1], bb + m) - bb;
              if (xb <= xa) continue;
              const int seg = sseg[k], cidx = scid[k];
              if (seg != run_seg) {
                if (run_seg >= 0) {
                  if (!emit_pending()) { ok = false; break; }
                  carry = close_run(run_seg, first_run, false);
                  first_run = false;
                }
                run_seg = seg;
              }
              const int T = seqT[seg / s.Hkv];
              const int nblk = (T + s.b - 1) / s.b;
              const int nn = xb - xa;  // <= C <= 32
              const int e = lane < nn ? ent_s[xa + lane] : 0;
              const int eb = e & kMaxBlocksPerSeq;
              const int up = __shfl_up_sync(0xffffffffu, eb, 1);
              // the entry before the first one, when it is in the same chunk and staged
              const int first_prev = (xa > 0 && bb + xa > spre[k]) ? (ent_s[xa - 1] & kMaxBlocksPerSeq) : -1;
              const unsigned f = lane < nn ? dev::list_entry_faults(C, G, nblk, cidx, e, lane == 0 ? first_prev : up) : 0u;
              if (__any_sync(0xffffffffu, f != 0u)) {
                if (lane == 0) atomicOr(a.status, kStatusList);
                ok = false;
                break;
              }
              bool bad = false;
              const long long rw = lane < nn ? lay.row(seg, eb, &bad) : 0;
              if (bad) atomicOr(a.status, kStatusRange);
              int okl = 1;
              for (int jj = 0; jj < nn; ++jj) {
                const int ent = __shfl_sync(0xffffffffu, e, jj);
                const long long er = __shfl_sync(0xffffffffu, rw, jj);
                if (lane == 0 && okl) {
                  const int blk = ent & kMaxBlocksPerSeq;
                  if (npend > 0 && seg != pend.seg && !emit()) okl = 0;
                  if (okl) {
                    if (npend == 0) pend = FInfo{seg, 0, 0, 0, 0, 0};
                    prow[npend] = static_cast<int>(er);
                    const int mask = static_cast<int>(static_cast<unsigned>(ent) >> kEntryBlockBits);
                    const int nrows = min(s.b, T - blk * s.b);
                    if (npend == 0) { pend.mask0 = mask; pend.nrows0 = nrows; }
                    else { pend.mask1 = mask; pend.nrows1 = nrows; }
                    ++npend;
                    if (npend == BPT && !emit()) okl = 0;
                  }
                }
              }
              ok = __shfl_sync(0xffffffffu, okl, 0) != 0;
            }
            __syncwarp();  // ent_s is restaged next round
          }
          u = P[sl] + pb;
        }
        if (ok && u != u1) {  // the slices ran out before the range did
          if (lane == 0) atomicOr(a.status, kStatusList);
          ok = false;
        }
      }
      if (ok) ok = emit_pending();
      if (ok) {
        const int mode = run_seg >= 0 ? close_run(run_seg, first_run, true) : 0;
        int r = 1;
        if (lane == 0) {
          if (wait_or_abort(&B.kv_empty[stage], phase ^ 1u, a.status, abort_flag)) {
            info[stage] = FInfo{-1, 0, 0, 0, 0, mode};
            dev::mbar_arrive(&B.kv_full[stage]);
          } else {
            r = 0;
          }
        }
        ok = __shfl_sync(0xffffffffu, r, 0) != 0;
      }
    }
    if (!ok && lane == 0) {
      *abort_flag = 1;
      for (int k = 0; k < kStages; ++k) {  // let issued copies land
        if (issued_parity[k] < 0) continue;
        const long long t0 = clock64();
        while (!dev::mbar_try_wait(&B.kv_full[k], static_cast<uint32_t>(issued_parity[k])) &&
               clock64() - t0 < dev::kWaitCycles) {
        }
      }
    }
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16(TR, NQ, 0);
    constexpr uint32_t idesc_pv = idesc_bf16(D, NQ, 1);
    bool ok = true;
    auto issue_pv = [&](int i) -> bool {
      const int pb = i & 1;
      const int st_i = i % kStages;
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
    for (int j = 0; ok; ++j) {
      const int st_j = j % kStages;
      const int sb = j & 1;
      if (!wait_or_abort(&B.kv_full[st_j], (j / kStages) & 1, a.status, abort_flag)) { ok = false; break; }
      if (info[st_j].seg < 0) {  // END
        if (j > 0) ok = issue_pv(j - 1);
        break;
      }
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
    // every MMA issued so far has completed once `done` flips
    if (lane == 0) mma_commit(B.done);
    __syncwarp();
    {
      const long long t0 = clock64();
      while (!dev::mbar_try_wait(B.done, 0) && clock64() - t0 < dev::kWaitCycles) {
      }
    }
  } else {
    // ============================================================ softmax / correction / merge
    const int q4 = warp & 3;  // TMEM lane quarter this warp may access
    const uint32_t tlane = static_cast<uint32_t>(32 * q4) << 16;
    const int row = 32 * q4 + lane;  // key row of the tile this thread owns in S^T
    const int rblk = row / BR, rrow = row - rblk * BR;
    const int dcol = 32 * q4 + lane;  // output coordinate of this thread in O^T
    const float scale = a.scale, beta = a.beta;
    constexpr int PS = partial_stride(D);
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
    auto write_out = [&](int seg, const float* l_tot, const float* m, const float* o) {
      const int i = seg / s.Hkv, g = seg - i * s.Hkv;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const size_t orow = static_cast<size_t>(i) * s.Hq + g * G + h;
        dev::store_out_slot(a.out, s.elt, orow * D + dcol, l_tot[h] > 0.f ? o[h] / l_tot[h] : 0.f);
        if (dcol == h && a.lse) a.lse[orow] = dev::lse_of(m[h], l_tot[h]);
      }
    };
    // The run of segment seg ends: written out, or left as this CTA's piece
    // (and merged here if it completes the segment's set of pieces).
    auto flush = [&](int seg, int mode) -> bool {
      float* sums = red + 2 * 4 * 8;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float lw = dev::warp_sum(l_thr[h]);
        if (lane == 0) sums[q4 * 8 + h] = lw;
      }
      if (!rendezvous()) return false;
      float l_tot[G];
#pragma unroll
      for (int h = 0; h < G; ++h) l_tot[h] = sums[h] + sums[8 + h] + sums[16 + h] + sums[24 + h];
      if (!(mode & kModeShared)) {
        write_out(seg, l_tot, m_run, acc);
        return true;
      }
      const int slot = 2 * cta + ((mode & kModeSlot1) ? 1 : 0);
      float* part = a.partials + static_cast<size_t>(slot) * G * PS;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        part[h * PS + dcol] = acc[h];
        if (dcol == h) {
          part[h * PS + D] = m_run[h];
          part[h * PS + D + 1] = l_tot[h];
        }
      }
      __threadfence();
      if (!rendezvous()) return false;  // also: every thread has read sums
      if (warp == 2 && lane == 0) {
        // one announcement per piece (see piece_announcement)
        const unsigned long long add = piece_announcement(mode, cta);
        unsigned long long* ctr = a.seg_ctr + seg;
        const PieceSet ps = piece_set(atom_add_acq_rel64(ctr, add) + add);
        const int cf = ps.c_first, cl = ps.c_last;
        const dev::UnitSplit us(static_cast<unsigned>(*units_total), static_cast<unsigned>(N));
        bool stale = false;
        const bool complete = piece_set_complete(ps, us, N, &stale);
        if (stale) atomicOr(a.status, kStatusList);
        if (complete) {
          *ctr = 0ull;  // every piece has arrived: nothing else touches it in this step
          // merged at the end, when the K/V ring is free to receive the pieces
          const int n = pm[0];
          pm[1 + 4 * n] = seg;
          pm[2 + 4 * n] = cf;
          pm[3 + 4 * n] = cl;
          pm[4 + 4 * n] = ps.slot_first;
          pm[0] = n + 1;
        }
      }
      return true;
    };
    // Merge the pieces of segment seg held by CTAs cf..cl (CTA order): the
    // pieces are copied into the idle K/V ring (16-byte asynchronous copies
    // from all softmax threads, batches of as many as fit), then each thread
    // combines four output coordinates of one head over them.
    auto merge = [&](int seg, int cf, int cl, int slot_cf) -> bool {
      const dev::UnitSplit us(static_cast<unsigned>(*units_total), static_cast<unsigned>(N));
      constexpr uint32_t kPiece = G * PS * sizeof(float);
      constexpr int kMaxPieces = static_cast<int>(static_cast<size_t>(kStages) * TL::STAGE / kPiece);
      constexpr int kAssign = (G * 32 + 127) / 128;  // (head, quad) pairs per thread
      uint8_t* ring = base + L.stages;
      float mx[kAssign], l[kAssign], o4[kAssign][4];
#pragma unroll
      for (int w = 0; w < kAssign; ++w) {
        mx[w] = -INFINITY;
        l[w] = 0.f;
        o4[w][0] = o4[w][1] = o4[w][2] = o4[w][3] = 0.f;
      }
      int c0 = cf;
      while (c0 <= cl) {
        // this batch's pieces (the CTAs from c0 on with a non-empty range, as
        // many as the ring holds): their slots, listed by warp 2
        if (warp == 2) {
          int np = 0, c = c0;
          while (c <= cl && np < kMaxPieces) {
            const int cc = c + lane;
            const bool has = cc <= cl && us.owns_any(static_cast<unsigned>(cc));
            const unsigned bal = __ballot_sync(0xffffffffu, has);
            const int before = __popc(bal & ((1u << lane) - 1u));
            if (has && np + before < kMaxPieces) ent_s[np + before] = 2 * cc + (cc == cf ? slot_cf : 0);
            if (np + __popc(bal) <= kMaxPieces) {
              np += __popc(bal);
              c += 32;
            } else {  // the next batch starts at the first piece that does not fit
              const unsigned first_out = __ballot_sync(0xffffffffu, has && np + before == kMaxPieces);
              c += __ffs(first_out) - 1;
              np = kMaxPieces;
            }
          }
          if (lane == 0) {
            mbatch[0] = np;
            mbatch[1] = min(c, cl + 1);
          }
        }
        if (!rendezvous()) return false;
        const int np = mbatch[0];
        const int next = mbatch[1];
        // all pieces in flight at once: 16-byte asynchronous copies through L2
        fence_proxy_async();  // the ring's earlier tensor copies and reads come first
        constexpr int kPc = static_cast<int>(kPiece / 16);
        for (int x = t - 64; x < np * kPc; x += 128) {
          const int p = x / kPc, o = x - p * kPc;
          dev::cp_async16(ring + static_cast<size_t>(p) * kPiece + o * 16,
                          reinterpret_cast<const uint8_t*>(a.partials + static_cast<size_t>(ent_s[p]) * G * PS) + o * 16);
        }
        dev::cp_async_commit();
        dev::cp_async_wait<0>();
        if (!rendezvous()) return false;  // every thread's copies have landed
#pragma unroll
        for (int w = 0; w < kAssign; ++w) {
          const int hq = (t - 64) + 128 * w;
          if (hq >= G * 32) continue;
          const int h = hq >> 5, quad = hq & 31;
          for (int p = 0; p < np; ++p) {
            const float* pp = reinterpret_cast<const float*>(ring + static_cast<size_t>(p) * kPiece) + h * PS;
            const float mc = pp[D], lc = pp[D + 1];
            const float4 oc = reinterpret_cast<const float4*>(pp)[quad];
            const float mn = fmaxf(mx[w], mc);
            const float fo = mx[w] == -INFINITY ? 0.f : dev::fast_exp2(mx[w] - mn);
            const float fc = mc == -INFINITY ? 0.f : dev::fast_exp2(mc - mn);
            l[w] = l[w] * fo + lc * fc;
            o4[w][0] = o4[w][0] * fo + oc.x * fc;
            o4[w][1] = o4[w][1] * fo + oc.y * fc;
            o4[w][2] = o4[w][2] * fo + oc.z * fc;
            o4[w][3] = o4[w][3] * fo + oc.w * fc;
            mx[w] = mn;
          }
        }
        if (!rendezvous()) return false;  // the ring may be refilled
        c0 = next;
      }
      const int i = seg / s.Hkv, g = seg - i * s.Hkv;
#pragma unroll
      for (int w = 0; w < kAssign; ++w) {
        const int hq = (t - 64) + 128 * w;
        if (hq >= G * 32) continue;
        const int h = hq >> 5, quad = hq & 31;
        const size_t orow = static_cast<size_t>(i) * s.Hq + g * G + h;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          dev::store_out_slot(a.out, s.elt, orow * D + 4 * quad + k, l[w] > 0.f ? o4[w][k] / l[w] : 0.f);
        if (quad == 0 && a.lse) a.lse[orow] = dev::lse_of(mx[w], l[w]);
      }
      return true;
    };

    int pending = -1;  // tile whose O^T is not folded in yet
    for (int j = 0; ok; ++j) {
      const int st_j = j % kStages;
      if (!wait_or_abort(&B.kv_full[st_j], (j / kStages) & 1, a.status, abort_flag)) { ok = false; break; }
      const FInfo in = info[st_j];
      if (j == 0 && in.seg >= 0 && warp == 2 && lane == 0) dev::trace_first(a.trace, ETA_TRACE_TILE_FIRST);
      if (in.seg != cur_seg || in.seg < 0) {  // a new segment, or END (also as the first entry of an empty range)
        if (pending >= 0) {
          if (!correction(pending) || !flush(cur_seg, in.prev_mode)) { ok = false; break; }
          pending = -1;
        }
        if (in.seg < 0) {  // END: the ring is free (every tile consumed, every MMA done)
          if (!rendezvous()) { ok = false; break; }  // the merges recorded by warp 2 are visible
          const int n = pm[0];
          for (int x = 0; x < n && ok; ++x) ok = merge(pm[1 + 4 * x], pm[2 + 4 * x], pm[3 + 4 * x], pm[4 + 4 * x]);
          break;
        }
        cur_seg = in.seg;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_run[h] = -INFINITY;
          l_thr[h] = 0.f;
          acc[h] = 0.f;
          tau_h[h] = __ldcg(a.tau + static_cast<size_t>(in.seg) * G + h);
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
          const int kp = row >> 6, tcl = row & 63;
          const int off = kp * 2048 + h * 128 + (((tcl >> 3) ^ (h & 7)) << 4) + (tcl & 7) * 2;
          *reinterpret_cast<uint16_t*>(pbuf + off) = pbits;
        }
        l_thr[h] = fmaf(l_thr[h], alpha[h], __uint_as_float(static_cast<uint32_t>(pbits) << 16));
        m_run[h] = m_new;
      }
      if (in.nrows0 < BR || (BPT == 2 && in.nrows1 < BR)) {
        // rows of a tile that hold no key (past a sequence end, or an absent
        // second block) are zeroed in V so that stale or non-finite bytes
        // there cannot reach the accumulator (0 * inf)
        uint8_t* vbuf = base + L.stages + st_j * TL::STAGE + TL::V0;
        for (int bi = 0; bi < BPT; ++bi) {
          const int nr = bi == 0 ? in.nrows0 : in.nrows1;
          const int nz = (BR - nr) * 8;  // 16-byte chunks per panel
          for (int c = t - 64; c < 2 * nz; c += 128) {
            const int pnl = c / nz, r = c - pnl * nz;
            *reinterpret_cast<uint4*>(vbuf + pnl * TL::PANEL + (bi * BR + nr) * 128 + r * 16) =
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
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  if (t == 0) dev::trace_last(a.trace, ETA_TRACE_FUSED_LAST);
  // The last CTA to finish clears the slice totals for the next step (every
  // CTA read them all before it got here).
  if (warp == 0) {
    unsigned last = 0;
    if (lane == 0) {
      __threadfence();
      last = atom_add_acq_rel(a.done_ctas, 1u) + 1u == static_cast<unsigned>(N) ? 1u : 0u;
    }
    if (__shfl_sync(0xffffffffu, last, 0)) {
      for (int x = lane; x < N; x += 32) a.flags[x] = 0u;
      if (lane == 0) {
        *a.arrived = 0u;
        *a.done_ctas = 0u;
      }
    }
  }
}

// ------------------------------------------------------------ host side

template <int BR, int G>
cudaError_t launch_typed(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const FusedArgs& a,
                         cudaStream_t st, size_t smem) {
  auto kern = fused_tc_kernel<BR, G>;
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
                          [&] { return cudaLaunchKernelEx(&cfg, kern, tk, tv, tq, a); });
}

template <int BR>
cudaError_t launch_g(const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tq, const FusedArgs& a,
                     cudaStream_t st, size_t smem) {
  switch (a.s.G) {
    case 2: return launch_typed<BR, 2>(tk, tv, tq, a, st, smem);
    case 4: return launch_typed<BR, 4>(tk, tv, tq, a, st, smem);
    case 8: return launch_typed<BR, 8>(tk, tv, tq, a, st, smem);
  }
  return cudaErrorInvalidValue;
}

constexpr size_t kSmemBudget = 227 * 1024;

}  // namespace

size_t fused_tc_smem(const Shape& s) {
  if (s.chunk < 1 || s.chunk > 32 || s.B > kFusedMaxSeqs || s.attend_ctas < 1 || s.attend_ctas > kFusedMaxCtas)
    return 0;
  const size_t n = fused_layout(s.attend_ctas).total;
  return n <= kSmemBudget ? n : 0;
}

cudaError_t launch_fused_tc(const FusedArgs& a, cudaStream_t st) {
  const size_t smem = fused_tc_smem(a.s);
  if (smem == 0) return cudaErrorInvalidConfiguration;
  CUtensorMap tk, tv, tq;
  const uint64_t rows = a.s.num_pages ? static_cast<uint64_t>(a.s.num_pages) * a.s.Hkv * a.s.b
                                      : static_cast<uint64_t>(a.s.nseg) * a.s.max_ctx;
  if (!make_map(&tk, a.k, rows, a.s.b) || !make_map(&tv, a.v, rows, a.s.b) ||
      !make_map(&tq, a.q, static_cast<uint64_t>(a.s.B) * a.s.Hq, NQ))
    return cudaErrorInvalidValue;
  return a.s.b == 64 ? launch_g<64>(tk, tv, tq, a, st, smem) : launch_g<128>(tk, tv, tq, a, st, smem);
}

}  // namespace eta
