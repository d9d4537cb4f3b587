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
// The pages screen and attend in one pass over positional chunks (section 3.2);
// this kernel does the same with chunks handed out dynamically.
//
// Work is split into positional chunks of `chunk` consecutive blocks of one
// (sequence, KV head), numbered in (sequence, KV head, block) order.  Each CTA
// (one per SM) runs:
//   warp 6    screen: takes chunk numbers from a global ticket counter (two
//             ahead), stages a chunk's metadata with bulk copies, scores its
//             blocks for the G heads, builds the chunk's admitted list (also
//             written out for the selection export) and queues its tiles (one
//             or two admitted blocks of the chunk, 128 key rows);
//   warp 0    producer: tensor copies (TMA, 128-byte swizzle) of each tile's
//             K and V blocks and the group's query rows into a 3-stage ring;
//   warp 1    MMA issuer: S^T = K Q^T and O^T = V^T P^T into tensor memory;
//   warps 2-5 softmax: gate, online softmax, P, folding O^T; at the end of a
//             chunk its partial (acc, m, l per head) goes to the chunk's own
//             slot and an event to warp 7; fold jobs from warp 7 are run at
//             chunk boundaries and, after the last tile, until warp 7 is done;
//   warp 7    completion: for every finished chunk (or fold) one release /
//             acquire atomic on the counter of its parent node in the
//             segment's fold tree (fan-in kFoldFan); the thread that completes
//             a node resets its counter and hands the node's fold to the
//             softmax warps.
// A node's fold combines its children's partials in index order; the root of
// a segment's tree writes the output rows and lse.  Whichever CTA handles a
// chunk, every partial and every fold is computed in the same order, so the
// result is bit-reproducible.  No CTA ever waits for another CTA.
//
// Counters (tickets, finished CTAs, fold-tree nodes) live in the workspace's
// control region and are back at zero when a step completes: the last CTA to
// finish resets the first two, the completer of a node resets its counter.

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
constexpr int NQ = 16;            // N of both MMAs (the G query rows, rest zero)
constexpr int TR = 128;           // key rows per tile
constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kScreenWarp = 6;
constexpr int kDoneWarp = 7;
constexpr int kTmemCols = 64;     // S buffers at columns 0, 16; O buffers at 32, 48
constexpr int kStages = 3;
constexpr int kQueue = 8;         // tiles queued from the screen warp to the producer
constexpr int kEvents = 32;       // events from the softmax warps to the completion warp
constexpr int kJobs = 8;          // fold jobs from the completion warp to the softmax warps
constexpr int kMaxChunk = 32;     // blocks per chunk (one lane each in the screen warp)
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kFirst = 1, kLast = 2, kEnd = 4;

struct Tile {
  static constexpr int PANEL = TR * 128;  // one 64-column (128-byte) panel of a 128-row tile
  static constexpr int K0 = 0, K1 = PANEL, V0 = 2 * PANEL, V1 = 3 * PANEL, Q0 = 4 * PANEL, Q1 = 4 * PANEL + 2048;
  static constexpr int STAGE = 4 * PANEL + 4096;
  static constexpr int P_BYTES = NQ * TR * 2;
};

// A tile as the screen warp hands it on: up to two admitted blocks of one
// chunk, their head masks, rows present (0: none) and first K/V rows, the
// chunk's identity and the thresholds of its heads.
struct FTile {
  int seq, kvh, cidx, pad0;
  int mask0, mask1, nrows0, nrows1;
  long long row0, row1;
  int flags, pad1;
  float tau[8];
};

// Softmax -> completion warp: a partial of fold level `level` (0: a chunk)
// was written for node `node` of segment (seq, kvh); kind 1 = the last
// tile's chunk is done and no chunk follows.
struct Event {
  int kind, seq, kvh, level, node, pad[3];
};

// Completion warp -> softmax warps: fold the children of node `node` at
// level `level` (>= 1) of segment (seq, kvh); kind 1 = nothing more to do.
struct Job {
  int kind, seq, kvh, level, node, pad[3];
};

struct Layout {
  size_t stages, pbuf, meta, mnorm, bars, info, queue, events, jobs, red, tabs, seen, pend, misc, total;
};

constexpr int kPendNodes = 128;  // completed fold-tree nodes the completion warp holds until the tiles are done

constexpr int kMaxSegs = 2048;  // segments (sequence, KV head) the screen warp's used-up mask covers

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kBars = 2 * kStages + 12 + 2 * kQueue + 2 + 2 * kEvents + 2 * kJobs + 1;

__host__ __device__ inline Layout fused_layout(int chunk) {
  Layout L;
  size_t off = 0;
  L.stages = off;
  off += static_cast<size_t>(kStages) * Tile::STAGE;
  L.pbuf = off;
  off += 2 * static_cast<size_t>(Tile::P_BYTES);
  L.meta = off;  // [2 buffers][mu, sigma][chunk][D] fp16
  off += 2 * 2 * static_cast<size_t>(chunk) * D * 2;
  L.mnorm = off;  // [2][chunk] fp32
  off += 2 * static_cast<size_t>(chunk) * sizeof(float);
  L.bars = off = align_up(off, 16);
  off += kBars * sizeof(uint64_t);
  L.info = off = align_up(off, 16);
  off += kStages * sizeof(FTile);
  L.queue = off = align_up(off, 16);
  off += kQueue * sizeof(FTile);
  L.events = off = align_up(off, 16);
  off += kEvents * sizeof(Event);
  L.jobs = off = align_up(off, 16);
  off += kJobs * sizeof(Job);
  L.red = off = align_up(off, 16);
  off += (2 * 4 * 8 + 4 * 8) * sizeof(float);
  L.tabs = off = align_up(off, 16);  // seqT[S]
  off += kFusedMaxSeqs * sizeof(int);
  L.seen = off = align_up(off, 16);  // segments this CTA found used up, one bit each
  off += kMaxSegs / 32 * sizeof(unsigned);
  L.pend = off = align_up(off, 16);
  off += kPendNodes * sizeof(unsigned);
  L.misc = off = align_up(off, 16);
  off += 64;
  L.total = align_up(off, 128) + 1024;  // + slack to align the dynamic base to 1024
  return L;
}

struct Bars {
  uint64_t* kv_full;   // [kStages] producer -> MMA, softmax (tx bytes)
  uint64_t* kv_empty;  // [kStages] MMA commit -> producer
  uint64_t* s_full;    // [2] MMA commit -> softmax
  uint64_t* s_free;    // [2] softmax (4 warps) -> MMA
  uint64_t* p_full;    // [2] softmax (4 warps) -> MMA
  uint64_t* o_full;    // [2] MMA commit -> softmax
  uint64_t* o_free;    // [2] softmax (4 warps) -> MMA
  uint64_t* rv;        // [1] softmax-warp rendezvous (4 warps)
  uint64_t* done;      // [1] final MMA commit
  uint64_t* q_full;    // [kQueue] screen -> producer
  uint64_t* q_empty;   // [kQueue] producer -> screen
  uint64_t* meta;      // [2] metadata bulk copies landed
  uint64_t* ev_full;   // [kEvents] softmax -> completion
  uint64_t* ev_empty;  // [kEvents] completion -> softmax
  uint64_t* job_full;  // [kJobs] completion -> softmax
  uint64_t* job_empty; // [kJobs] softmax (4 warps) -> completion
  uint64_t* fold;      // [1] a fold's children staged in shared memory (bulk copy)
};

// Atomic add with release and acquire semantics at GPU scope: the partials
// written before it (by this CTA, ordered by a CTA barrier) are visible to
// whoever reads the counter afterwards, and this thread sees the partials of
// everyone who incremented it before.
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------- sequence tables

struct Tables {
  const int* seqT;  // clamped lengths
  int b, chunk;
  __device__ __forceinline__ int nb(int i) const { return (seqT[i] + b - 1) / b; }
  __device__ __forceinline__ int nch(int i) const { return (nb(i) + chunk - 1) / chunk; }
  // nodes of sequence i's trees at fold level l
  __device__ __forceinline__ int nodes(int i, int l) const {
    int n = nch(i);
    for (int k = 0; k < l; ++k) n = (n + kFoldFan - 1) / kFoldFan;
    return n;
  }
};

// ---------------------------------------------------------------- folds

// Folds n <= kFoldFan partials (slots first .. first + n - 1 of `src`, each
// [G][FPS]: acc[D], m, l shares[4]) in slot order for the heads h0,
// h0 + hstep, ... of the calling warp; lanes own 4 output coordinates.  The
// result goes to slot `dst` of a partial array (l in the first share), or
// (dst == nullptr) to the output rows (normalised) and lse.
template <int G>
__device__ void fold_partials(const float* src, size_t first, int n, float* dst, const FusedArgs& a, int seq, int kvh,
                              int h0, int hstep, int lane) {
  constexpr int FPS = fused_partial_stride(D);
  constexpr int kB = 8;  // loads in flight per round (registers; a rarely used path)
  for (int h = h0; h < G; h += hstep) {
    float mx = -INFINITY, ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = 0; k0 < n; k0 += kB) {
      float4 ml[kB];
      float l3[kB];
      float4 x[kB];
#pragma unroll
      for (int u = 0; u < kB; ++u) {  // all loads of the round in flight
        const int k = min(k0 + u, n - 1);
        const float* p = src + ((first + k) * G + h) * FPS;
        ml[u] = __ldcg(reinterpret_cast<const float4*>(p + D));
        l3[u] = __ldcg(p + D + 4);
        x[u] = __ldcg(reinterpret_cast<const float4*>(p) + lane);
      }
#pragma unroll
      for (int u = 0; u < kB; ++u) {
        const float l = ((ml[u].y + ml[u].z) + ml[u].w) + l3[u];
        if (k0 + u >= n || !(l > 0.f)) continue;  // empty partial (l = 0, m = -inf)
        const float m = ml[u].x;
        if (m > mx) {
          const float f = mx == -INFINITY ? 0.f : dev::fast_exp2(mx - m);
          ls = fmaf(ls, f, l);
          acc.x = fmaf(acc.x, f, x[u].x);
          acc.y = fmaf(acc.y, f, x[u].y);
          acc.z = fmaf(acc.z, f, x[u].z);
          acc.w = fmaf(acc.w, f, x[u].w);
          mx = m;
        } else {
          const float f = dev::fast_exp2(m - mx);
          ls = fmaf(l, f, ls);
          acc.x = fmaf(x[u].x, f, acc.x);
          acc.y = fmaf(x[u].y, f, acc.y);
          acc.z = fmaf(x[u].z, f, acc.z);
          acc.w = fmaf(x[u].w, f, acc.w);
        }
      }
    }
    if (dst) {
      float* p = dst + h * FPS;
      reinterpret_cast<float4*>(p)[lane] = acc;
      if (lane == 0) {
        *reinterpret_cast<float4*>(p + D) = make_float4(mx, ls, 0.f, 0.f);
        p[D + 4] = 0.f;
      }
    } else {
      const size_t orow = static_cast<size_t>(seq) * a.s.Hq + static_cast<size_t>(kvh) * G + h;
      const float inv = ls > 0.f ? 1.f / ls : 0.f;
      const float o[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
#pragma unroll
      for (int e = 0; e < 4; ++e) dev::store_out_slot(a.out, a.s.elt, orow * D + lane * 4 + e, o[e]);
      if (lane == 0 && a.lse) a.lse[orow] = dev::lse_of(mx, ls);
    }
  }
}

// The same fold with the n children staged in shared memory at `sm`
// ([n][G][FPS], one bulk copy), for the heads of softmax warp w4.
template <int G>
__device__ void fold_staged(const float* sm, int n, float* dst, const FusedArgs& a, int seq, int kvh, int w4, int lane) {
  constexpr int FPS = fused_partial_stride(D);
  for (int h = w4; h < G; h += 4) {
    float mx = -INFINITY, ls = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k = 0; k < n; ++k) {
      const float* p = sm + (static_cast<size_t>(k) * G + h) * FPS;
      const float4 ml = *reinterpret_cast<const float4*>(p + D);
      const float l = ((ml.y + ml.z) + ml.w) + p[D + 4];
      if (!(l > 0.f)) continue;  // empty partial (l = 0, m = -inf)
      const float4 x = reinterpret_cast<const float4*>(p)[lane];
      const float m = ml.x;
      if (m > mx) {
        const float f = mx == -INFINITY ? 0.f : dev::fast_exp2(mx - m);
        ls = fmaf(ls, f, l);
        acc.x = fmaf(acc.x, f, x.x);
        acc.y = fmaf(acc.y, f, x.y);
        acc.z = fmaf(acc.z, f, x.z);
        acc.w = fmaf(acc.w, f, x.w);
        mx = m;
      } else {
        const float f = dev::fast_exp2(m - mx);
        ls = fmaf(l, f, ls);
        acc.x = fmaf(x.x, f, acc.x);
        acc.y = fmaf(x.y, f, acc.y);
        acc.z = fmaf(x.z, f, acc.z);
        acc.w = fmaf(x.w, f, acc.w);
      }
    }
    if (dst) {
      float* p = dst + h * FPS;
      reinterpret_cast<float4*>(p)[lane] = acc;
      if (lane == 0) {
        *reinterpret_cast<float4*>(p + D) = make_float4(mx, ls, 0.f, 0.f);
        p[D + 4] = 0.f;
      }
    } else {
      const size_t orow = static_cast<size_t>(seq) * a.s.Hq + static_cast<size_t>(kvh) * G + h;
      const float inv = ls > 0.f ? 1.f / ls : 0.f;
      const float o[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
#pragma unroll
      for (int e = 0; e < 4; ++e) dev::store_out_slot(a.out, a.s.elt, orow * D + lane * 4 + e, o[e]);
      if (lane == 0 && a.lse) a.lse[orow] = dev::lse_of(mx, ls);
    }
  }
}

// ---------------------------------------------------------------- kernel

template <int BR, int G>
__global__ void __launch_bounds__(kThreads, 1)
    fused_tc_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ CUtensorMap tq, FusedArgs a) {
  using TL = Tile;
  constexpr int BPT = TR / BR;  // blocks per tile
  constexpr int FPS = fused_partial_stride(D);
  extern __shared__ uint8_t smem_raw[];
  const Shape& s = a.s;
  const int C = s.chunk;
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw);
  const Layout L = fused_layout(C);

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
  B.q_full = B.done + 1;
  B.q_empty = B.q_full + kQueue;
  B.meta = B.q_empty + kQueue;
  B.ev_full = B.meta + 2;
  B.ev_empty = B.ev_full + kEvents;
  B.job_full = B.ev_empty + kEvents;
  B.job_empty = B.job_full + kJobs;
  B.fold = B.job_empty + kJobs;
  FTile* info = reinterpret_cast<FTile*>(base + L.info);
  FTile* queue = reinterpret_cast<FTile*>(base + L.queue);
  Event* events = reinterpret_cast<Event*>(base + L.events);
  Job* jobs = reinterpret_cast<Job*>(base + L.jobs);
  float* red = reinterpret_cast<float*>(base + L.red);
  int* seqT = reinterpret_cast<int*>(base + L.tabs);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + L.misc + 4);
  int* issued_parity = reinterpret_cast<int*>(base + L.misc + 16);

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
      dev::mbar_init(&B.meta[k], 1);
    }
    for (int k = 0; k < kQueue; ++k) {
      dev::mbar_init(&B.q_full[k], 1);
      dev::mbar_init(&B.q_empty[k], 1);
    }
    for (int k = 0; k < kEvents; ++k) {
      dev::mbar_init(&B.ev_full[k], 4);  // one arrival per softmax warp
      dev::mbar_init(&B.ev_empty[k], 1);
    }
    for (int k = 0; k < kJobs; ++k) {
      dev::mbar_init(&B.job_full[k], 1);
      dev::mbar_init(&B.job_empty[k], 4);
    }
    dev::mbar_init(B.rv, 4);
    dev::mbar_init(B.done, 1);
    dev::mbar_init(B.fold, 1);
    *abort_flag = 0;
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
  // Nothing written by the previous kernel of the stream (an append, the
  // previous step) is read before this point; the next kernel may start its
  // own prologue now (nothing here waits for another CTA).
  dev::pdl_trigger();
  dev::pdl_wait();

  for (int x = t; x < s.B; x += kThreads) {
    int tt = a.seq_lens[x];
    if (tt < 0 || tt > s.max_ctx) {
      if (blockIdx.x == 0) atomicOr(a.status, kStatusRange);
      tt = tt < 0 ? 0 : s.max_ctx;
    }
    seqT[x] = tt;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const Tables tb{seqT, s.b, C};
  const uint32_t tmem = *tmem_slot;

  if (warp == kScreenWarp) {
    // ============================================================ screen
    constexpr int CPL = D / 32;  // coordinates per lane
    constexpr int NV = 2 * G;    // values per block: <q_h, mu>, sum q_h^2 sigma^2
    constexpr int NB = 32 / NV;  // blocks reduced together
    // empty sequences have no chunk: their outputs are 0, lse -inf
    for (int i = blockIdx.x; i < s.B; i += gridDim.x) {
      if (seqT[i] != 0) continue;
      for (int x = lane; x < s.Hq * D; x += 32) dev::store_out_slot(a.out, s.elt, static_cast<size_t>(i) * s.Hq * D + x, 0.f);
      for (int x = lane; x < s.Hq; x += 32)
        if (a.lse) a.lse[static_cast<size_t>(i) * s.Hq + x] = -INFINITY;
    }
    const KvLayout lay{a.block_table, s.Hkv, s.b, s.max_ctx, s.nbmax, s.num_pages};
    float qr[G][CPL], q2[G][CPL], tau_h[G], qn_h[G];
    int cur_seg = -1;
    int qslot = 0;
    uint32_t qphase = 0;
    bool ok = true;
    // Chunks are handed out per (sequence, KV head) segment.  Each CTA has a
    // home segment (CTAs spread evenly over the segments); the first two
    // chunks of every home CTA are fixed by its rank in the segment's group
    // (chunks rank and rank + group size), later ones come from the
    // segment's counter (offset by the fixed ones), and when a segment is
    // used up the CTA moves on to the next segments not yet marked used up.
    // A CTA therefore stays on one segment for most of its chunks, and no
    // counter is hit by every CTA at once when the kernel starts.
    struct Job2 { int seq, kvh, cidx, nloc, nscreen; };
    unsigned* segtk = a.counters;             // [nseg] chunks handed out per segment, beyond the fixed ones
    unsigned* used_up = a.counters + s.nseg;  // [ceil(nseg / 32)] bit per segment
    const unsigned grid = gridDim.x;
    auto group_lo = [&](int sg) -> int {  // first CTA whose home is segment sg
      return static_cast<int>((static_cast<long long>(sg) * grid + s.nseg - 1) / s.nseg);
    };
    // segments this warp itself found used up: its own marks may not be
    // visible to its next reads of the global bits yet, and must never be
    // visited again
    unsigned* seen = reinterpret_cast<unsigned*>(base + L.seen);
    for (int x = lane; x < kMaxSegs / 32; x += 32) seen[x] = 0u;
    __syncwarp();
    const int home = static_cast<int>(static_cast<long long>(blockIdx.x) * s.nseg / grid);
    const int rank = static_cast<int>(blockIdx.x) - group_lo(home);
    const int hsize = group_lo(home + 1) - group_lo(home);
    int gseg = home;
    auto fixed = [&](int sg) -> int { return 2 * (group_lo(sg + 1) - group_lo(sg)); };
    auto grab = [&]() -> unsigned {  // the atomic's result is used later, so its latency overlaps work
      unsigned tk = 0;
      if (lane == 0) tk = atomicAdd(&segtk[gseg], 1u);
      return tk;
    };
    // the first segment after `from` (circularly, `from` itself excluded) not
    // marked used up, or -1
    auto next_open = [&](int from) -> int {
      for (int k0 = 1; k0 < s.nseg; k0 += 32) {
        const int k = k0 + lane;
        const int sg = (from + k) % s.nseg;
        const bool open = k < s.nseg && (((__ldcg(used_up + (sg >> 5)) | seen[sg >> 5]) >> (sg & 31)) & 1u) == 0u;
        const unsigned bal = __ballot_sync(0xffffffffu, open);
        if (bal) return (from + k0 + __ffs(bal) - 1) % s.nseg;
      }
      return -1;
    };
    // a counter value taken from segment gs, as a chunk index
    auto dyn = [&](unsigned raw, int gs) -> int {
      return static_cast<int>(__shfl_sync(0xffffffffu, raw, 0)) + fixed(gs);
    };
    // Counter values taken but not yet looked at wait in a small queue (two
    // atomics overlap the scoring); every value taken is looked at before the
    // warp may stop, so no chunk handed out is ever dropped.
    constexpr int kPend = 4;
    unsigned pq_raw[kPend];
    int pq_seg[kPend], pq_fixed[kPend];
    int pq_head = 0, pq_n = 0;
    auto pq_push = [&](unsigned raw, int sg, int is_fixed) {
      const int k = (pq_head + pq_n) % kPend;
#pragma unroll
      for (int u = 0; u < kPend; ++u)
        if (u == k) { pq_raw[u] = raw; pq_seg[u] = sg; pq_fixed[u] = is_fixed; }
      ++pq_n;
    };
    // the next chunk to process: the oldest queued value, else a value taken
    // now; a value past its segment's end marks the segment used up and moves
    // the warp on to the next open segment
    auto next_job = [&](Job2& j) -> bool {
      for (int iter = 0; iter < 8 + 2 * s.nseg; ++iter) {
        if (pq_n == 0) {
          if (gseg < 0) return false;
          pq_push(grab(), gseg, 0);
        }
        unsigned raw = 0;
        int sg = 0, fx = 0;
#pragma unroll
        for (int u = 0; u < kPend; ++u)
          if (u == pq_head) { raw = pq_raw[u]; sg = pq_seg[u]; fx = pq_fixed[u]; }
        pq_head = (pq_head + 1) % kPend;
        --pq_n;
        const int cidx = fx ? static_cast<int>(raw) : dyn(raw, sg);
        const int i = sg / s.Hkv;
        if (cidx < tb.nch(i)) {
          j.seq = i;
          j.kvh = sg - i * s.Hkv;
          j.cidx = cidx;
          const int nb = tb.nb(i);
          const int blk0 = cidx * C;
          j.nloc = min(C, nb - blk0);
          const int first_forced = a.screen_enabled ? max(0, nb - 1 - a.lwb) : 0;
          j.nscreen = max(0, min(j.nloc, first_forced - blk0));
          return true;
        }
        if (lane == 0) {
          atomicOr(&used_up[sg >> 5], 1u << (sg & 31));
          seen[sg >> 5] |= 1u << (sg & 31);
        }
        __syncwarp();
        if (sg == gseg) gseg = next_open(sg);
      }
      if (lane == 0) atomicOr(a.status, kStatusTimeout);  // cannot happen: counted as a failed wait
      return false;
    };
    uint32_t meta_phase[2] = {0u, 0u};
    int meta_pending[2] = {0, 0};
    // A chunk's metadata: mu and sigma rows by bulk copy (completion on the
    // buffer's mbarrier), the block norms by 4-byte asynchronous copies (one
    // commit group per staged chunk, so the scoring waits only for its own).
    auto stage_meta = [&](const Job2& j, int buf) {
      if (j.nscreen > 0) {
        const size_t seg = static_cast<size_t>(j.seq) * s.Hkv + j.kvh;
        const size_t row = seg * s.nbmax + static_cast<size_t>(j.cidx) * C;
        float* mn = reinterpret_cast<float*>(base + L.mnorm) + buf * C;
        if (lane < j.nscreen) dev::cp_async4(&mn[lane], &a.max_norm[row + lane]);
        if (lane == 0) {
          fence_proxy_async();  // this buffer's previous contents were read through the generic proxy
          uint8_t* mb = base + L.meta + static_cast<size_t>(buf) * 2 * C * D * 2;
          const uint32_t bytes = static_cast<uint32_t>(j.nscreen) * D * 2;
          dev::mbar_arrive_expect_tx(&B.meta[buf], 2 * bytes);
          dev::bulk_g2s(mb, static_cast<const uint8_t*>(a.mu) + row * D * 2, bytes, &B.meta[buf]);
          dev::bulk_g2s(mb + C * D * 2, static_cast<const uint8_t*>(a.sigma) + row * D * 2, bytes, &B.meta[buf]);
        }
        meta_pending[buf] = 1;
      }
      dev::cp_async_commit();
    };
    auto push = [&](const FTile& ft) -> bool {
      if (!dev::warp_wait_or_abort(&B.q_empty[qslot], qphase ^ 1u, a.status, abort_flag)) return false;
      if (lane == 0) {
        queue[qslot] = ft;
        dev::mbar_arrive(&B.q_full[qslot]);
      }
      __syncwarp();
      if (++qslot == kQueue) { qslot = 0; qphase ^= 1u; }
      return true;
    };
    // Two chunks are staged ahead of the one being scored: cur (metadata in
    // buffer buf), nxt (buffer buf ^ 1); the ticket after nxt is taken while
    // cur is scored.
    // cur and nxt are resolved and their metadata staged.  Each iteration
    // takes one more counter value; its atomic's result is first read one
    // iteration later (queued then), so the warp never waits for it.
    Job2 cur, nxt;
    pq_push(static_cast<unsigned>(rank), home, 1);  // the two fixed chunks of the home segment
    pq_push(static_cast<unsigned>(rank + hsize), home, 1);
    bool have_cur = next_job(cur);
    bool have_nxt = false;
    int buf = 0;
    if (have_cur) {
      stage_meta(cur, 0);
      have_nxt = next_job(nxt);
      if (have_nxt) stage_meta(nxt, 1);
    }
    while (have_cur && ok) {
      int r_seg = -1;
      const unsigned r_new = (have_nxt && gseg >= 0) ? grab() : 0u;
      if (have_nxt && gseg >= 0) r_seg = gseg;
      const int seg = cur.seq * s.Hkv + cur.kvh;
      const int T = seqT[cur.seq];
      const int blk0 = cur.cidx * C;
      if (seg != cur_seg) {
        // the heads' queries, thresholds and norms (all loads issued first)
        cur_seg = seg;
        uint2 qu[G];
        float wv[G][CPL], bc[G];
        const bool learned = a.tau_mode == ETA_TAU_LEARNED;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const int hq = cur.kvh * G + h;
          const size_t qo = (static_cast<size_t>(cur.seq) * s.Hq + hq) * D;
          qu[h] = *reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(a.q) + qo + lane * CPL);
#pragma unroll
          for (int k = 0; k < CPL; ++k) wv[h][k] = learned ? a.w_tau[static_cast<size_t>(hq) * D + lane * CPL + k] : 0.f;
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
          for (int k = 0; k < CPL; ++k) {
            q2[h][k] = qr[h][k] * qr[h][k];
            qq = fmaf(qr[h][k], qr[h][k], qq);
            tw = fmaf(wv[h][k], qr[h][k], tw);
          }
          tw = dev::warp_sum(tw);
          qq = dev::warp_sum(qq);
          tau_h[h] = (learned ? tw + bc[h] : bc[h]) - a.offset_a;
          qn_h[h] = sqrtf(qq);
        }
      }
      // head masks of the chunk's blocks: lane l <-> block blk0 + l
      unsigned mymask = lane < cur.nloc ? ((1u << G) - 1u) : 0u;  // forced window / screen off
      if (cur.nscreen > 0) {
        if (have_nxt) dev::cp_async_wait<1>(); else dev::cp_async_wait<0>();  // this chunk's block norms
        __syncwarp();
        if (!dev::warp_wait_or_abort(&B.meta[buf], meta_phase[buf], a.status, abort_flag)) { ok = false; break; }
        meta_phase[buf] ^= 1u;
        meta_pending[buf] = 0;
        const uint8_t* mu_s = base + L.meta + static_cast<size_t>(buf) * 2 * C * D * 2;
        const uint8_t* sg_s = mu_s + C * D * 2;
        const float* mn = reinterpret_cast<const float*>(base + L.mnorm) + buf * C;
        const float scale = a.scale, z = a.z;
        const bool strict = isinf(z);
        const int vb = lane / NV, vq = lane % NV;
        for (int gb = 0; gb < cur.nscreen; gb += NB) {
          float v[32];
#pragma unroll
          for (int u = 0; u < NB; ++u) {
            const int lb = min(gb + u, cur.nscreen - 1);
            const uint2 mm = *reinterpret_cast<const uint2*>(mu_s + (lb * D + lane * CPL) * 2);
            const uint2 gg = *reinterpret_cast<const uint2*>(sg_s + (lb * D + lane * CPL) * 2);
            float mu[CPL], s2[CPL];
            mu[0] = dev::fp16_to_f32(static_cast<uint16_t>(mm.x & 0xffffu));
            mu[1] = dev::fp16_to_f32(static_cast<uint16_t>(mm.x >> 16));
            mu[2] = dev::fp16_to_f32(static_cast<uint16_t>(mm.y & 0xffffu));
            mu[3] = dev::fp16_to_f32(static_cast<uint16_t>(mm.y >> 16));
            const float g0 = dev::fp16_to_f32(static_cast<uint16_t>(gg.x & 0xffffu));
            const float g1 = dev::fp16_to_f32(static_cast<uint16_t>(gg.x >> 16));
            const float g2 = dev::fp16_to_f32(static_cast<uint16_t>(gg.y & 0xffffu));
            const float g3 = dev::fp16_to_f32(static_cast<uint16_t>(gg.y >> 16));
            s2[0] = g0 * g0;
            s2[1] = g1 * g1;
            s2[2] = g2 * g2;
            s2[3] = g3 * g3;
#pragma unroll
            for (int h = 0; h < G; ++h) {
              float dot = 0.f, sq = 0.f;
#pragma unroll
              for (int k = 0; k < CPL; ++k) {
                dot = fmaf(qr[h][k], mu[k], dot);
                sq = fmaf(q2[h][k], s2[k], sq);
              }
              v[u * NV + h] = dot;
              v[u * NV + G + h] = sq;
            }
          }
          float redv = dev::transpose_reduce32<32>(v, lane);
          const float sqv = __shfl_down_sync(0xffffffffu, redv, G);  // sum q^2 sigma^2 of the same (block, head)
          const int lb = gb + vb;
          bool pass = false;
          if (vq < G && lb < cur.nscreen) {
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
            const unsigned m = (bal >> (u * NV)) & ((1u << G) - 1u);
            if (lane == gb + u && gb + u < cur.nscreen) mymask = m;
          }
        }
      }
      // ascending admitted list of the chunk (selection export) and its tiles
      const unsigned adm = __ballot_sync(0xffffffffu, mymask != 0u);
      const int nadm = __popc(adm);
      if (mymask != 0u) {
        const int k = __popc(adm & ((1u << lane) - 1u));
        a.chunk_list[static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(cur.cidx) * C + k] =
            (blk0 + lane) | static_cast<int>(mymask << kEntryBlockBits);
      }
      if (lane == 0) a.chunk_count[static_cast<size_t>(seg) * s.nchunks + cur.cidx] = nadm;
      // rows of every block of the chunk (page table lookups in parallel)
      bool bad = false;
      const long long myrow = lane < cur.nloc ? lay.row(seg, blk0 + lane, &bad) : 0;
      if (bad) atomicOr(a.status, kStatusRange);
      const int ntile = nadm == 0 ? 1 : (nadm + BPT - 1) / BPT;
      unsigned rest = adm;
      for (int ti = 0; ti < ntile && ok; ++ti) {
        FTile ft;
        ft.seq = cur.seq;
        ft.kvh = cur.kvh;
        ft.cidx = cur.cidx;
        ft.pad0 = 0;
        ft.flags = (ti == 0 ? kFirst : 0) | (ti == ntile - 1 ? kLast : 0);
        ft.pad1 = 0;
#pragma unroll
        for (int h = 0; h < 8; ++h) ft.tau[h] = h < G ? tau_h[h] : 0.f;
        int l0 = -1, l1 = -1;
        if (rest) { l0 = __ffs(rest) - 1; rest &= rest - 1u; }
        if (BPT == 2 && rest) { l1 = __ffs(rest) - 1; rest &= rest - 1u; }
        const unsigned m0 = __shfl_sync(0xffffffffu, mymask, l0 < 0 ? 0 : l0);
        const unsigned m1 = __shfl_sync(0xffffffffu, mymask, l1 < 0 ? 0 : l1);
        const long long r0 = __shfl_sync(0xffffffffu, myrow, l0 < 0 ? 0 : l0);
        const long long r1 = __shfl_sync(0xffffffffu, myrow, l1 < 0 ? 0 : l1);
        ft.mask0 = l0 < 0 ? 0 : static_cast<int>(m0);
        ft.mask1 = l1 < 0 ? 0 : static_cast<int>(m1);
        ft.nrows0 = l0 < 0 ? 0 : min(s.b, T - (blk0 + l0) * s.b);
        ft.nrows1 = l1 < 0 ? 0 : min(s.b, T - (blk0 + l1) * s.b);
        ft.row0 = l0 < 0 ? 0 : r0;
        ft.row1 = l1 < 0 ? 0 : r1;
        if (!push(ft)) ok = false;
      }
      if (!ok) break;
      // advance: nxt becomes cur; the ticket taken above becomes nxt (its
      // metadata into the buffer cur just released)
      cur = nxt;
      have_cur = have_nxt;
      buf ^= 1;
      if (r_seg >= 0) pq_push(r_new, r_seg, 0);
      if (have_cur) {
        have_nxt = next_job(nxt);
        if (have_nxt) stage_meta(nxt, buf ^ 1);
      }
    }
    if (ok) {
      FTile end{};
      end.flags = kEnd;
      ok = push(end);
    }
    dev::cp_async_wait<0>();  // no asynchronous copy outlives the warp
    if (!ok && lane == 0) {
      *abort_flag = 1;
      for (int k = 0; k < 2; ++k) {  // staged copies land before the CTA exits
        if (!meta_pending[k]) continue;
        const long long t0 = clock64();
        while (!dev::mbar_try_wait(&B.meta[k], meta_phase[k]) && clock64() - t0 < dev::kWaitCycles) {
        }
      }
    }
  } else if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      int stage = 0, qslot = 0;
      uint32_t phase = 0, qphase = 0;
      bool ok = true;
      while (ok) {
        if (!wait_or_abort(&B.q_full[qslot], qphase, a.status, abort_flag)) { ok = false; break; }
        const FTile ft = queue[qslot];
        dev::mbar_arrive(&B.q_empty[qslot]);
        if (++qslot == kQueue) { qslot = 0; qphase ^= 1u; }
        if (!wait_or_abort(&B.kv_empty[stage], phase ^ 1u, a.status, abort_flag)) { ok = false; break; }
        info[stage] = ft;
        if (ft.flags & kEnd) {
          dev::mbar_arrive(&B.kv_full[stage]);
          break;
        }
        const uint32_t st = base_u32 + static_cast<uint32_t>(L.stages + stage * TL::STAGE);
        const int nblk = (ft.nrows0 > 0) + (ft.nrows1 > 0);
        dev::mbar_arrive_expect_tx(&B.kv_full[stage], static_cast<uint32_t>(nblk * 4 * BR * 128 + 4096));
        for (int i = 0; i < BPT; ++i) {
          const int nr = i == 0 ? ft.nrows0 : ft.nrows1;
          if (nr <= 0) continue;
          const int krow = static_cast<int>(i == 0 ? ft.row0 : ft.row1);
          const uint32_t ro = static_cast<uint32_t>(i * BR * 128);
          tma_load_2d(st + TL::K0 + ro, &tk, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::K1 + ro, &tk, 64, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V0 + ro, &tv, 0, krow, &B.kv_full[stage]);
          tma_load_2d(st + TL::V1 + ro, &tv, 64, krow, &B.kv_full[stage]);
        }
        const int qrow = (ft.seq * s.Hkv + ft.kvh) * G;
        tma_load_2d(st + TL::Q0, &tq, 0, qrow, &B.kv_full[stage]);
        tma_load_2d(st + TL::Q1, &tq, 64, qrow, &B.kv_full[stage]);
        issued_parity[stage] = static_cast<int>(phase);
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        for (int k = 0; k < kStages; ++k) {  // let issued copies land
          if (issued_parity[k] < 0) continue;
          const long long t0 = clock64();
          while (!dev::mbar_try_wait(&B.kv_full[k], static_cast<uint32_t>(issued_parity[k])) &&
                 clock64() - t0 < dev::kWaitCycles) {
          }
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
    int j = 0;
    for (;; ++j) {
      const int st_j = j % kStages;
      const int sb = j & 1;
      if (!wait_or_abort(&B.kv_full[st_j], (j / kStages) & 1, a.status, abort_flag)) { ok = false; break; }
      if (info[st_j].flags & kEnd) break;
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
    if (ok && j > 0) issue_pv(j - 1);
    if (lane == 0) mma_commit(B.done);
    __syncwarp();
    {
      const long long t0 = clock64();
      while (!dev::mbar_try_wait(B.done, 0) && clock64() - t0 < dev::kWaitCycles) {
      }
    }
  } else if (warp == kDoneWarp) {
    // ============================================================ completion
    // Events arrive in the order the softmax warps posted them; each
    // increments the counter of its parent node, and the thread that
    // completes a node resets the counter.  While the CTA still streams tiles
    // the completed nodes only queue up here (counting never waits for a
    // fold, so a busy CTA does not attract more folds); once the softmax
    // warps are done (their END event) the nodes go to them as fold jobs,
    // each staged with one bulk copy into the then idle K/V stage memory.
    // A node whose fold completes its parent queues the parent in turn.
    int eslot = 0, jslot = 0, outstanding = 0;
    uint32_t ephase = 0, jphase = 0;
    bool got_end = false, ok = true;
    unsigned* pend_nodes = reinterpret_cast<unsigned*>(base + L.pend);
    int phead = 0, npend = 0;
    auto pack = [](int level, int seg, int node) -> unsigned {
      return (static_cast<unsigned>(level) << 28) | (static_cast<unsigned>(seg) << 14) | static_cast<unsigned>(node);
    };
    // node (level, node) of segment seg has its partial (or, at the root,
    // the output): count it at its parent; a completed parent is queued (or,
    // with the queue full, folded by this warp alone from global memory)
    auto complete_up = [&](int seq, int kvh, int level, int node) {
      const int seg = seq * s.Hkv + kvh;
      for (;;) {
        const int nl = tb.nodes(seq, level);
        if (level > 0 && nl == 1) return;  // the root: the output is written
        const int lp = level + 1;
        const int parent = node / kFoldFan;
        const int nchild = min(kFoldFan, nl - parent * kFoldFan);
        unsigned* ctr = a.counters + a.cbase[lp] + static_cast<size_t>(seg) * s.M[lp] + parent;
        int complete = 0;
        __syncwarp();  // this warp's fold writes precede the release below
        if (lane == 0) {
          const unsigned before = atom_add_acq_rel(ctr, 1u);
          complete = before + 1u == static_cast<unsigned>(nchild);
          if (complete) *ctr = 0u;  // back to zero for the next step
        }
        complete = __shfl_sync(0xffffffffu, complete, 0);
        if (!complete) return;
        __syncwarp();  // the other lanes' reads of the children follow lane 0's acquire
        if (npend < kPendNodes) {
          if (lane == 0) pend_nodes[(phead + npend) % kPendNodes] = pack(lp, seg, parent);
          __syncwarp();
          ++npend;
          return;
        }
        const int nparent = tb.nodes(seq, lp);
        const size_t first = static_cast<size_t>(seg) * s.M[level] + static_cast<size_t>(parent) * kFoldFan;
        float* dst = nparent == 1 ? nullptr : a.lpart[lp] + (static_cast<size_t>(seg) * s.M[lp] + parent) * G * FPS;
        fold_partials<G>(a.lpart[level], first, nchild, dst, a, seq, kvh, 0, 1, lane);
        level = lp;
        node = parent;
      }
    };
    long long idle_since = clock64();
    while (ok) {
      if (got_end && outstanding == 0 && npend == 0) break;
      bool progress = false;
      // a queued node to the softmax warps, if a job slot is free
      if (got_end && npend > 0 &&
          __shfl_sync(0xffffffffu, dev::mbar_test_wait(&B.job_empty[jslot], jphase ^ 1u) ? 1 : 0, 0)) {
        if (lane == 0) {
          const unsigned pk = pend_nodes[phead];
          const int seg = static_cast<int>((pk >> 14) & 0x3fffu);
          jobs[jslot] = Job{0, seg / s.Hkv, seg % s.Hkv, static_cast<int>(pk >> 28), static_cast<int>(pk & 0x3fffu),
                            {0, 0, 0}};
          dev::mbar_arrive(&B.job_full[jslot]);
        }
        __syncwarp();
        if (++jslot == kJobs) { jslot = 0; jphase ^= 1u; }
        phead = (phead + 1) % kPendNodes;
        --npend;
        ++outstanding;
        progress = true;
      }
      // the next event, if one is there
      if (__shfl_sync(0xffffffffu, dev::mbar_test_wait(&B.ev_full[eslot], ephase) ? 1 : 0, 0)) {
        const Event ev = events[eslot];
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&B.ev_empty[eslot]);
        if (++eslot == kEvents) { eslot = 0; ephase ^= 1u; }
        if (ev.kind == 1) {
          got_end = true;
        } else {
          if (ev.level > 0) --outstanding;  // a fold the softmax warps ran
          complete_up(ev.seq, ev.kvh, ev.level, ev.node);
        }
        progress = true;
      }
      if (progress) {
        idle_since = clock64();
      } else if (*abort_flag) {
        ok = false;
      } else if (clock64() - idle_since > dev::kWaitCycles) {
        if (lane == 0) atomicOr(a.status, kStatusTimeout);
        ok = false;
      }
    }
    Job fin{1, 0, 0, 0, 0, {0, 0, 0}};
    if (!ok) *abort_flag = 1;
    // lets the softmax warps finish (they also stop on an abort)
    if (dev::warp_wait_or_abort(&B.job_empty[jslot], jphase ^ 1u, a.status, abort_flag)) {
      if (lane == 0) {
        jobs[jslot] = fin;
        dev::mbar_arrive(&B.job_full[jslot]);
      }
      __syncwarp();
    }
  } else {
    // ============================================================ softmax / correction / folds
    const int q4 = warp & 3;  // tensor-memory lane quarter of this warp
    const int w4 = warp - 2;  // 0..3
    const uint32_t tlane = static_cast<uint32_t>(32 * q4) << 16;
    const int row = 32 * q4 + lane;  // key row of the tile this thread owns in S^T
    const int rblk = row / BR, rrow = row - rblk * BR;
    const int dcol = 32 * q4 + lane;  // output coordinate of this thread in O^T
    const float scale = a.scale, beta = a.beta;
    // the current chunk's running state, and the previous chunk's while its
    // last tile's O^T is folded in (one tile after the chunk ended)
    float m_run[G], l_thr[G], acc[G], alpha_prev[G], tau_h[G];
    float m_old[G], l_old[G], acc_old[G], alpha_old[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_run[h] = -INFINITY;
      l_thr[h] = 0.f;
      acc[h] = 0.f;
      alpha_prev[h] = 1.f;
      tau_h[h] = 0.f;
      m_old[h] = -INFINITY;
      l_old[h] = 0.f;
      acc_old[h] = 0.f;
      alpha_old[h] = 1.f;
    }
    int cur_seq = 0, cur_kvh = 0, cur_cidx = 0, old_seq = 0, old_kvh = 0, old_cidx = 0;
    bool have_old = false;
    uint32_t rv_phase = 0;
    int eslot = 0, jslot = 0;
    uint32_t ephase = 0, jphase = 0;
    bool ok = true;

    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(B.rv);
      const bool r = wait_or_abort(B.rv, rv_phase, a.status, abort_flag);
      rv_phase ^= 1u;
      return r;
    };
    // Every softmax warp waits for the slot, (w4 == 0) writes the record,
    // and arrives once after its own writes: the completion warp sees the
    // event when all four warps' writes are done.
    auto post_event = [&](const Event& ev) -> bool {
      if (!dev::warp_wait_or_abort(&B.ev_empty[eslot], ephase ^ 1u, a.status, abort_flag)) return false;
      if (w4 == 0 && lane == 0) events[eslot] = ev;
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.ev_full[eslot]);
      if (++eslot == kEvents) { eslot = 0; ephase ^= 1u; }
      return true;
    };
    // One fold job (all four warps), after the last tile: the children are
    // staged with one bulk copy into the K/V stage memory (idle by now),
    // folded from there, and the job's event follows.
    uint32_t fold_phase = 0;
    auto run_job = [&](const Job& jb) -> bool {
      if (!rendezvous()) return false;  // the previous job's reads of the staged children are done
      const int seg = jb.seq * s.Hkv + jb.kvh;
      const int nl = tb.nodes(jb.seq, jb.level);
      const int nprev = tb.nodes(jb.seq, jb.level - 1);
      const int first = jb.node * kFoldFan;
      const int n = min(kFoldFan, nprev - first);
      const float* src = a.lpart[jb.level - 1] + (static_cast<size_t>(seg) * s.M[jb.level - 1] + first) * G * FPS;
      float* sm = reinterpret_cast<float*>(base + L.stages);
      if (w4 == 0 && lane == 0) {
        // the children were written by other CTAs (ordered before the
        // completion warp's acquire): visible to the bulk copy's proxy too
        asm volatile("fence.proxy.async.global;" ::: "memory");
        const uint32_t bytes = static_cast<uint32_t>(n) * G * FPS * sizeof(float);
        dev::mbar_arrive_expect_tx(B.fold, bytes);
        dev::bulk_g2s(sm, src, bytes, B.fold);
      }
      if (!dev::warp_wait_or_abort(B.fold, fold_phase, a.status, abort_flag)) return false;
      fold_phase ^= 1u;
      float* dst = nl == 1 ? nullptr : a.lpart[jb.level] + (static_cast<size_t>(seg) * s.M[jb.level] + jb.node) * G * FPS;
      fold_staged<G>(sm, n, dst, a, jb.seq, jb.kvh, w4, lane);
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.job_empty[jslot]);
      if (++jslot == kJobs) { jslot = 0; jphase ^= 1u; }
      Event ev{0, jb.seq, jb.kvh, jb.level, jb.node, {0, 0, 0}};
      return post_event(ev);
    };
    auto correction = [&](int i, float (&accx)[G], const float (&alphax)[G]) -> bool {
      const int ob = i & 1;
      if (!dev::warp_wait_or_abort(&B.o_full[ob], (i >> 1) & 1, a.status, abort_flag)) return false;
      tc_fence_after();
      float o[8];
      tmem_ld8(tmem + tlane + 32 + ob * 16, o);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.o_free[ob]);
#pragma unroll
      for (int h = 0; h < G; ++h) accx[h] = fmaf(accx[h], alphax[h], o[h]);
      return true;
    };
    // A finished chunk's partial into its slot (each warp its columns and
    // its share of l), then its event.
    auto flush = [&](const float (&accx)[G], const float (&mx)[G], const float (&lx)[G], int seq, int kvh,
                     int cidx) -> bool {
      const int seg = seq * s.Hkv + kvh;
      float* part = a.lpart[0] + (static_cast<size_t>(seg) * s.M[0] + cidx) * G * FPS;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        part[h * FPS + dcol] = accx[h];
        const float lw = dev::warp_sum(lx[h]);
        if (lane == 0) {
          part[h * FPS + D + 1 + q4] = lw;
          if (q4 == 0) part[h * FPS + D] = mx[h];
        }
      }
      Event ev{0, seq, kvh, 0, cidx, {0, 0, 0}};
      return post_event(ev);
    };

    int pending = -1;  // tile whose O^T is not folded in yet
    for (int j = 0; ok; ++j) {
      const int st_j = j % kStages;
      if (!wait_or_abort(&B.kv_full[st_j], (j / kStages) & 1, a.status, abort_flag)) { ok = false; break; }
      const FTile in = info[st_j];
      if (in.flags & kEnd) break;
      if (in.flags & kFirst) {
        if (pending >= 0) {  // the previous chunk is folded in and flushed after this tile's softmax
#pragma unroll
          for (int h = 0; h < G; ++h) {
            m_old[h] = m_run[h];
            l_old[h] = l_thr[h];
            acc_old[h] = acc[h];
            alpha_old[h] = alpha_prev[h];
          }
          old_seq = cur_seq;
          old_kvh = cur_kvh;
          old_cidx = cur_cidx;
          have_old = true;
        }
        cur_seq = in.seq;
        cur_kvh = in.kvh;
        cur_cidx = in.cidx;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          m_run[h] = -INFINITY;
          l_thr[h] = 0.f;
          acc[h] = 0.f;
          tau_h[h] = in.tau[h];
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
        // rows of a tile that hold no key (past a sequence end, an absent
        // second block, or a chunk with nothing admitted) are zeroed in V so
        // that stale or non-finite bytes there cannot reach the accumulator
        uint8_t* vb = base + L.stages + st_j * TL::STAGE + TL::V0;
        for (int bi = 0; bi < BPT; ++bi) {
          const int nr = max(0, bi == 0 ? in.nrows0 : in.nrows1);
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
      if (pending >= 0) {
        if (have_old) {
          if (!correction(pending, acc_old, alpha_old) ||
              !flush(acc_old, m_old, l_old, old_seq, old_kvh, old_cidx)) { ok = false; break; }
          have_old = false;
        } else if (!correction(pending, acc, alpha_prev)) {
          ok = false;
          break;
        }
      }
#pragma unroll
      for (int h = 0; h < G; ++h) alpha_prev[h] = alpha[h];
      pending = j;
    }
    if (ok && pending >= 0) ok = correction(pending, acc, alpha_prev) && flush(acc, m_run, l_thr, cur_seq, cur_kvh, cur_cidx);
    // no chunk follows: tell the completion warp, then run the folds it
    // hands over until it reports that nothing is left
    if (ok) {
      Event fin{1, 0, 0, 0, 0, {0, 0, 0}};
      ok = post_event(fin);
    }
    while (ok) {
      if (!dev::warp_wait_or_abort(&B.job_full[jslot], jphase, a.status, abort_flag)) { ok = false; break; }
      const Job jb = jobs[jslot];
      if (jb.kind == 1) break;
      if (!run_job(jb)) ok = false;
    }
    if (!ok) *abort_flag = 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
  // The last CTA to finish sets the hand-out counters back to zero for the
  // next step (the fold-tree counters were reset by their completers).
  if (t == 0) *reinterpret_cast<volatile int*>(base + L.misc + 32) =
      atom_add_acq_rel(&a.ctrl[1], 1u) + 1u == gridDim.x ? 1 : 0;
  __syncthreads();
  if (*reinterpret_cast<volatile int*>(base + L.misc + 32)) {
    const int nw = (s.nseg + 31) / 32;
    for (int x = t; x < s.nseg + nw; x += kThreads) a.counters[x] = 0u;
    if (t == 0) a.ctrl[1] = 0u;
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
  if (s.chunk < 1 || s.chunk > kMaxChunk || s.B > kFusedMaxSeqs) return 0;
  const size_t n = fused_layout(s.chunk).total;
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
