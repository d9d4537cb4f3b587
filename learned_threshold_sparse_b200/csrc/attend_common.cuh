// Work split shared by the attention kernels.
//
// The screen writes, per (segment = (sequence, KV head), chunk), the admitted
// blocks of the chunk in ascending order plus their count.  Read in
// (segment, chunk) order these lists form one global sequence of "units"
// (segment, block, head mask).  Every persistent attention CTA takes an equal
// contiguous range [U c / N, U (c + 1) / N) of it, so the K/V bytes a CTA
// streams do not depend on how the densities vary across sequences and heads.
#pragma once

#include "eta_device.cuh"

namespace eta {
namespace dev {

struct UnitInfo {
  int seg, blk, mask, nrows;
  long long row;  // first K/V row of the block in the cache's [rows, d] view
};

// Exclusive prefix of the chunk counts into prefix[0..n] (prefix[n] = total),
// computed by all `nthreads` threads of the CTA: one coalesced pass copies the
// counts into shared memory, then every thread scans a contiguous slice in
// place.  Ends with __syncthreads().
template <int NTHREADS>
__device__ __forceinline__ void chunk_prefix(const int* __restrict__ counts, int n, int* prefix) {
  __shared__ int s_warp[NTHREADS / 32];
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  for (int x = t; x < n; x += NTHREADS) prefix[x] = counts[x];
  __syncthreads();
  const int per = (n + NTHREADS - 1) / NTHREADS;
  const int lo = min(n, t * per), hi = min(n, lo + per);
  int sum = 0;
  for (int x = lo; x < hi; ++x) sum += prefix[x];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int woff = 0;
  for (int k = 0; k < warp; ++k) woff += s_warp[k];
  int run = woff + incl - sum;
  for (int x = lo; x < hi; ++x) {
    const int c = prefix[x];
    prefix[x] = run;
    run += c;
  }
  if (t == NTHREADS - 1) prefix[n] = woff + incl;
  __syncthreads();
}

// The same prefix computed by one warp alone (no CTA-wide barrier), for
// tables small enough that a lane's slice stays short.  Ends with __syncwarp().
constexpr int kWarpPrefixMax = 2048;

__device__ __forceinline__ void warp_prefix(const int* __restrict__ counts, int n, int* prefix) {
  const int lane = threadIdx.x & 31;
  for (int x = lane; x < n; x += 32) prefix[x] = counts[x];
  __syncwarp();
  const int per = (n + 31) / 32;
  const int lo = min(n, lane * per), hi = min(n, lo + per);
  int sum = 0;
  for (int x = lo; x < hi; ++x) sum += prefix[x];
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - sum;
  for (int x = lo; x < hi; ++x) {
    const int c = prefix[x];
    prefix[x] = run;
    run += c;
  }
  if (lane == 31) prefix[n] = incl;
  __syncwarp();
}

// Split of the U units over N CTAs: CTA c owns [start(c), start(c + 1)) with
// start(c) = floor(U c / N).  The host keeps U below 2^24 (segments x chunks
// and the chunk size are both bounded) and N is a few hundred at most, so
// with U = q N + r every product below fits in 32 bits.
struct UnitSplit {
  unsigned U, N, q, r;
  __device__ __forceinline__ UnitSplit(unsigned u, unsigned n) : U(u), N(n), q(u / n), r(u % n) {}
  __device__ __forceinline__ unsigned start(unsigned c) const { return q * c + (r * c) / N; }
  __device__ __forceinline__ bool owns_any(unsigned c) const { return start(c) != start(c + 1); }
  // The CTA whose range holds unit u < U: a floating-point estimate of
  // u N / U, corrected to the exact range boundaries.
  __device__ __forceinline__ unsigned owner(unsigned u) const {
    unsigned c = static_cast<unsigned>((static_cast<float>(u) + 0.5f) * static_cast<float>(N) / static_cast<float>(U));
    if (c > N - 1) c = N - 1;
    while (c + 1 < N && start(c + 1) <= u) ++c;
    while (c > 0 && start(c) > u) --c;
    return c;
  }
};

// What the screen (and the top-1 rescue after it) promise about chunk cin of
// a segment: 0 <= count <= chunk, and `count` entries (head mask << 24 |
// block) whose blocks ascend strictly inside [cin chunk, min((cin + 1) chunk,
// nblocks)), nblocks = ceil(T / b), each with a non-zero mask inside the
// group's G bits.  A walker checks every entry before it reads the page
// table or streams a row; an entry that breaks the promise stops the CTA and
// sets kStatusList, so a corrupted or stale table yields an error, never rows
// the screen did not admit.  Both predicates compile for the host as well.
// ETA_LIST_CHECK_BEGIN
constexpr unsigned kFaultCount = 1u;  // count outside [0, chunk]
constexpr unsigned kFaultBlock = 2u;  // block outside the chunk or past the sequence
constexpr unsigned kFaultOrder = 4u;  // block not above the entry before it
constexpr unsigned kFaultMask = 8u;   // empty head mask, or bits beyond G

__host__ __device__ __forceinline__ unsigned chunk_count_faults(int chunk, int count) {
  return (count < 0 || count > chunk) ? kFaultCount : 0u;
}

// prev_blk: the block of the entry before this one in the same chunk, or -1.
__host__ __device__ __forceinline__ unsigned list_entry_faults(int chunk, int G, int nblocks, int cin, int entry,
                                                               int prev_blk) {
  const int blk = entry & ((1 << 24) - 1);
  const unsigned mask = static_cast<unsigned>(entry) >> 24;
  const int lo = cin * chunk;
  const int hi = nblocks < lo + chunk ? nblocks : lo + chunk;
  unsigned f = 0u;
  if (blk < lo || blk >= hi) f |= kFaultBlock;
  if (blk <= prev_blk) f |= kFaultOrder;
  if (mask == 0u || (mask >> G) != 0u) f |= kFaultMask;
  return f;
}
// ETA_LIST_CHECK_END

// Walk the units [u0, u0 + nunits) with one warp.  `issue(info)` runs on lane
// 0 for every unit, in order, and returns false to stop (abort).  Returns
// false if the walk was stopped or the tables broke the promise above (then
// kStatusList is set).  seq_T, when not null, holds the clamped sequence
// lengths in shared memory.
template <class Issue>
__device__ __forceinline__ bool walk_units(const AttendArgs& a, const int* prefix, int nprefix, int u0, int nunits,
                                           const int* seq_T, Issue&& issue) {
  const Shape& s = a.s;
  const int lane = threadIdx.x & 31;
  int lo = 0, hi = nprefix;  // invariant prefix[lo] <= u0 < prefix[hi]
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] <= u0) lo = mid; else hi = mid;
  }
  int x = lo;
  int idx = u0 - prefix[x];
  int remaining = nunits;
  int cur_seg = -1, T = 0, nblk = 0;
  const KvLayout lay{a.block_table, s.Hkv, s.b, s.max_ctx, s.nbmax, s.num_pages};
  auto fail = [&]() {
    if (lane == 0) atomicOr(a.status, kStatusList);
    return false;
  };
  while (remaining > 0) {
    if (x >= nprefix) return fail();
    const int cnt = prefix[x + 1] - prefix[x];
    if (chunk_count_faults(s.chunk, cnt)) return fail();
    const int take = min(cnt - idx, remaining);
    if (take <= 0) { ++x; idx = 0; continue; }
    const int seg = x / s.nchunks;
    const int cin = x - seg * s.nchunks;
    if (seg != cur_seg) {
      cur_seg = seg;
      if (seq_T) {
        T = seq_T[seg / s.Hkv];
      } else {
        const int tt = a.seq_lens[seg / s.Hkv];
        T = tt < 0 ? 0 : (tt > s.max_ctx ? s.max_ctx : tt);
      }
      nblk = (T + s.b - 1) / s.b;
    }
    const int* list = a.chunk_list + static_cast<size_t>(seg) * s.list_stride + static_cast<size_t>(cin) * s.chunk + idx;
    int last = -1;  // block of the entry before the batch (-1: none read in this chunk)
    for (int j0 = 0; j0 < take; j0 += 32) {
      const int nn = min(32, take - j0);
      const int e = lane < nn ? list[j0 + lane] : 0;
      const int eb = e & kMaxBlocksPerSeq;
      const int up = __shfl_up_sync(0xffffffffu, eb, 1);
      const unsigned f = lane < nn ? list_entry_faults(s.chunk, s.G, nblk, cin, e, lane == 0 ? last : up) : 0u;
      if (__any_sync(0xffffffffu, f != 0u)) return fail();
      last = __shfl_sync(0xffffffffu, eb, nn - 1);
      // the rows of the 32 listed blocks (one page-table read per lane)
      bool bad = false;
      const long long rw = lane < nn ? lay.row(seg, e & kMaxBlocksPerSeq, &bad) : 0;
      if (bad) atomicOr(a.status, kStatusRange);
      for (int jj = 0; jj < nn; ++jj) {
        const int ent = __shfl_sync(0xffffffffu, e, jj);
        const long long er = __shfl_sync(0xffffffffu, rw, jj);
        int ok = 1;
        if (lane == 0) {
          const int blk = ent & kMaxBlocksPerSeq;
          const UnitInfo in{seg, blk, static_cast<int>(static_cast<unsigned>(ent) >> kEntryBlockBits),
                            min(s.b, T - blk * s.b), er};
          ok = issue(in) ? 1 : 0;
        }
        if (__shfl_sync(0xffffffffu, ok, 0) == 0) return false;
      }
    }
    remaining -= take;
    idx = 0;
    ++x;
  }
  return true;
}

// Tiles of up to BPT consecutive units of one segment that the unit range
// [u0, u1) splits into (a tile never crosses a segment boundary).
template <int BPT>
__device__ __forceinline__ int count_tiles(const int* prefix, const Shape& s, int u0, int u1) {
  if (u1 <= u0) return 0;
  int lo = 0, hi = s.nseg;  // last segment whose first unit is <= u0
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid * s.nchunks] <= u0) lo = mid; else hi = mid;
  }
  int tiles = 0;
  for (int seg = lo; seg < s.nseg; ++seg) {
    const int a = max(u0, prefix[seg * s.nchunks]);
    const int b = min(u1, prefix[(seg + 1) * s.nchunks]);
    if (a >= u1) break;
    if (b > a) tiles += (b - a + BPT - 1) / BPT;
  }
  return tiles;
}

// Output element idx (kv dtype: fp32, or bf16 rounded to nearest even).
__device__ __forceinline__ void store_out_slot(void* out, int elt, size_t idx, float o) {
  if (elt == 4) {
    static_cast<float*>(out)[idx] = o;
  } else {
    static_cast<uint16_t*>(out)[idx] = f32_to_bf16_rn(o);
  }
}

__device__ __forceinline__ void store_out(const AttendArgs& a, size_t idx, float o) {
  store_out_slot(a.out, a.s.elt, idx, o);
}

__device__ __forceinline__ float lse_of(float m2, float l) {
  return l > 0.f ? (m2 + log2f(l)) * 0.6931471805599453f : -INFINITY;
}

// Bounded wait that also gives up as soon as another role raised the CTA's
// abort flag; a timeout raises it.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity, unsigned* status,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) {
      atomicOr(status, kStatusTimeout);
      *abort_flag = 1;
      return false;
    }
  }
  return true;
}

// wait_or_abort by a whole warp with one answer for all lanes: warp-wide
// instructions (tensor-memory loads and stores) may follow it.
__device__ __forceinline__ bool warp_wait_or_abort(uint64_t* bar, uint32_t parity, unsigned* status,
                                                   volatile int* abort_flag) {
  return __all_sync(0xffffffffu, wait_or_abort(bar, parity, status, abort_flag) ? 1 : 0) != 0;
}

}  // namespace dev
}  // namespace eta
