// Internal declarations shared by the launchers and the C ABI of the ETA
// decode library.  Not installed; the public interface is include/eta.h.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

#include "eta.h"

namespace eta {

// Floats per (partial slot, head): d accumulator entries, m, l, 2 pad so
// every row starts 16-byte aligned.
__host__ __device__ constexpr int partial_stride(int d) { return d + 4; }
// Fused path: d accumulator entries, m, the four softmax warps' shares of l
// (summed in a fixed order when read), 3 pad.

// Device status word bits (first word of the workspace).
constexpr unsigned kStatusTimeout = ETA_DEVICE_STATUS_TIMEOUT;  // a bounded wait ran out
constexpr unsigned kStatusRange = ETA_DEVICE_STATUS_RANGE;      // a device-resident length was clamped
constexpr unsigned kStatusList = ETA_DEVICE_STATUS_LIST;        // a walker found inconsistent chunk tables

// List entries written by the screen: block id in the low 24 bits, the
// admitting heads of the group in the high 8 bits.
constexpr int kEntryBlockBits = 24;
constexpr int kMaxBlocksPerSeq = (1 << kEntryBlockBits) - 1;

// Shape of one decode launch, derived on the host from eta_decode_params.
struct Shape {
  int B, Hq, Hkv, G, d, b, max_ctx, nbmax;
  int elt;           // bytes per K/V element
  int nseg;          // B * Hkv  (one segment = one (sequence, KV head))
  int chunk;         // blocks screened per screen CTA (multiple of 32)
  int nchunks;       // chunks per segment
  int list_stride;   // list entries per segment = nchunks * chunk
  int attend_ctas;   // persistent attention CTAs
  int attend_kind;   // ETA_ATTEND_SIMT or ETA_ATTEND_TC
  int rescue;        // 1 when n_local_blocks < 0 (top-1 rescue may fire)
  int num_pages;     // paged cache: pages in the pools (0: contiguous cache)
  int fused;         // 1: one fused kernel screens, attends and merges (chunks of `chunk` blocks)
};

// Fused path: sequence tables of up to kFusedMaxSeqs sequences live in
// shared memory, a CTA's slice holds at most kFusedMaxSlice chunks, and the
// grid has at most kFusedMaxCtas CTAs (one slice total each in the control
// region).
constexpr int kFusedMaxSeqs = 256;
constexpr int kFusedMaxSlice = 64;
constexpr int kFusedMaxCtas = 1024;

// Where the K/V rows of logical block blk of segment seg (sequence
// seg / Hkv, KV head seg % Hkv) start, as a row index of the [rows, d] view
// of the cache: contiguous  seg max_ctx + blk b;  paged
// (page Hkv + g) b with page = table[i nb_max + blk].  An out-of-range page
// id reads page 0 and sets *bad.
struct KvLayout {
  const int* table;  // null: contiguous
  int Hkv, b, max_ctx, nbmax, num_pages;
  __host__ __device__ long long row(int seg, int blk, bool* bad) const {
    if (!table) return static_cast<long long>(seg) * max_ctx + static_cast<long long>(blk) * b;
    const int i = seg / Hkv, g = seg - i * Hkv;
    int page = table[static_cast<size_t>(i) * nbmax + blk];
    if (page < 0 || page >= num_pages) {
      *bad = true;
      page = 0;
    }
    return (static_cast<long long>(page) * Hkv + g) * b;
  }
};

// Byte offsets of the workspace regions (all 256-byte aligned).
struct Workspace {
  size_t status, ctrl, counters, tau, chunk_count, chunk_list, head_count, head_best, partials, total;
};

// Leading control region of every workspace, at fixed offsets whatever the
// shapes of a call: the status word, the fused path's finished-CTA counter,
// its published slice totals and its per-segment piece counters.  They are
// back at zero after every completed step (the last CTA to finish clears the
// totals, the merger of a segment clears its counter), so calls of any
// shapes may share a workspace; the region must be zero before the first
// call.
constexpr size_t kCtrlOffset = 64;
constexpr size_t kCounterOffset = 4096;
constexpr int kMaxCounters = 16384;
// Inside the counter area: [kFusedMaxCtas] slice totals, then the segment
// counters (64-bit, at most 2048 segments).
constexpr int kFusedSegCtrOffset = kFusedMaxCtas;
constexpr size_t kControlBytes = kCounterOffset + kMaxCounters * sizeof(unsigned);
static_assert(kControlBytes == ETA_WORKSPACE_CONTROL_BYTES, "control region size in the public header");

Workspace workspace_layout(const Shape& s);

// Arguments of the screen kernel.
struct ScreenArgs {
  const void* q;
  const float* w_tau;
  const float* b_tau;
  const float* c_tau;
  const void* mu;         // fp16 bits or e4m3 codes (meta_fmt)
  const void* sigma;
  const float* max_norm;
  const float* mu_scale;     // fp8 format: per-block scales
  const float* sigma_scale;
  int meta_fmt;              // ETA_META_FP16 / ETA_META_FP8
  const int* seq_lens;
  int tau_mode, lwb, screen_enabled;
  float scale, offset_a, z;
  Shape s;
  unsigned* status;
  float* tau;              // [B, Hq] tau~
  int* chunk_count;        // [nseg, nchunks]
  int* chunk_list;         // [nseg, list_stride]
  void* out;               // written here only for empty sequences
  float* lse;
  int* head_count;         // [B, Hq]   (rescue mode)
  unsigned long long* head_best;  // [B, Hq] (rescue mode)
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

struct AttendArgs {
  const void* k;
  const void* v;
  const int* block_table;  // paged cache (else null), see KvLayout
  const void* q;
  const int* seq_lens;
  const float* tau;
  const int* chunk_count;
  const int* chunk_list;
  float scale, beta;
  Shape s;
  unsigned* status;
  float* partials;         // [nseg + attend_ctas][G][partial_stride(d)]
  void* out;               // [B, Hq, d] kv dtype: segments owned by one CTA
  float* lse;              // [B, Hq] or null
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

// Arguments of the fused decode kernel (screen + attention + merge).
struct FusedArgs {
  const void* k;
  const void* v;
  const int* block_table;  // paged cache (else null), see KvLayout
  const void* q;
  const int* seq_lens;
  const float* w_tau;
  const float* b_tau;
  const float* c_tau;
  const void* mu;          // fp16 metadata
  const void* sigma;
  const float* max_norm;
  int tau_mode, lwb, screen_enabled;
  float scale, beta, offset_a, z;
  Shape s;
  unsigned* status;
  unsigned* done_ctas;             // [1] CTAs finished
  unsigned* arrived;               // [1] slice totals published
  unsigned* flags;                 // [grid] slice totals + 1 (0: not published yet)
  unsigned long long* seg_ctr;     // [nseg] pieces announced per segment (fields: see the kernel)
  float* tau;                      // [B, Hq] tau~ (written by the screen, read by the softmax)
  int* chunk_count;                // [nseg, nchunks]  admitted blocks per chunk
  int* chunk_list;                 // [nseg, list_stride]
  float* partials;                 // [2 grid][G][partial_stride(d)] pieces of shared segments
  void* out;
  float* lse;
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

struct MergeArgs {
  const int* chunk_count;  // [nseg, nchunks] admitted entries per chunk (screen output)
  const float* partials;
  Shape s;
  void* out;
  float* lse;
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

struct ExportArgs {
  const int* chunk_count;
  const int* chunk_list;
  const int* seq_lens;
  Shape s;
  int* admitted_count;
  int* union_count;
  int* union_list;
  unsigned* union_mask;
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

// Arguments of the causal forward (prefill) kernel; q, k, v also feed the
// host-side tensor maps.
struct PrefillArgs {
  const void* q;
  const void* k;
  const void* v;
  const float* w_tau;
  const float* b_tau;
  const float* c_tau;
  void* out;
  float* lse;
  float* gate_sum;
  unsigned* status;
  int B, Hq, Hkv, G, T, kv_stride, tau_mode;
  float scale, beta, offset_a;
};

// Arguments of the calibration histogram kernel.
struct CalibArgs {
  const void* q;           // [B, Hq, T, d] kv dtype
  const void* k;           // [B, Hkv, kv_stride, d]
  double* hist;            // [Hq, nbins + 2] (underflow, nbins bins, overflow)
  int B, Hq, Hkv, G, T, kv_stride, d, elt, nbins;
  float scale, lo, inv_width;
};

struct SummaryArgs {
  const void* k;
  const int* block_table;  // paged cache (else null), see KvLayout
  int num_pages;
  const int* seq_lens;
  const int* first_token;
  void* mu;                // fp16 bits or e4m3 codes (fmt)
  void* sigma;
  float* max_norm;
  float* mu_scale;         // fp8 format: per-block scales
  float* sigma_scale;
  int fmt;                 // ETA_META_FP16 / ETA_META_FP8
  int B, Hkv, d, b, max_ctx, nbmax, elt, max_blocks;
  // append only: the token's query rows [B, Hkv * G, d] copied from q_src
  // (device or mapped page-locked host memory) to q_dst by the same launch
  const void* q_src = nullptr;
  void* q_dst = nullptr;
  int G = 0;
  unsigned long long* trace = nullptr;  // step trace (include/eta.h) or null
};

// The append of eta_append_kv, optionally also copying the token's query
// rows q_src -> q_dst ([batch, n_q_heads, head_dim]) in the same launch
// (api.cu; used by the recorded serving step).
eta_status append_step(const eta_cache_desc* cache, const eta_summary_desc* summary, const void* k_new,
                       const void* v_new, const int* pos, const void* q_src, void* q_dst, void* stream,
                       unsigned long long* trace = nullptr);

// ---------------------------------------------------------------- host helpers
// Driver attribute queries and settings cost on the order of a microsecond
// each; a decode issues several launches, so their per-device results are
// cached here (api.cu).

constexpr int kMaxDevices = 64;

// Largest dynamic shared memory already allowed for one kernel, per device.
struct SmemLimit {
  std::atomic<int> bytes[kMaxDevices];
  void forget(int dev) {
    if (dev >= 0 && dev < kMaxDevices) bytes[dev].store(0, std::memory_order_relaxed);
  }
};

// Raises `kern`'s dynamic shared memory limit on the current device to at
// least `bytes` unless the cache says it already is; *skipped reports that.
cudaError_t ensure_smem(const void* kern, size_t bytes, SmemLimit& lim, bool* skipped);

// ensure_smem + launch().  If the launch fails after the attribute call was
// skipped (the setting can be lost, e.g. by a device reset), the attribute is
// set again and the launch retried once.
template <class Launch>
cudaError_t launch_with_smem(const void* kern, size_t bytes, SmemLimit& lim, Launch&& launch) {
  bool skipped = false;
  cudaError_t e = ensure_smem(kern, bytes, lim, &skipped);
  if (e != cudaSuccess) return e;
  e = launch();
  if (e != cudaSuccess && skipped) {
    (void)cudaGetLastError();
    int dev = -1;
    if (cudaGetDevice(&dev) == cudaSuccess) lim.forget(dev);
    e = ensure_smem(kern, bytes, lim, &skipped);
    if (e == cudaSuccess) e = launch();
  }
  return e;
}

// Streaming multiprocessors of the current device (0 on error), cached.
int device_sms();

// Launchers (each returns the launch's cudaError_t).
cudaError_t launch_summary(const SummaryArgs& a, cudaStream_t st);
cudaError_t launch_append(const SummaryArgs& a, const void* k_new, const void* v_new, const int* pos,
                          void* k_cache, void* v_cache, cudaStream_t st);
cudaError_t launch_screen(const ScreenArgs& a, cudaStream_t st);
cudaError_t launch_rescue(const ScreenArgs& a, cudaStream_t st);
cudaError_t launch_attend_simt(const AttendArgs& a, cudaStream_t st);
size_t attend_simt_smem(const Shape& s);
int attend_simt_ctas_per_sm(const Shape& s);
cudaError_t launch_attend_tc(const AttendArgs& a, cudaStream_t st);
size_t attend_tc_smem(const Shape& s);
bool attend_tc_supported(const Shape& s);
cudaError_t launch_merge(const MergeArgs& a, cudaStream_t st);
cudaError_t launch_fused_tc(const FusedArgs& a, cudaStream_t st);
size_t fused_tc_smem(const Shape& s);
cudaError_t launch_export(const ExportArgs& a, cudaStream_t st);
cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st);
cudaError_t launch_calib(const CalibArgs& a, cudaStream_t st);
size_t calib_smem(int d, int nbins);

}  // namespace eta
