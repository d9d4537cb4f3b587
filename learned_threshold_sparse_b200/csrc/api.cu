// C ABI of the ETA decode library: host-side validation, workspace layout and
// the stream-ordered launch sequence
//   screen (+ rescue) -> attention over the admitted union -> merge of the
//   split partials of segments shared by several attention CTAs (+ export).
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "eta_internal.h"

namespace eta {

namespace {

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

eta_status check_cache(const eta_cache_desc* c) {
  if (!c) return ETA_ERR_INVALID_ARG;
  if (c->batch < 1 || c->n_kv_heads < 1 || c->n_q_heads < 1 || c->max_ctx < 1 || c->block_size < 1)
    return ETA_ERR_INVALID_ARG;
  if (c->n_q_heads % c->n_kv_heads != 0) return ETA_ERR_INVALID_ARG;
  if (c->kv_dtype != ETA_F32 && c->kv_dtype != ETA_BF16) return ETA_ERR_INVALID_ARG;
  if (c->batch > 65535 || c->n_kv_heads > 65535 || c->n_q_heads > 65535) return ETA_ERR_UNSUPPORTED;
  const int G = c->n_q_heads / c->n_kv_heads;
  if (c->head_dim != 64 && c->head_dim != 128) return ETA_ERR_UNSUPPORTED;
  if (c->block_size != 16 && c->block_size != 32 && c->block_size != 64 && c->block_size != 128)
    return ETA_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return ETA_ERR_UNSUPPORTED;
  const long long nbmax = (static_cast<long long>(c->max_ctx) + c->block_size - 1) / c->block_size;
  if (nbmax > kMaxBlocksPerSeq) return ETA_ERR_UNSUPPORTED;
  if (!c->k_cache || !c->v_cache || !c->seq_lens) return ETA_ERR_INVALID_ARG;
  if (!aligned(c->k_cache, 16) || !aligned(c->v_cache, 16) || !aligned(c->seq_lens, 4))
    return ETA_ERR_INVALID_ARG;
  if (c->block_table) {
    if (!aligned(c->block_table, 4) || c->num_pages < 1) return ETA_ERR_INVALID_ARG;
    if (static_cast<long long>(c->num_pages) * c->n_kv_heads * c->block_size >= (1ll << 31))
      return ETA_ERR_UNSUPPORTED;
  }
  return ETA_OK;
}

eta_status check_summary(const eta_summary_desc* s) {
  if (!s || !s->mu || !s->sigma || !s->max_norm) return ETA_ERR_INVALID_ARG;
  if (!aligned(s->mu, 16) || !aligned(s->sigma, 16) || !aligned(s->max_norm, 4)) return ETA_ERR_INVALID_ARG;
  if (s->format != ETA_META_FP16 && s->format != ETA_META_FP8 && s->format != ETA_META_BOX)
    return ETA_ERR_INVALID_ARG;
  if (s->format == ETA_META_FP8 &&
      (!s->mu_scale || !s->sigma_scale || !aligned(s->mu_scale, 4) || !aligned(s->sigma_scale, 4)))
    return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

// The summary descriptor's fields into the kernels' arguments.
template <class Args>
void set_summary(Args& a, const eta_summary_desc* s) {
  a.mu = s->mu;
  a.sigma = s->sigma;
  a.max_norm = s->max_norm;
  a.mu_scale = s->mu_scale;
  a.sigma_scale = s->sigma_scale;
}

eta_status make_shape(const eta_decode_params* p, Shape* out) {
  const eta_cache_desc& c = p->cache;
  Shape s;
  s.B = c.batch;
  s.Hq = c.n_q_heads;
  s.Hkv = c.n_kv_heads;
  s.G = c.n_q_heads / c.n_kv_heads;
  s.d = c.head_dim;
  s.b = c.block_size;
  s.max_ctx = c.max_ctx;
  s.nbmax = (c.max_ctx + c.block_size - 1) / c.block_size;
  s.num_pages = c.block_table ? c.num_pages : 0;
  s.elt = c.kv_dtype == ETA_F32 ? 4 : 2;
  s.nseg = s.B * s.Hkv;
  // Screen CTAs cover `chunk` blocks: about two screen CTAs per SM (one
  // resident wave), and at most 4096 (segment, chunk) pairs so the attention
  // kernel's prefix table fits in shared memory.
  const int sms = device_sms();
  if (sms <= 0) return ETA_ERR_CUDA;
  const int sms_for_chunk = sms;
  int chunk = 32;
  auto pairs = [&](int ch) { return static_cast<long long>(s.nseg) * ((s.nbmax + ch - 1) / ch); };
  while (chunk < 1024 && (pairs(chunk) > 2LL * sms_for_chunk || pairs(chunk) > 4096)) chunk *= 2;
  s.chunk = chunk;
  s.nchunks = (s.nbmax + chunk - 1) / chunk;
  if (static_cast<long long>(s.nseg) * s.nchunks > 16384) return ETA_ERR_UNSUPPORTED;
  s.list_stride = s.nchunks * chunk;
  s.rescue = (p->n_local_blocks < 0 && p->screen_enabled) ? 1 : 0;
  s.fused = 0;
  const bool tc_ok = attend_tc_supported(s);
  if ((p->attend_impl == ETA_ATTEND_TC || p->attend_impl == ETA_ATTEND_FUSED) && !tc_ok) return ETA_ERR_UNSUPPORTED;
  s.attend_kind = (p->attend_impl == ETA_ATTEND_SIMT || !tc_ok) ? ETA_ATTEND_SIMT : ETA_ATTEND_TC;
  if (s.attend_kind == ETA_ATTEND_SIMT) {
    if (attend_simt_smem(s) == 0) return ETA_ERR_UNSUPPORTED;
    s.attend_ctas = sms * attend_simt_ctas_per_sm(s);
  } else {
    if (attend_tc_smem(s) == 0) return ETA_ERR_UNSUPPORTED;
    s.attend_ctas = sms;
  }
  // The fused kernel (screen, attention and merge in one launch) covers the
  // tensor-core shapes with fp16 metadata (or the screen off), the window on
  // (no rescue), batches of up to kFusedMaxSeqs sequences and up to 2048
  // (sequence, KV head) segments.
  const bool fused_ok = s.attend_kind == ETA_ATTEND_TC && !s.rescue &&
                        (!p->screen_enabled || p->summary.format == ETA_META_FP16) && s.B <= kFusedMaxSeqs &&
                        s.nseg <= 2048 && sms <= kFusedMaxCtas;
  if (fused_ok && p->attend_impl == ETA_ATTEND_FUSED) {
    // chunks of about 256 KB of K+V (8 blocks of 64 rows, 4 of 128), larger
    // when a slice (the chunks one CTA screens) would exceed kFusedMaxSlice
    Shape f = s;
    int c = s.b == 64 ? 8 : 4;
    auto chunks = [&](int cc) { return static_cast<long long>(s.nseg) * ((s.nbmax + cc - 1) / cc); };
    while (c < 32 && chunks(c) > static_cast<long long>(sms) * kFusedMaxSlice) c *= 2;
    f.fused = 1;
    f.chunk = c;
    f.nchunks = (s.nbmax + c - 1) / c;
    f.list_stride = f.nchunks * c;
    f.attend_ctas = sms;
    if (chunks(c) <= static_cast<long long>(sms) * kFusedMaxSlice && fused_tc_smem(f) != 0) {
      *out = f;
      return ETA_OK;
    }
  }
  if (p->attend_impl == ETA_ATTEND_FUSED) return ETA_ERR_UNSUPPORTED;
  *out = s;
  return ETA_OK;
}

eta_status check_params(const eta_decode_params* p) {
  if (!p) return ETA_ERR_INVALID_ARG;
  eta_status st = check_cache(&p->cache);
  if (st != ETA_OK) return st;
  if (p->screen_enabled) {
    st = check_summary(&p->summary);
    if (st != ETA_OK) return st;
  }
  if (!p->q || !aligned(p->q, 16) || !p->out || !aligned(p->out, 16)) return ETA_ERR_INVALID_ARG;
  if (p->tau_mode == ETA_TAU_LEARNED) {
    if (!p->w_tau || !p->b_tau || !aligned(p->w_tau, 4) || !aligned(p->b_tau, 4)) return ETA_ERR_INVALID_ARG;
  } else if (p->tau_mode == ETA_TAU_CALIBRATED) {
    if (!p->c_tau || !aligned(p->c_tau, 4)) return ETA_ERR_INVALID_ARG;
  } else {
    return ETA_ERR_INVALID_ARG;
  }
  if (!(p->scale > 0.f) || !isfinite(p->scale)) return ETA_ERR_INVALID_ARG;
  if (!(p->beta > 0.f) || !isfinite(p->beta)) return ETA_ERR_INVALID_ARG;
  if (!isfinite(p->offset_a)) return ETA_ERR_INVALID_ARG;
  if (!(p->z > 0.f)) return ETA_ERR_INVALID_ARG;  // +inf allowed, NaN rejected
  if (p->n_local_blocks < -1) return ETA_ERR_INVALID_ARG;
  if (p->attend_impl < ETA_ATTEND_AUTO || p->attend_impl > ETA_ATTEND_FUSED) return ETA_ERR_INVALID_ARG;
  if (p->lse && !aligned(p->lse, 4)) return ETA_ERR_INVALID_ARG;
  if ((p->admitted_count && !aligned(p->admitted_count, 4)) || (p->union_count && !aligned(p->union_count, 4)) ||
      (p->union_list && !aligned(p->union_list, 4)) || (p->union_mask && !aligned(p->union_mask, 4)))
    return ETA_ERR_INVALID_ARG;
  return ETA_OK;
}

}  // namespace

int device_sms() {
  static std::atomic<int> cache[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot) {
    const int c = cache[dev].load(std::memory_order_relaxed);
    if (c > 0) return c;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  if (slot) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

cudaError_t ensure_smem(const void* kern, size_t bytes, SmemLimit& lim, bool* skipped) {
  *skipped = false;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const int want = static_cast<int>(bytes);
  const bool slot = dev >= 0 && dev < kMaxDevices;
  if (slot && lim.bytes[dev].load(std::memory_order_relaxed) >= want) {
    *skipped = true;
    return cudaSuccess;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, want);
  if (e == cudaSuccess && slot) {
    int cur = lim.bytes[dev].load(std::memory_order_relaxed);
    while (cur < want && !lim.bytes[dev].compare_exchange_weak(cur, want, std::memory_order_relaxed)) {
    }
  }
  return e;
}

Workspace workspace_layout(const Shape& s) {
  Workspace w;
  w.status = 0;
  w.ctrl = kCtrlOffset;
  w.counters = kCounterOffset;
  size_t off = kControlBytes;  // the fixed control region comes first
  w.tau = off;
  off = align256(off + static_cast<size_t>(s.B) * s.Hq * sizeof(float));
  w.chunk_count = off;
  off = align256(off + static_cast<size_t>(s.nseg) * s.nchunks * sizeof(int));
  w.chunk_list = off;
  off = align256(off + static_cast<size_t>(s.nseg) * s.list_stride * sizeof(int) + 4 * sizeof(int));
  w.head_count = off;
  off = align256(off + static_cast<size_t>(s.B) * s.Hq * sizeof(int));
  w.head_best = off;
  off = align256(off + static_cast<size_t>(s.B) * s.Hq * sizeof(unsigned long long));
  const size_t pbytes = static_cast<size_t>(s.G) * partial_stride(s.d) * sizeof(float);
  w.partials = off;
  if (s.fused) {
    off = align256(off + 2 * static_cast<size_t>(s.attend_ctas) * pbytes);  // two pieces per CTA
  } else {
    off = align256(off + static_cast<size_t>(s.nseg + s.attend_ctas) * pbytes);
  }
  w.total = off;
  return w;
}

}  // namespace eta

using namespace eta;

extern "C" {

const char* eta_status_string(eta_status s) {
  switch (s) {
    case ETA_OK: return "ok";
    case ETA_ERR_INVALID_ARG: return "invalid argument";
    case ETA_ERR_UNSUPPORTED: return "unsupported shape or option";
    case ETA_ERR_WORKSPACE: return "workspace missing or too small";
    case ETA_ERR_CUDA: return "CUDA runtime error";
    case ETA_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait ran out";
    case ETA_ERR_DEVICE_RANGE: return "a device-resident length was out of range (clamped)";
    case ETA_ERR_DEVICE_LIST: return "inconsistent admitted-block tables (attention stopped; output not valid)";
  }
  return "unknown status";
}

const char* eta_build_info(void) {
  return "eta decode library: sm_100a; kernels: block_summary, append, fused_tc (screen + attention + merge), "
         "screen, rescue, attend_simt, attend_tc, merge, export, prefill_tc, calib_hist, io_copy, diag_wait; decode "
         "step and serving step as CUDA graphs";
}

eta_status eta_block_summary_update(const eta_cache_desc* cache, const eta_summary_desc* summary,
                                    const int* first_token, int max_blocks, void* stream) {
  eta_status st = check_cache(cache);
  if (st != ETA_OK) return st;
  st = check_summary(summary);
  if (st != ETA_OK) return st;
  if (!first_token || !aligned(first_token, 4)) return ETA_ERR_INVALID_ARG;
  const int nbmax = (cache->max_ctx + cache->block_size - 1) / cache->block_size;
  if (max_blocks < 1 || max_blocks > nbmax) return ETA_ERR_INVALID_ARG;
  SummaryArgs a;
  a.k = cache->k_cache;
  a.block_table = cache->block_table;
  a.num_pages = cache->num_pages;
  a.seq_lens = cache->seq_lens;
  a.first_token = first_token;
  set_summary(a, summary);
  a.fmt = summary->format;
  a.B = cache->batch;
  a.Hkv = cache->n_kv_heads;
  a.d = cache->head_dim;
  a.b = cache->block_size;
  a.max_ctx = cache->max_ctx;
  a.nbmax = nbmax;
  a.elt = cache->kv_dtype == ETA_F32 ? 4 : 2;
  a.max_blocks = max_blocks;
  return launch_summary(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

eta_status eta_append_kv(const eta_cache_desc* cache, const eta_summary_desc* summary, const void* k_new,
                         const void* v_new, const int* pos, void* stream) {
  return eta::append_step(cache, summary, k_new, v_new, pos, nullptr, nullptr, stream);
}

}  // extern "C"

namespace eta {

eta_status append_step(const eta_cache_desc* cache, const eta_summary_desc* summary, const void* k_new,
                       const void* v_new, const int* pos, const void* q_src, void* q_dst, void* stream,
                       unsigned long long* trace) {
  eta_status st = check_cache(cache);
  if (st != ETA_OK) return st;
  st = check_summary(summary);
  if (st != ETA_OK) return st;
  if (!k_new || !v_new || !pos || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(pos, 4))
    return ETA_ERR_INVALID_ARG;
  if ((q_src == nullptr) != (q_dst == nullptr)) return ETA_ERR_INVALID_ARG;
  if (q_src && (!aligned(q_src, 16) || !aligned(q_dst, 16))) return ETA_ERR_INVALID_ARG;
  SummaryArgs a;
  a.trace = trace;
  a.q_src = q_src;
  a.q_dst = q_dst;
  a.G = cache->n_q_heads / cache->n_kv_heads;
  a.k = cache->k_cache;
  a.block_table = cache->block_table;
  a.num_pages = cache->num_pages;
  a.seq_lens = cache->seq_lens;
  a.first_token = nullptr;
  set_summary(a, summary);
  a.fmt = summary->format;
  a.B = cache->batch;
  a.Hkv = cache->n_kv_heads;
  a.d = cache->head_dim;
  a.b = cache->block_size;
  a.max_ctx = cache->max_ctx;
  a.nbmax = (cache->max_ctx + cache->block_size - 1) / cache->block_size;
  a.elt = cache->kv_dtype == ETA_F32 ? 4 : 2;
  a.max_blocks = 1;
  // The cache descriptor's pointers are const for the decode; the append
  // writes through them by contract of this entry point.
  return launch_append(a, k_new, v_new, pos, const_cast<void*>(cache->k_cache), const_cast<void*>(cache->v_cache),
                       static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? ETA_OK
             : ETA_ERR_CUDA;
}

}  // namespace eta

extern "C" {

eta_status eta_decode_workspace_size(const eta_decode_params* p, size_t* bytes) {
  if (!bytes) return ETA_ERR_INVALID_ARG;
  eta_status st = check_params(p);
  if (st != ETA_OK) return st;
  Shape s;
  st = make_shape(p, &s);
  if (st != ETA_OK) return st;
  *bytes = workspace_layout(s).total;
  return ETA_OK;
}

eta_status eta_decode(const eta_decode_params* p, void* stream) {
  eta_status st = check_params(p);
  if (st != ETA_OK) return st;
  Shape s;
  st = make_shape(p, &s);
  if (st != ETA_OK) return st;
  const Workspace w = workspace_layout(s);
  if (!p->workspace || !aligned(p->workspace, 256)) return ETA_ERR_WORKSPACE;
  if (p->workspace_bytes < w.total) return ETA_ERR_WORKSPACE;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(p->workspace);
  auto ev = [&](int k) {
    if (p->timing_events[k]) cudaEventRecord(static_cast<cudaEvent_t>(p->timing_events[k]), cs);
  };

  ScreenArgs sa;
  sa.trace = p->trace;
  sa.q = p->q;
  sa.w_tau = p->w_tau;
  sa.b_tau = p->b_tau;
  sa.c_tau = p->c_tau;
  set_summary(sa, &p->summary);
  sa.meta_fmt = p->summary.format;
  sa.seq_lens = p->cache.seq_lens;
  sa.tau_mode = p->tau_mode;
  sa.lwb = p->n_local_blocks;
  sa.screen_enabled = p->screen_enabled ? 1 : 0;
  sa.scale = p->scale;
  sa.offset_a = p->offset_a;
  sa.z = p->z;
  sa.s = s;
  sa.status = reinterpret_cast<unsigned*>(ws + w.status);
  sa.tau = reinterpret_cast<float*>(ws + w.tau);
  sa.chunk_count = reinterpret_cast<int*>(ws + w.chunk_count);
  sa.chunk_list = reinterpret_cast<int*>(ws + w.chunk_list);
  sa.out = p->out;
  sa.lse = p->lse;
  sa.head_count = reinterpret_cast<int*>(ws + w.head_count);
  sa.head_best = reinterpret_cast<unsigned long long*>(ws + w.head_best);

  if (s.fused) {
    FusedArgs fa;
    fa.trace = p->trace;
    fa.k = p->cache.k_cache;
    fa.v = p->cache.v_cache;
    fa.block_table = p->cache.block_table;
    fa.q = p->q;
    fa.seq_lens = p->cache.seq_lens;
    fa.w_tau = p->w_tau;
    fa.b_tau = p->b_tau;
    fa.c_tau = p->c_tau;
    fa.mu = p->summary.mu;
    fa.sigma = p->summary.sigma;
    fa.max_norm = p->summary.max_norm;
    fa.tau_mode = p->tau_mode;
    fa.lwb = p->n_local_blocks;
    fa.screen_enabled = p->screen_enabled ? 1 : 0;
    fa.scale = p->scale;
    fa.beta = p->beta;
    fa.offset_a = p->offset_a;
    fa.z = p->z;
    fa.s = s;
    fa.status = reinterpret_cast<unsigned*>(ws + w.status);
    fa.done_ctas = reinterpret_cast<unsigned*>(ws + w.ctrl) + 1;
    fa.arrived = reinterpret_cast<unsigned*>(ws + w.ctrl) + 2;
    fa.flags = reinterpret_cast<unsigned*>(ws + w.counters);
    fa.seg_ctr = reinterpret_cast<unsigned long long*>(ws + w.counters + kFusedSegCtrOffset * sizeof(unsigned));
    fa.tau = reinterpret_cast<float*>(ws + w.tau);
    fa.chunk_count = reinterpret_cast<int*>(ws + w.chunk_count);
    fa.chunk_list = reinterpret_cast<int*>(ws + w.chunk_list);
    fa.partials = reinterpret_cast<float*>(ws + w.partials);
    fa.out = p->out;
    fa.lse = p->lse;
    ev(0);
    ev(1);
    if (launch_fused_tc(fa, cs) != cudaSuccess) return ETA_ERR_CUDA;
    ev(2);
    if (p->admitted_count || p->union_count || p->union_list || p->union_mask) {
      ExportArgs xa;
      xa.trace = p->trace;
      xa.chunk_count = fa.chunk_count;
      xa.chunk_list = fa.chunk_list;
      xa.seq_lens = p->cache.seq_lens;
      xa.s = s;
      xa.admitted_count = p->admitted_count;
      xa.union_count = p->union_count;
      xa.union_list = p->union_list;
      xa.union_mask = p->union_mask;
      if (launch_export(xa, cs) != cudaSuccess) return ETA_ERR_CUDA;
    }
    ev(3);
    return ETA_OK;
  }

  ev(0);
  if (s.rescue) {
    if (cudaMemsetAsync(ws + w.head_count, 0, w.partials - w.head_count, cs) != cudaSuccess) return ETA_ERR_CUDA;
  }
  if (launch_screen(sa, cs) != cudaSuccess) return ETA_ERR_CUDA;
  if (s.rescue && launch_rescue(sa, cs) != cudaSuccess) return ETA_ERR_CUDA;

  AttendArgs aa;
  aa.trace = p->trace;
  aa.k = p->cache.k_cache;
  aa.block_table = p->cache.block_table;
  aa.v = p->cache.v_cache;
  aa.q = p->q;
  aa.seq_lens = p->cache.seq_lens;
  aa.tau = sa.tau;
  aa.chunk_count = sa.chunk_count;
  aa.chunk_list = sa.chunk_list;
  aa.scale = p->scale;
  aa.beta = p->beta;
  aa.s = s;
  aa.status = sa.status;
  aa.partials = reinterpret_cast<float*>(ws + w.partials);
  aa.out = p->out;
  aa.lse = p->lse;
  ev(1);
  const cudaError_t ea = s.attend_kind == ETA_ATTEND_TC ? launch_attend_tc(aa, cs) : launch_attend_simt(aa, cs);
  if (ea != cudaSuccess) return ETA_ERR_CUDA;

  ev(2);
  MergeArgs ma;
  ma.trace = p->trace;
  ma.chunk_count = sa.chunk_count;
  ma.partials = aa.partials;
  ma.s = s;
  ma.out = p->out;
  ma.lse = p->lse;
  if (launch_merge(ma, cs) != cudaSuccess) return ETA_ERR_CUDA;

  if (p->admitted_count || p->union_count || p->union_list || p->union_mask) {
    ExportArgs xa;
    xa.trace = p->trace;
    xa.chunk_count = sa.chunk_count;
    xa.chunk_list = sa.chunk_list;
    xa.seq_lens = p->cache.seq_lens;
    xa.s = s;
    xa.admitted_count = p->admitted_count;
    xa.union_count = p->union_count;
    xa.union_list = p->union_list;
    xa.union_mask = p->union_mask;
    if (launch_export(xa, cs) != cudaSuccess) return ETA_ERR_CUDA;
  }
  ev(3);
  return ETA_OK;
}

eta_status eta_prefill(const eta_prefill_params* p, void* stream) {
  if (!p) return ETA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 || p->seq_len < 1 || p->kv_stride < p->seq_len)
    return ETA_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return ETA_ERR_INVALID_ARG;
  if (p->dtype != ETA_BF16 && p->dtype != ETA_F32) return ETA_ERR_INVALID_ARG;
  if (p->dtype != ETA_BF16 || p->head_dim != 128) return ETA_ERR_UNSUPPORTED;
  if (p->batch > 65535 || p->n_q_heads > 65535) return ETA_ERR_UNSUPPORTED;
  if (static_cast<long long>(p->batch) * p->n_q_heads * p->seq_len >= (1ll << 31) ||
      static_cast<long long>(p->batch) * p->n_kv_heads * p->kv_stride >= (1ll << 31))
    return ETA_ERR_UNSUPPORTED;
  // one grid row per 128-query tile (the grid's y extent is at most 65535)
  constexpr int kPrefillMaxSeq = 65535 * 128;
  if (p->seq_len > kPrefillMaxSeq) return ETA_ERR_UNSUPPORTED;
  if (!p->q || !p->k || !p->v || !p->out) return ETA_ERR_INVALID_ARG;
  if (!aligned(p->q, 16) || !aligned(p->k, 16) || !aligned(p->v, 16) || !aligned(p->out, 16))
    return ETA_ERR_INVALID_ARG;
  if (p->tau_mode == ETA_TAU_LEARNED) {
    if (!p->w_tau || !p->b_tau || !aligned(p->w_tau, 16) || !aligned(p->b_tau, 4)) return ETA_ERR_INVALID_ARG;
  } else if (p->tau_mode == ETA_TAU_CALIBRATED) {
    if (!p->c_tau || !aligned(p->c_tau, 4)) return ETA_ERR_INVALID_ARG;
  } else {
    return ETA_ERR_INVALID_ARG;
  }
  if (!(p->scale > 0.f) || !isfinite(p->scale)) return ETA_ERR_INVALID_ARG;
  if (!(p->beta >= 0.f) || !isfinite(p->beta)) return ETA_ERR_INVALID_ARG;
  if (!isfinite(p->offset_a)) return ETA_ERR_INVALID_ARG;
  if ((p->lse && !aligned(p->lse, 4)) || (p->gate_sum && !aligned(p->gate_sum, 4))) return ETA_ERR_INVALID_ARG;
  if (!p->workspace || !aligned(p->workspace, 256) || p->workspace_bytes < ETA_PREFILL_WORKSPACE_BYTES)
    return ETA_ERR_WORKSPACE;
  PrefillArgs a;
  a.q = p->q;
  a.k = p->k;
  a.v = p->v;
  a.w_tau = p->w_tau;
  a.b_tau = p->b_tau;
  a.c_tau = p->c_tau;
  a.out = p->out;
  a.lse = p->lse;
  a.gate_sum = p->gate_sum;
  a.status = static_cast<unsigned*>(p->workspace);
  a.B = p->batch;
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.G = p->n_q_heads / p->n_kv_heads;
  a.T = p->seq_len;
  a.kv_stride = p->kv_stride;
  a.tau_mode = p->tau_mode;
  a.scale = p->scale;
  a.beta = p->beta;
  a.offset_a = p->offset_a;
  return launch_prefill_tc(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

eta_status eta_calibration_histogram(const eta_calib_params* p, void* stream) {
  if (!p) return ETA_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 || p->seq_len < 1 || p->kv_stride < p->seq_len)
    return ETA_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return ETA_ERR_INVALID_ARG;
  if (p->dtype != ETA_BF16 && p->dtype != ETA_F32) return ETA_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return ETA_ERR_UNSUPPORTED;
  if (p->batch > 65535 || p->n_q_heads > 65535) return ETA_ERR_UNSUPPORTED;
  if (!p->q || !p->k || !p->hist || !aligned(p->q, 4) || !aligned(p->k, 4) || !aligned(p->hist, 8))
    return ETA_ERR_INVALID_ARG;
  if (!(p->scale > 0.f) || !isfinite(p->scale) || !isfinite(p->lo) || !isfinite(p->hi) || !(p->hi > p->lo))
    return ETA_ERR_INVALID_ARG;
  if (p->nbins < 1 || p->nbins > 8192) return ETA_ERR_INVALID_ARG;
  CalibArgs a;
  a.q = p->q;
  a.k = p->k;
  a.hist = p->hist;
  a.B = p->batch;
  a.Hq = p->n_q_heads;
  a.Hkv = p->n_kv_heads;
  a.G = p->n_q_heads / p->n_kv_heads;
  a.T = p->seq_len;
  a.kv_stride = p->kv_stride;
  a.d = p->head_dim;
  a.elt = p->dtype == ETA_F32 ? 4 : 2;
  a.nbins = p->nbins;
  a.scale = p->scale;
  a.lo = p->lo;
  a.inv_width = static_cast<float>(p->nbins / (static_cast<double>(p->hi) - p->lo));
  return launch_calib(a, static_cast<cudaStream_t>(stream)) == cudaSuccess ? ETA_OK : ETA_ERR_CUDA;
}

eta_status eta_calibrate_constants(const double* hist, int n_heads, int nbins, float lo, float hi,
                                   const float* target, float* c) {
  if (!hist || !target || !c || n_heads < 1 || nbins < 1 || !(hi > lo)) return ETA_ERR_INVALID_ARG;
  const double width = (static_cast<double>(hi) - lo) / nbins;
  for (int h = 0; h < n_heads; ++h) {
    if (!(target[h] >= 0.f && target[h] <= 1.f)) return ETA_ERR_INVALID_ARG;
    const double* x = hist + static_cast<size_t>(h) * (nbins + 2);
    double total = 0.0;
    for (int b = 0; b < nbins + 2; ++b) total += x[b];
    const double need = target[h] * total;
    double acc = x[nbins + 1];  // logits >= hi
    double val = lo;
    if (acc >= need) {
      val = hi;
    } else {
      for (int b = nbins; b >= 1; --b) {  // slot b: [lo + (b - 1) width, lo + b width)
        if (acc + x[b] >= need) {
          val = lo + b * width - (need - acc) / x[b] * width;
          break;
        }
        acc += x[b];
      }
    }
    c[h] = static_cast<float>(val);
  }
  return ETA_OK;
}

eta_status eta_read_device_status(void* workspace, void* stream) {
  if (!workspace || !aligned(workspace, 256)) return ETA_ERR_INVALID_ARG;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  unsigned word = 0;
  if (cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, cs) != cudaSuccess) return ETA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return ETA_ERR_CUDA;
  const unsigned zero = 0;
  if (cudaMemcpyAsync(workspace, &zero, sizeof(zero), cudaMemcpyHostToDevice, cs) != cudaSuccess) return ETA_ERR_CUDA;
  if (cudaStreamSynchronize(cs) != cudaSuccess) return ETA_ERR_CUDA;
  if (word & kStatusTimeout) return ETA_ERR_DEVICE_TIMEOUT;
  if (word & kStatusList) return ETA_ERR_DEVICE_LIST;
  if (word & kStatusRange) return ETA_ERR_DEVICE_RANGE;
  return ETA_OK;
}

}  // extern "C"
