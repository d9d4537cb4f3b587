/*
 * eta.h - C ABI of the B200 (sm_100a) library for the decode step of
 * Elastic Threshold Attention (ETA).
 *
 * Source of the operations: "Elastic Threshold Attention: Learned Contextual
 * Sparsity for Long-Context Decoding"
 *   - query-conditioned threshold tau = w_tau . q + b_tau, or frozen per-head
 *     constants c (section 1; section 4.7; Appendix D.1, D.2)
 *   - effective threshold tau~ = tau - a and the tempered logit
 *     S~ = S * sigmoid(beta (S - tau~)), S = q k / sqrt(d) (Appendix G.1)
 *   - per-block metadata mu_B (fp16), sigma_B (fp16), M_B (fp32) per KV head
 *     (Appendix F.1; section 3.2)
 *   - O(1) block screen, GQA union loading with per-head masking (section 3.1,
 *     section 4.3 "Dual Bound", Appendix F.1)
 *   - split-KV chunks merged by an associative online-softmax reduction,
 *     top-1 rescue, predicated tail block (section 3.2; Appendix F.3, F.4)
 *   - always-loaded window: lwb = 2 blocks plus the tail block (section 4.8)
 *
 * Conventions shared by every entry point:
 *   - Every pointer inside a descriptor is DEVICE memory of the current CUDA
 *     device, borrowed (never freed or retained by the library), and 16-byte
 *     aligned unless said otherwise.  Descriptors themselves are host memory
 *     read during the call only.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls are
 *     asynchronous and stream-ordered; none synchronises the host except
 *     eta_read_device_status.
 *   - The library never allocates or frees device memory.  Scratch memory is
 *     the caller's `workspace`, sized by eta_decode_workspace_size.
 *   - Arguments are validated on the host before any launch; a failed
 *     validation returns an error code and launches nothing.  Values that
 *     live in device memory (seq_lens, first_token) are checked by the
 *     kernels: an out-of-range value is clamped and recorded in the device
 *     status word, read back with eta_read_device_status.
 *   - Layouts (row-major, contiguous):
 *       K, V cache   [batch, n_kv_heads, max_ctx, head_dim]   kv_dtype
 *       q, out       [batch, n_q_heads, head_dim]             kv_dtype
 *       mu, sigma    [batch, n_kv_heads, nb_max, head_dim]     fp16
 *       max_norm     [batch, n_kv_heads, nb_max]               fp32
 *     with nb_max = ceil(max_ctx / block_size).  Query head h reads KV head
 *     h / (n_q_heads / n_kv_heads).
 *   - Supported: head_dim in {64, 128}; block_size in {16, 32, 64, 128};
 *     group size n_q_heads / n_kv_heads in {1, 2, 4, 8}.
 */
#ifndef ETA_H
#define ETA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ETA_OK = 0,
  ETA_ERR_INVALID_ARG = 1,     /* bad pointer, size, alignment or value     */
  ETA_ERR_UNSUPPORTED = 2,     /* valid but not implemented (e.g. d = 96)   */
  ETA_ERR_WORKSPACE = 3,       /* workspace NULL or smaller than required   */
  ETA_ERR_CUDA = 4,            /* a CUDA runtime call failed                */
  ETA_ERR_DEVICE_TIMEOUT = 5,  /* a bounded device-side wait ran out        */
  ETA_ERR_DEVICE_RANGE = 6,    /* a device-resident length was out of range */
  ETA_ERR_DEVICE_LIST = 7      /* the admitted-block tables an attention
                                  kernel read broke the screen's contract
                                  (counts, block range, order, head masks);
                                  the step's output is not valid          */
} eta_status;

typedef enum { ETA_F32 = 0, ETA_BF16 = 1 } eta_dtype;
typedef enum { ETA_TAU_LEARNED = 0, ETA_TAU_CALIBRATED = 1 } eta_tau_mode;

/* Attention-kernel choice (eta_decode_params.attend_impl). */
typedef enum {
  ETA_ATTEND_AUTO = 0,   /* tensor-core kernel where supported, else CUDA-core */
  ETA_ATTEND_SIMT = 1,   /* CUDA-core FMA kernel (all supported shapes)       */
  ETA_ATTEND_TC = 2,     /* tcgen05 tensor-core kernel (bf16, d = 128,
                            block_size in {64, 128}, group size >= 2) between
                            a separate screen kernel and a merge kernel       */
  ETA_ATTEND_FUSED = 3   /* one tcgen05 kernel that screens, attends and
                            merges (the tensor-core shapes above, fp16
                            metadata or the screen off, n_local_blocks >= 0,
                            batch <= 256, at most 2048 (sequence, KV head)
                            segments)                                         */
} eta_attend_impl;

/* The KV cache of one attention layer.  Two layouts:
 *   contiguous (block_table == NULL): k_cache, v_cache are
 *       [batch, n_kv_heads, max_ctx, head_dim];
 *   paged (block_table != NULL): k_cache, v_cache are pools of pages
 *       [num_pages, n_kv_heads, block_size, head_dim], one page per KV block,
 *       and block_table [batch, nb_max] (int32, device) gives the page of
 *       logical block j of sequence i (only blocks below ceil(seq_len / b)
 *       are read; a page id outside [0, num_pages) is replaced by page 0 and
 *       reported as ETA_ERR_DEVICE_RANGE).  Block metadata stays indexed by
 *       logical block.
 * A zero-initialised tail (block_table, num_pages) is the contiguous layout. */
typedef struct {
  int batch;          /* >= 1                                                */
  int n_q_heads;      /* multiple of n_kv_heads                              */
  int n_kv_heads;     /* >= 1                                                */
  int head_dim;       /* 64 or 128                                           */
  int block_size;     /* tokens per KV block b                               */
  int max_ctx;        /* token capacity per (sequence, KV head), >= 1        */
  eta_dtype kv_dtype; /* dtype of K, V, q and out                            */
  const void* k_cache;
  const void* v_cache;
  const int* seq_lens; /* [batch] device, 0 <= seq_lens[i] <= max_ctx         */
  const int* block_table; /* paged layout: [batch, nb_max] device, else NULL */
  int num_pages;          /* paged layout: pages in k_cache / v_cache, >= 1  */
} eta_cache_desc;

/* Storage of the centroid and spread in eta_summary_desc. */
typedef enum {
  ETA_META_FP16 = 0,  /* fp16 values (Appendix F.1)                            */
  ETA_META_FP8 = 1,   /* e4m3 codes with one fp32 scale per block and field:
                         value = code * scale, the scale mapping the block's
                         largest magnitude to 448 (FP8 metadata, named as a
                         systems extension in section 5; format is this
                         library's choice)                                    */
  ETA_META_BOX = 2    /* the comparison screen of section 4.3 (Quest): mu
                         holds the per-coordinate minimum and sigma the
                         maximum of the block's keys (fp16, rounded outward);
                         Score = scale sum_i max(q_i min_i, q_i max_i), a
                         strict bound; max_norm is not used                   */
} eta_meta_format;

/* Per-block, per-KV-head metadata (Appendix F.1): centroid mu_B, coordinate
 * standard deviation sigma_B, maximum norm M_B (fp32) of the block's keys
 * around the stored (dequantised) centroid, rounded up so that the geometric
 * bound <q, mu_B> + ||q|| M_B never under-estimates a key's logit.  A
 * zero-initialised descriptor with mu, sigma and max_norm set is the fp16
 * format. */
typedef struct {
  void* mu;        /* [batch, n_kv_heads, nb_max, head_dim]: fp16 values, or
                      e4m3 codes (one byte each) in the fp8 format           */
  void* sigma;     /* same layout and type as mu                             */
  float* max_norm; /* fp32 [batch, n_kv_heads, nb_max] (4-byte aligned)      */
  int format;      /* eta_meta_format                                        */
  float* mu_scale;    /* fp32 [batch, n_kv_heads, nb_max] (fp8 format only)  */
  float* sigma_scale; /* fp32 [batch, n_kv_heads, nb_max] (fp8 format only)  */
} eta_summary_desc;

/*
 * eta_block_summary_update - refresh the metadata of the blocks touched by a
 * KV append ("metadata ... refreshed on KV append"; Appendix F.1).
 *
 * For every sequence i, recomputes the blocks j with
 *   first_token[i] / block_size <= j < ceil(seq_lens[i] / block_size),
 * at most `max_blocks` of them per sequence (pass 1 for a one-token append,
 * nb_max to rebuild everything).  A partial tail block is summarised over its
 * present tokens only.  Other blocks are left untouched.
 *   first_token : [batch] device int, lowest position written since the last
 *                 update (4-byte aligned).
 * Errors: ETA_ERR_INVALID_ARG for NULL/misaligned pointers or bad sizes,
 * ETA_ERR_UNSUPPORTED for an unsupported head_dim/block_size,
 * ETA_ERR_CUDA if the launch fails.
 */
eta_status eta_block_summary_update(const eta_cache_desc* cache,
                                    const eta_summary_desc* summary,
                                    const int* first_token, int max_blocks,
                                    void* stream);

/*
 * eta_append_kv - the KV append of one decode step, fused with the metadata
 * refresh it requires ("refreshed on KV append"; Appendix F.1): for every
 * sequence i and KV head g, writes k_new[i, g, :] and v_new[i, g, :] into
 * row pos[i] of the caches and recomputes the summary of the block holding
 * that row over its present tokens [j b, seq_lens[i]) (seq_lens must already
 * count the new token).  One launch.
 *   k_new, v_new : [batch, n_kv_heads, head_dim] device, kv_dtype, 16-byte aligned
 *   pos          : [batch] device int, 4-byte aligned; a position outside
 *                  [0, max_ctx) writes nothing for that sequence
 * The cache descriptor's k_cache / v_cache are written (they must be
 * writable device memory).
 * Errors: ETA_ERR_INVALID_ARG, ETA_ERR_UNSUPPORTED, ETA_ERR_CUDA.
 */
eta_status eta_append_kv(const eta_cache_desc* cache, const eta_summary_desc* summary,
                         const void* k_new, const void* v_new, const int* pos,
                         void* stream);

/* All inputs and outputs of one decode step. */
typedef struct {
  eta_cache_desc cache;
  eta_summary_desc summary;          /* must be current for seq_lens         */
  const void* q;                     /* [batch, n_q_heads, head_dim]         */
  eta_tau_mode tau_mode;
  const float* w_tau;                /* [n_q_heads, head_dim] (learned)      */
  const float* b_tau;                /* [n_q_heads]           (learned)      */
  const float* c_tau;                /* [n_q_heads]           (calibrated)   */
  float scale;                       /* logit scale, usually 1/sqrt(d), > 0  */
  float beta;                        /* gate sharpness, > 0 (5 = terminal)   */
  float offset_a;                    /* tau~ = tau - a                       */
  float z;                           /* probabilistic half's z (> 0);
                                        INFINITY = strict geometric screen   */
  int n_local_blocks;                /* lwb >= 0: the tail block and the lwb
                                        blocks before it are always loaded;
                                        -1: none is, every block is screened  */
  int screen_enabled;                /* 0: every block is loaded (dense path) */
  int attend_impl;                   /* eta_attend_impl                      */
  void* out;                         /* [batch, n_q_heads, head_dim] written */
  float* lse;                        /* [batch, n_q_heads] or NULL: log-sum-
                                        exp of the tempered logits (-inf for
                                        an empty sequence)                   */
  /* Optional selection outputs (NULL to skip; all int32/uint32, 4-aligned): */
  int* admitted_count;               /* [batch, n_q_heads] blocks per head   */
  int* union_count;                  /* [batch, n_kv_heads] union blocks     */
  int* union_list;                   /* [batch, n_kv_heads, nb_max]: union
                                        block ids ascending, then -1 fill    */
  unsigned* union_mask;              /* [batch, n_kv_heads, nb_max]: bit j set
                                        if query head g*G + j admitted block
                                        union_list[...]; 0 fill              */
  void* workspace;                   /* device scratch, 256-byte aligned; its
                                        first ETA_WORKSPACE_CONTROL_BYTES must
                                        be zero before its first use        */
  size_t workspace_bytes;
  void* timing_events[4];            /* optional cudaEvent_t (NULL = none):
                                        recorded before the screen, before
                                        the attention kernel, before the
                                        merge and after the last kernel
                                        (events between the kernels keep
                                        them from overlapping their launch) */
  unsigned long long* trace;         /* optional device array of
                                        ETA_TRACE_SLOTS words (NULL = off),
                                        zeroed by the caller before the step:
                                        see ETA_TRACE_* below               */
} eta_decode_params;

/*
 * Step trace.  With eta_decode_params.trace set, the kernels of a step
 * record device times (the GPU's global nanosecond timer) into the array:
 * every slot is updated with an atomic maximum, so it must be zero before
 * the step.  A "first" slot holds the bitwise complement of the earliest
 * time (first CTA), a "last" slot the latest time (last CTA); a slot no
 * kernel wrote stays 0.  A kernel starts when its first CTA has passed its
 * wait for the previous kernel.  Costs two atomics per CTA when on; nothing
 * when off.  No counterpart in the paper: a measurement aid.
 */
#define ETA_TRACE_SLOTS 24
#define ETA_TRACE_SCREEN_FIRST 0   /* ~ start of the screen kernel          */
#define ETA_TRACE_SCREEN_LAST 1    /* end of the screen kernel              */
#define ETA_TRACE_ATTEND_FIRST 2   /* ~ start of the attention kernel       */
#define ETA_TRACE_ATTEND_LAST 3    /* end of the attention kernel           */
#define ETA_TRACE_TILE_FIRST 4     /* ~ first K/V tile in shared memory (tensor-core kernels) */
#define ETA_TRACE_MERGE_FIRST 6    /* ~ start of the merge kernel           */
#define ETA_TRACE_MERGE_LAST 7     /* end of the merge kernel               */
#define ETA_TRACE_FUSED_FIRST 8    /* ~ start of the single-launch kernel   */
#define ETA_TRACE_FUSED_LAST 9     /* end of the single-launch kernel       */
#define ETA_TRACE_EXPORT_FIRST 10  /* ~ start of the selection export       */
#define ETA_TRACE_EXPORT_LAST 11   /* end of the selection export           */
/* a recorded serving step (eta_step_graph_create) also records:            */
#define ETA_TRACE_APPEND_FIRST 12  /* ~ start of the append                 */
#define ETA_TRACE_APPEND_LAST 13   /* end of the append                     */
#define ETA_TRACE_IN_FIRST 14      /* ~ start of the input copy (kernel path) */
#define ETA_TRACE_IN_LAST 15       /* end of the input copy                 */
#define ETA_TRACE_OUT_FIRST 16     /* ~ start of the output copy (kernel path) */
#define ETA_TRACE_OUT_LAST 17      /* end of the output copy                */

/*
 * Leading control region of a decode workspace: the device status word and
 * the counters of the fused kernel (finished CTAs, published slice totals
 * and their arrival count, per-segment piece counters of the merge).
 * It must be zero before the workspace's first use; every completed step
 * leaves it at zero again (apart from the status word, which
 * eta_read_device_status clears), so one workspace serves calls of any shapes
 * in turn.  After a step that reported ETA_ERR_DEVICE_TIMEOUT, zero it again
 * before the next call.  The rest of the workspace needs no initialisation.
 */
#define ETA_WORKSPACE_CONTROL_BYTES ((size_t)69632)

/*
 * eta_decode_workspace_size - bytes of workspace eta_decode needs for these
 * shapes (host-only, launches nothing).  Depends on the cache shape, the
 * attention-kernel choice and the current device's SM count.
 * Errors: ETA_ERR_INVALID_ARG / ETA_ERR_UNSUPPORTED as eta_decode.
 */
eta_status eta_decode_workspace_size(const eta_decode_params* p, size_t* bytes);

/*
 * eta_decode - one ETA decode step for every (sequence, query head):
 *   1. tau~ per head (projection or constant, minus a);
 *   2. every screenable block scored against tau~; admitted set per head =
 *      screened blocks with Score >= tau~ plus the always-loaded window; a
 *      head left with no block admits its highest-scoring block (top-1
 *      rescue, lowest index on ties); the GQA union of a KV head's admitted
 *      sets is the load set;
 *   3. only the union's K/V blocks are read; each query head attends over the
 *      tokens (< seq_len) of its own admitted blocks with
 *      S~ = S sigmoid(beta (S - tau~)), weights exp(S~);
 *   4. split partials merged: out = sum e^{S~} v / sum e^{S~}, lse.
 * Outputs are written in kv_dtype (round-to-nearest-even for bf16).
 * Errors: ETA_ERR_INVALID_ARG, ETA_ERR_UNSUPPORTED, ETA_ERR_WORKSPACE,
 * ETA_ERR_CUDA (launch failure).  Device-side problems (a bounded wait that
 * ran out, a seq_len outside [0, max_ctx]) are reported by
 * eta_read_device_status.
 */
eta_status eta_decode(const eta_decode_params* p, void* stream);

/* Size of the fixed device scratch used by eta_decode_noalloc (8 MiB). */
#define ETA_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

/* Bits of the device status word (eta_decode_noalloc's device_status). */
#define ETA_DEVICE_STATUS_TIMEOUT 1u  /* a bounded device-side wait ran out  */
#define ETA_DEVICE_STATUS_RANGE 2u    /* a device-resident length or page id
                                         was out of range and was clamped    */
#define ETA_DEVICE_STATUS_LIST 4u     /* an attention kernel found the chunk
                                         counts or lists inconsistent and
                                         stopped (see ETA_ERR_DEVICE_LIST)   */

/*
 * eta_decode_noalloc - eta_decode for callers that cannot allocate device
 * memory.  No counterpart in the paper: this is a deployment variant.
 *
 * eta_decode needs a workspace from the caller.  Some callers cannot provide
 * one: a plugin running inside a host program that owns every device
 * allocation, or a code path where a cudaMalloc would synchronise the whole
 * device.  This entry point takes the same parameters, ignores
 * p->workspace and p->workspace_bytes, and uses a fixed array of
 * ETA_NOALLOC_SCRATCH_BYTES that the library declares in device memory
 * (every GPU that loads the library holds it until the process exits).  It
 * calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Every call looks up the array's device address in the current
 *     device's context (with that device current).  The first call on a
 *     device may load the library's device code; make it before any stream
 *     capture.
 *   - Every call shares the one array, which keeps the last call's contents.
 *     Calls that overlap on the GPU (different streams, or different host
 *     threads without ordering) race on it and give wrong results.
 *   - The step's device status word lives in that array and is cleared at
 *     the start of every call.  device_status, when not NULL, is a 4-byte
 *     aligned word in device memory that receives it after the step (stream-
 *     ordered): 0, or ETA_DEVICE_STATUS_* bits.  Without it, device-side
 *     problems (a bounded wait that ran out, a seq_len outside [0, max_ctx]
 *     that was clamped, a page id outside the pool) go unreported.
 * Errors: as eta_decode, plus ETA_ERR_WORKSPACE when
 * eta_decode_workspace_size(p) exceeds ETA_NOALLOC_SCRATCH_BYTES,
 * ETA_ERR_INVALID_ARG for a misaligned device_status, and ETA_ERR_CUDA if the
 * array's address cannot be obtained or the status copy fails.
 */
eta_status eta_decode_noalloc(const eta_decode_params* p, unsigned* device_status, void* stream);

/*
 * eta_decode_graph_* - one decode step captured once into a CUDA graph and
 * replayed.  No counterpart in the paper: a launch-path variant of eta_decode
 * for serving loops that run the same step shape every token.
 *
 * eta_decode_graph_create validates p exactly as eta_decode does, then
 * records eta_decode(p) on a private stream under stream capture
 * (thread-local mode) and instantiates the graph; nothing runs on the GPU.
 * On success *out receives a handle the caller owns and must release with
 * eta_decode_graph_destroy; on failure *out is NULL and nothing is kept.
 * The graph holds the addresses and scalars of p as they were at creation:
 *   - every buffer p names (q, caches, seq_lens, summary, tau parameters,
 *     out, lse, selection outputs, workspace) must stay allocated at the
 *     same address for the graph's lifetime; their CONTENTS may change
 *     between launches (a new query, appended tokens, new seq_lens within
 *     [0, max_ctx]): each launch reads them afresh on the device;
 *   - shapes, tau mode, scale, beta, offset_a, z, n_local_blocks and the
 *     attention kernel choice are fixed; a new value needs a new graph;
 *   - timing_events must all be NULL (ETA_ERR_INVALID_ARG otherwise).
 * eta_decode_graph_launch enqueues one step on `stream` (stream-ordered and
 * asynchronous like eta_decode).  Launches of one graph must not overlap on
 * the GPU (they share its workspace).  Device-side problems are reported by
 * eta_read_device_status on the workspace, as for eta_decode.
 * Errors: as eta_decode for create (and ETA_ERR_CUDA if capture or
 * instantiation fails); ETA_ERR_INVALID_ARG for a NULL handle;
 * ETA_ERR_CUDA if the graph launch fails.
 */
typedef struct eta_decode_graph eta_decode_graph;
eta_status eta_decode_graph_create(const eta_decode_params* p, eta_decode_graph** out);
eta_status eta_decode_graph_launch(const eta_decode_graph* g, void* stream);
eta_status eta_decode_graph_destroy(eta_decode_graph* g);

/*
 * eta_step_graph_create - one token of a serving loop recorded into a CUDA
 * graph: an optional host-to-device copy of the token's inputs, an optional
 * KV append (eta_append_kv on the decode step's cache and summary), the
 * decode step, an optional device-to-host copy of its output, in that order.
 * No counterpart in the paper: a launch-path variant for serving loops.
 *   decode      : the decode step, as for eta_decode_graph_create (required)
 *   k_new, v_new, positions : as eta_append_kv's arguments; all three NULL =
 *                 no append, all three set = append (anything else is
 *                 ETA_ERR_INVALID_ARG); k_new and v_new may be page-locked
 *                 host memory mapped into the device's address space (the
 *                 append kernel reads them there)
 *   q_new       : optional, [batch, n_q_heads, head_dim] kv_dtype, 16-byte
 *                 aligned, device or mapped page-locked host memory: the
 *                 token's queries, copied into decode->q by the append launch
 *                 (so decode->q is written; requires the append)
 *   h2d_src -> h2d_dst, h2d_bytes : copied first; h2d_src must be page-locked
 *                 host memory (recording fails with ETA_ERR_CUDA otherwise),
 *                 h2d_dst device memory; h2d_bytes 0 = no copy
 *   d2h_src -> d2h_dst, d2h_bytes : copied last; d2h_dst page-locked host
 *                 memory; d2h_bytes 0 = no copy
 * When the host end of a copy is mapped into the device's address space
 * (page-locked memory under unified addressing) and the other end is device
 * memory, the copy is a small kernel that reads or writes the host buffer
 * directly; otherwise it is a copy-engine transfer.  The cheapest token
 * needs neither copy: q_new, k_new, v_new in mapped host memory and
 * decode->out pointing at mapped host memory (the decode kernels store the
 * output there directly; pass the device view of the buffer, which under
 * unified addressing is the host pointer of cudaHostAlloc memory).
 * The handle is launched and released with eta_decode_graph_launch /
 * eta_decode_graph_destroy, under the same rules (addresses and scalars
 * fixed at creation, contents read at every launch).
 * Errors: as eta_decode_graph_create and eta_append_kv; ETA_ERR_INVALID_ARG
 * for a NULL pointer with a non-zero copy size.
 */
typedef struct {
  const eta_decode_params* decode;
  const void* k_new;
  const void* v_new;
  const int* positions;
  const void* q_new;
  const void* h2d_src;
  void* h2d_dst;
  size_t h2d_bytes;
  const void* d2h_src;
  void* d2h_dst;
  size_t d2h_bytes;
} eta_step_desc;

eta_status eta_step_graph_create(const eta_step_desc* d, eta_decode_graph** out);

/*
 * ------------------------------------------------------------------------
 * Causal forward pass over whole sequences (prefill / training forward).
 *
 * Source: Elastic Threshold Attention, section 2.3 (fused training kernel:
 * no T x T matrix in HBM), Appendix E.1 (query tiles with their own
 * thresholds, causal inner loop over key tiles), Appendix E.3 (inclusion
 * probability sigma_ij = sigmoid(beta (S_ij - tau~_i)), multiplicative mask
 * S~ = S sigma, row sum R_i = sum_j sigma_ij), Appendix E.4 (O, the
 * log-sum-exp and the row vector kept for the backward pass).
 *
 * For every sequence b, query head h (KV head h / G, G = n_q_heads /
 * n_kv_heads) and query row i < seq_len:
 *   tau~_i  = w_tau[h] . q_i + b_tau[h] - a  (learned) or c_tau[h] - a,
 *   S_ij    = scale q_i . k_j  for the keys j <= i,
 *   out_i   = sum_j e^{S~_ij} v_j / sum_j e^{S~_ij},
 *   lse_i   = ln sum_j e^{S~_ij},   gate_sum_i = sum_j sigma_ij.
 * Layouts (row-major): q, out [batch, n_q_heads, seq_len, head_dim];
 * k, v [batch, n_kv_heads, kv_stride, head_dim] (a KV cache with
 * max_ctx = kv_stride; rows >= seq_len of a head are never used);
 * lse, gate_sum [batch, n_q_heads, seq_len] fp32.
 * Supported: bf16, head_dim = 128, any group size, 1 <= seq_len <= kv_stride,
 * seq_len <= 65535 * 128 (8388480), batch * n_q_heads * seq_len and
 * batch * n_kv_heads * kv_stride < 2^31.
 * ------------------------------------------------------------------------
 */
typedef struct {
  int batch, n_q_heads, n_kv_heads, head_dim;
  int seq_len;                       /* tokens per sequence (queries = keys) */
  int kv_stride;                     /* rows per KV head in k and v, >= seq_len */
  eta_dtype dtype;                   /* ETA_BF16                              */
  const void* q;                     /* [batch, n_q_heads, seq_len, d]        */
  const void* k;                     /* [batch, n_kv_heads, kv_stride, d]     */
  const void* v;                     /* same layout as k                      */
  eta_tau_mode tau_mode;
  const float* w_tau;                /* [n_q_heads, d] (learned), 16-aligned  */
  const float* b_tau;                /* [n_q_heads]    (learned)              */
  const float* c_tau;                /* [n_q_heads]    (calibrated)           */
  float scale;                       /* > 0, usually 1/sqrt(d)                */
  float beta;                        /* >= 0 (0: sigma = 1/2 everywhere)      */
  float offset_a;                    /* tau~ = tau - a                        */
  void* out;                         /* [batch, n_q_heads, seq_len, d] bf16   */
  float* lse;                        /* or NULL                               */
  float* gate_sum;                   /* or NULL                               */
  void* workspace;                   /* >= ETA_PREFILL_WORKSPACE_BYTES, 256-
                                        aligned: holds the device status word
                                        read by eta_read_device_status        */
  size_t workspace_bytes;
} eta_prefill_params;

#define ETA_PREFILL_WORKSPACE_BYTES ((size_t)256)

/*
 * eta_prefill - the causal forward pass above, one launch.
 * Errors: ETA_ERR_INVALID_ARG (NULL or misaligned pointer, bad size or
 * value), ETA_ERR_UNSUPPORTED (dtype, head_dim, sizes past the limits),
 * ETA_ERR_WORKSPACE, ETA_ERR_CUDA (launch failure).  A bounded device-side
 * wait that ran out is reported by eta_read_device_status.
 */
eta_status eta_prefill(const eta_prefill_params* p, void* stream);

/*
 * ------------------------------------------------------------------------
 * Offline per-head threshold calibration (section 4.7; Appendix D.2):
 * frozen constants that replace the threshold projection for a stationary
 * deployment.  Every causal logit S_tj = scale q_t . k_j (j <= t) of a
 * query head enters a histogram with weight 1/(t + 1), so each query row
 * weighs 1; the constant of a head is the logit at which the weighted
 * fraction of logits at or above it equals the head's target density
 * (a token-level density; the block screen admits somewhat more).  The value
 * returned is the effective threshold tau~: use c_tau = value + offset_a.
 * ------------------------------------------------------------------------
 */
typedef struct {
  int batch, n_q_heads, n_kv_heads, head_dim;
  int seq_len;                       /* calibration tokens per sequence      */
  int kv_stride;                     /* rows per KV head in k, >= seq_len    */
  eta_dtype dtype;                   /* ETA_F32 or ETA_BF16                  */
  const void* q;                     /* [batch, n_q_heads, seq_len, d]: the
                                        query of every position              */
  const void* k;                     /* [batch, n_kv_heads, kv_stride, d]    */
  float scale;                       /* > 0                                   */
  float lo, hi;                      /* histogram range of the logits, lo<hi */
  int nbins;                         /* 1 <= nbins <= 8192                    */
  double* hist;                      /* device [n_q_heads, nbins + 2],
                                        8-aligned: slot 0 counts logits < lo,
                                        slots 1..nbins the equal bins,
                                        slot nbins+1 logits >= hi.  The call
                                        ADDS to it (zero it once, then call
                                        per calibration batch)              */
} eta_calib_params;

/* eta_calibration_histogram - accumulate the weighted logit histogram of
 * every query head over the batch (one launch, stream-ordered).
 * Errors: ETA_ERR_INVALID_ARG, ETA_ERR_UNSUPPORTED (head_dim not 64/128),
 * ETA_ERR_CUDA. */
eta_status eta_calibration_histogram(const eta_calib_params* p, void* stream);

/* eta_calibrate_constants - host-only solver: for each head h, the logit at
 * which the weighted fraction at or above it reaches target[h] (searching
 * the bins from the top, linear inside the crossing bin; error at most one
 * bin width).  hist, target and c are HOST arrays ([n_heads][nbins + 2],
 * [n_heads], [n_heads]).  Errors: ETA_ERR_INVALID_ARG. */
eta_status eta_calibrate_constants(const double* hist, int n_heads, int nbins, float lo, float hi,
                                   const float* target, float* c);

/*
 * eta_read_device_status - synchronise `stream`, read and clear the device
 * status word kept in `workspace`.  Returns ETA_OK, ETA_ERR_DEVICE_TIMEOUT,
 * ETA_ERR_DEVICE_LIST or ETA_ERR_DEVICE_RANGE, in that order of precedence
 * when several bits are set (or ETA_ERR_CUDA if the copy fails).
 */
eta_status eta_read_device_status(void* workspace, void* stream);

/*
 * eta_diag_wait_timeout - diagnostic: one warp waits, with the same bounded
 * wait the kernels use, on a shared-memory mbarrier that nothing completes;
 * after the wait's cycle limit (about one second) it gives up and sets the
 * timeout bit of the status word at the start of `workspace`.  A following
 * eta_read_device_status(workspace) then returns ETA_ERR_DEVICE_TIMEOUT and
 * the context stays usable.  It checks the failure-reporting path end to end
 * without a fault or a hang.  No counterpart in the paper.
 *   workspace : device memory, 256-byte aligned, at least 4 bytes (a decode
 *               workspace serves)
 * Errors: ETA_ERR_INVALID_ARG (NULL or misaligned), ETA_ERR_CUDA (launch).
 */
eta_status eta_diag_wait_timeout(void* workspace, void* stream);

/* Static description of a status code. */
const char* eta_status_string(eta_status s);

/* Library build description (kernels compiled, architecture). */
const char* eta_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* ETA_H */
