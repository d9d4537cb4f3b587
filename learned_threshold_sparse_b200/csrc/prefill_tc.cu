// Causal ETA forward pass over whole sequences (prefill / training forward)
// on the 5th-generation tensor cores, bf16 Q/K/V, d = 128.
//
// Source: Elastic Threshold Attention,
//   section 2.3          fused kernel: no T x T matrix in HBM,
//   Appendix E.1         query tiles with their own thresholds; the inner
//                        loop runs causally over key tiles,
//   Appendix E.3         sigma_ij = sigmoid(beta (S_ij - tau~_i)),
//                        S~ = S sigma (multiplicative mask), R_i = sum_j sigma_ij,
//   Appendix E.4         O, the log-sum-exp L and the row vector kept for the
//                        backward pass,
//   Appendix G.1         tau~ = tau - a, tau = w_tau . q + b_tau or a constant.
//
// One CTA per (128 query rows, query head, sequence); heavy (late) query tiles
// of all heads and sequences are dispatched first.  Per key tile j of 128 keys:
//   S [128 q x 128 k]  = Q . K_j^T   (M = 128, N = 128; Q, K from shared memory)
//   O_h [128 q x 128 d] += P_j,h . V_j,h   (h = 0, 1: keys 0-63 / 64-127 of
//                                          the tile; A = P from tensor
//                                          memory, B = V MN-major)
// Tensor memory: S double-buffered in columns 0-127 / 128-255, O_0 in
// 256-383, O_1 in 384-511.  P_j,h (bf16, two per column) overwrites the S_j
// columns it was computed from, so tile j + 2's S (issued after P_j . V_j by
// the same thread, and the MMAs run in issue order) never races it.
//
// Roles: warp 0 issues the tensor copies (Q once; K and V tiles into two
// 2-stage rings with their own barriers, so K_{j+2} is copied as soon as
// Q K_j^T is done, not after P_j V_j); warp 1 owns tensor memory and issues
// the MMAs; warps 2-9 run the
// softmax, two warps per query-row quarter (tensor-memory lane quarter),
// each on one half h of the key columns with its own running max, sum and
// accumulator O_h (two split-KV partials of the row, merged once at the end
// by the associative combine), so the halves never wait on each other.  The
// running max moves lazily: O_h is rescaled in tensor memory only when a
// row's max grows by more than 2^8, so the weights stay <= 2^8.  Off the
// diagonal the softmax runs on column pairs with the packed fp32x2 forms,
// and 3/8 of the weights' 2^x are computed on the FMA pipes (the gate's tanh
// and the weight's 2^x otherwise both occupy the special-function unit).
#include <math.h>
#include <string.h>

#include "attend_common.cuh"
#include "tc_common.cuh"

namespace eta {
namespace {

using namespace tc;
using dev::wait_or_abort;
using dev::warp_wait_or_abort;

constexpr int D = 128;
constexpr int BM = 128;  // query rows per CTA
constexpr int BN = 128;  // keys per tile
constexpr int kSoftWarps = 8;
constexpr int kWarps = 2 + kSoftWarps;
constexpr int kThreads = kWarps * 32;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;  // S0 0..127, S1 128..255, O_0 256..383, O_1 384..511
constexpr uint32_t kOCol = 256;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLazy = 8.0f;  // rescale O only when the max grows by more than this (base 2)

constexpr uint32_t PANEL = BM * 128;  // one 64-column panel of 128 rows (16 KB)
constexpr uint32_t TILE = 2 * PANEL;  // 128 rows x 128 bf16 (32 KB)
constexpr uint32_t OFF_Q = 0;
constexpr uint32_t OFF_STAGE = TILE;  // stage s: K at OFF_STAGE + 2 s TILE, V after it
constexpr uint32_t OFF_RED = OFF_STAGE + kStages * 2 * TILE;  // [m, l, R][2 halves][128] float
constexpr uint32_t OFF_BARS = OFF_RED + 3 * 2 * BM * 4;
constexpr uint32_t kSmemBytes = OFF_BARS + 256 + 1024;  // barriers, flags, alignment slack

__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Two floats to a bf16 pair (lo in the low half), round to nearest even.
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_lo_f(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi_f(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// ETA_EXP2_BEGIN
// Packed pairs of fp32 operations (one instruction for two columns on the
// device): a b + c, a b, a + b, each element rounded exactly as its scalar
// form (the host forms are those scalar forms).
__host__ __device__ inline float2 ffma2(float2 a, float2 b, float2 c) {
#ifdef __CUDA_ARCH__
  float2 d;
  asm("{.reg .b64 ra, rb, rc, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
#else
  return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
}
__host__ __device__ inline float2 fmul2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
#else
  return make_float2(a.x * b.x, a.y * b.y);
#endif
}
__host__ __device__ inline float2 fadd2(float2 a, float2 b) {
#ifdef __CUDA_ARCH__
  float2 d;
  asm("{.reg .b64 ra, rb, rd;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
#else
  return make_float2(a.x + b.x, a.y + b.y);
#endif
}

__host__ __device__ inline uint32_t bits_of(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(x);
#else
  uint32_t u;
  memcpy(&u, &x, 4);
  return u;
#endif
}
__host__ __device__ inline float float_of(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float x;
  memcpy(&x, &u, 4);
  return x;
#endif
}

// 2^y for a pair on the FMA pipes, to take part of the weights off the
// special-function unit.  Cody-Waite style reduction: y = n + f with
// n = rint(y) (adding 1.5 2^23 leaves n in the low mantissa bits) and f in
// [-1/2, 1/2]; 2^f by the cubic of least maximum relative error on that
// interval (Remez exchange; 7.5e-5), and n added to its exponent field.  y is
// clamped at -126 first, so the result stays near 2^-126 or above (where the
// special-function form flushes its results below 2^-126 to 0); the clamp
// also maps a NaN y (a NaN key inside the sequence) to 2^-126, where the
// special-function form gives NaN.
__host__ __device__ inline float2 exp2_fma2(float2 y) {
  constexpr float kRound = 12582912.f;  // 1.5 2^23
  const float2 yc = make_float2(fmaxf(y.x, -126.f), fmaxf(y.y, -126.f));
  const float2 t = fadd2(yc, make_float2(kRound, kRound));
  const float2 n = fadd2(t, make_float2(-kRound, -kRound));
  const float2 f = fadd2(yc, make_float2(-n.x, -n.y));
  float2 q = ffma2(make_float2(0.05517167f, 0.05517167f), f, make_float2(0.24261113f, 0.24261113f));
  q = ffma2(q, f, make_float2(0.69326097f, 0.69326097f));
  q = ffma2(q, f, make_float2(0.99992806f, 0.99992806f));
  return make_float2(float_of(bits_of(q.x) + (bits_of(t.x) << 23)), float_of(bits_of(q.y) + (bits_of(t.y) << 23)));
}
// ETA_EXP2_END

// max(a, b, c) in one instruction.
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Tensor-memory column of the 8 P columns feeding K step kk (16 keys) of
// half h's P V MMA in S buffer sb: half h wrote its 64 keys as 32 columns
// starting at column 64 h of the buffer.
__device__ __forceinline__ uint32_t p_col(int sb, int h, int kk) {
  return static_cast<uint32_t>(sb * BN + h * 64 + kk * 8);
}

struct Bars {
  uint64_t* q_full;    // producer -> MMA (tx bytes)
  uint64_t* k_full;    // [2] producer -> MMA (tx bytes)
  uint64_t* k_empty;   // [2] Q K^T commit -> producer
  uint64_t* v_full;    // [2] producer -> MMA, and the softmax before it zeroes rows of V
  uint64_t* v_empty;   // [2] P V commit -> producer
  uint64_t* s_full;    // [2] MMA commit -> softmax
  uint64_t* p_full;    // [2 buffers][2 halves] softmax (4 warps) -> MMA
  uint64_t* o_done;    // MMA commit after every P V -> softmax
  uint64_t* done;      // final commit of the MMA warp
  uint64_t* rv;        // rendezvous of the 8 softmax warps (bounded waits)
};

__global__ void __launch_bounds__(kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, PrefillArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = dev::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw);
  uint64_t* bar = reinterpret_cast<uint64_t*>(base + OFF_BARS);
  Bars Bs;
  Bs.q_full = bar;
  Bs.k_full = bar + 1;
  Bs.k_empty = bar + 3;
  Bs.v_full = bar + 5;
  Bs.v_empty = bar + 7;
  Bs.s_full = bar + 9;
  Bs.p_full = bar + 11;
  Bs.o_done = bar + 15;
  Bs.done = bar + 16;
  Bs.rv = bar + 17;
  float* red = reinterpret_cast<float*>(base + OFF_RED);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + OFF_BARS + 160);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(base + OFF_BARS + 164);
  int* issued_k = reinterpret_cast<int*>(base + OFF_BARS + 168);  // [2] parity of the last K copy per stage, -1 none
  int* issued_v = reinterpret_cast<int*>(base + OFF_BARS + 176);  // [2] same for V

  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  // blockIdx.x runs over (head, sequence) and blockIdx.y over query tiles,
  // last tile first: CTAs are dispatched in linear order, so the whole grid
  // goes heaviest first and the light tiles fill the end
  const int nqt = (a.T + BM - 1) / BM;
  const int qt = nqt - 1 - static_cast<int>(blockIdx.y);
  const int h = static_cast<int>(blockIdx.x) % a.Hq, b = static_cast<int>(blockIdx.x) / a.Hq;
  const int g = h / a.G;
  const int q0 = qt * BM;
  const int nt = qt + 1;  // key tiles 0..qt (causal)

  if (t == 0) {
    dev::mbar_init(Bs.q_full, 1);
    for (int k = 0; k < kStages; ++k) {
      dev::mbar_init(&Bs.k_full[k], 1);
      dev::mbar_init(&Bs.k_empty[k], 1);
      dev::mbar_init(&Bs.v_full[k], 1);
      dev::mbar_init(&Bs.v_empty[k], 1);
      dev::mbar_init(&Bs.s_full[k], 1);
      dev::mbar_init(&Bs.p_full[2 * k], kSoftWarps / 2);
      dev::mbar_init(&Bs.p_full[2 * k + 1], kSoftWarps / 2);
      issued_k[k] = -1;
      issued_v[k] = -1;
    }
    dev::mbar_init(Bs.o_done, 1);
    dev::mbar_init(Bs.done, 1);
    dev::mbar_init(Bs.rv, kSoftWarps);
    *abort_flag = 0;
    dev::fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, kTmemCols);
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tq)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tk)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tv)) : "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      bool ok = true;
      dev::mbar_arrive_expect_tx(Bs.q_full, TILE);
      const int qrow = (b * a.Hq + h) * a.T + q0;
      tma_load_2d(base_u32 + OFF_Q, &tq, 0, qrow, Bs.q_full);
      tma_load_2d(base_u32 + OFF_Q + PANEL, &tq, 64, qrow, Bs.q_full);
      const int krow0 = (b * a.Hkv + g) * a.kv_stride;
      for (int j = 0; j < nt; ++j) {
        const int st = j & 1;
        const uint32_t par = static_cast<uint32_t>(((j >> 1) & 1) ^ 1);
        const uint32_t ks = base_u32 + OFF_STAGE + static_cast<uint32_t>(st) * 2 * TILE, vs = ks + TILE;
        const int krow = krow0 + j * BN;
        if (!wait_or_abort(&Bs.k_empty[st], par, a.status, abort_flag)) {
          ok = false;
          break;
        }
        dev::mbar_arrive_expect_tx(&Bs.k_full[st], TILE);
        tma_load_2d(ks, &tk, 0, krow, &Bs.k_full[st]);
        tma_load_2d(ks + PANEL, &tk, 64, krow, &Bs.k_full[st]);
        issued_k[st] = (j >> 1) & 1;
        if (!wait_or_abort(&Bs.v_empty[st], par, a.status, abort_flag)) {
          ok = false;
          break;
        }
        dev::mbar_arrive_expect_tx(&Bs.v_full[st], TILE);
        tma_load_2d(vs, &tv, 0, krow, &Bs.v_full[st]);
        tma_load_2d(vs + PANEL, &tv, 64, krow, &Bs.v_full[st]);
        issued_v[st] = (j >> 1) & 1;
      }
      if (!ok) {
        *abort_flag = 1;
        // let the copies already issued land before the CTA winds down
        const long long t0 = clock64();
        while (!dev::mbar_try_wait(Bs.q_full, 0) && clock64() - t0 < dev::kWaitCycles) {
        }
        for (int k = 0; k < kStages; ++k) {
          if (issued_k[k] >= 0) {
            const long long t1 = clock64();
            while (!dev::mbar_try_wait(&Bs.k_full[k], static_cast<uint32_t>(issued_k[k])) &&
                   clock64() - t1 < dev::kWaitCycles) {
            }
          }
          if (issued_v[k] >= 0) {
            const long long t1 = clock64();
            while (!dev::mbar_try_wait(&Bs.v_full[k], static_cast<uint32_t>(issued_v[k])) &&
                   clock64() - t1 < dev::kWaitCycles) {
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // Issue order QK(0), QK(1), PV(0), QK(2), PV(1), ...: QK(j + 2) rewrites
    // S buffer j & 1 only after PV(j) read P_j from it.
    constexpr uint32_t idesc_qk = idesc_bf16(BM, BN, 0, 0);
    constexpr uint32_t idesc_pv = idesc_bf16(BM, D, 0, 1);
    bool ok = wait_or_abort(Bs.q_full, 0, a.status, abort_flag);
    auto issue_pv = [&](int i) -> bool {
      const int sb = i & 1;
      const uint32_t vs = base_u32 + OFF_STAGE + static_cast<uint32_t>(sb) * 2 * TILE + TILE;
      if (!wait_or_abort(&Bs.v_full[sb], static_cast<uint32_t>((i >> 1) & 1), a.status, abort_flag)) return false;
      for (int hh = 0; hh < 2; ++hh) {
        if (!wait_or_abort(&Bs.p_full[2 * sb + hh], static_cast<uint32_t>((i >> 1) & 1), a.status, abort_flag))
          return false;
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sw128_desc(vs + (hh * 4 + kk) * 2048, PANEL, 1024);
            mma_bf16_tmem_a(tmem + kOCol + hh * BN, tmem + p_col(sb, hh, kk), bd, idesc_pv,
                            (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (lane == 0) {
        mma_commit(Bs.o_done);
        mma_commit(&Bs.v_empty[sb]);
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int st = j & 1;
      if (!wait_or_abort(&Bs.k_full[st], (j >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (lane == 0) {
        const uint32_t ks = base_u32 + OFF_STAGE + static_cast<uint32_t>(st) * 2 * TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * PANEL + (kk & 3) * 32;
          const uint64_t ad = sw128_desc(base_u32 + OFF_Q + off, 16, 1024);
          const uint64_t bd = sw128_desc(ks + off, 16, 1024);
          mma_bf16(tmem + static_cast<uint32_t>(st) * BN, ad, bd, idesc_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(&Bs.s_full[st]);
        mma_commit(&Bs.k_empty[st]);
      }
      __syncwarp();
      if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok) issue_pv(nt - 1);
    // every MMA issued so far has completed once `done` flips
    if (lane == 0) mma_commit(Bs.done);
    __syncwarp();
    {
      const long long t0 = clock64();
      while (!dev::mbar_try_wait(Bs.done, 0) && clock64() - t0 < dev::kWaitCycles) {
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    const int qq = warp & 3;               // tensor-memory lane quarter of this warp
    const int hf = (warp - 2) >> 2;        // which 64 key columns (and 64 O columns)
    const uint32_t lane_base = static_cast<uint32_t>(32 * qq) << 16;
    const int r = 32 * qq + lane;          // query row of the tile
    const int i = q0 + r;
    const bool row_ok = i < a.T;
    const size_t row = static_cast<size_t>(b * a.Hq + h) * a.T + i;
    const int st_id = t - 64;              // 0..255 among the softmax threads
    float tau = 0.f;
    if (row_ok) {
      if (a.tau_mode == ETA_TAU_LEARNED) {
        const uint4* qp = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.q) + row * D);
        const float4* wp = reinterpret_cast<const float4*>(a.w_tau + static_cast<size_t>(h) * D);
        float acc = 0.f;
#pragma unroll 4
        for (int c = 0; c < D / 8; ++c) {
          const uint4 u = qp[c];
          const float4 w0 = wp[2 * c], w1 = wp[2 * c + 1];
          acc = fmaf(bf16_lo_f(u.x), w0.x, acc);
          acc = fmaf(bf16_hi_f(u.x), w0.y, acc);
          acc = fmaf(bf16_lo_f(u.y), w0.z, acc);
          acc = fmaf(bf16_hi_f(u.y), w0.w, acc);
          acc = fmaf(bf16_lo_f(u.z), w1.x, acc);
          acc = fmaf(bf16_hi_f(u.z), w1.y, acc);
          acc = fmaf(bf16_lo_f(u.w), w1.z, acc);
          acc = fmaf(bf16_hi_f(u.w), w1.w, acc);
        }
        tau = acc + a.b_tau[h] - a.offset_a;
      } else {
        tau = a.c_tau[h] - a.offset_a;
      }
    }
    const float scale = a.scale, beta = a.beta;
    float m_run = -INFINITY, l_part = 0.f, r_part = 0.f;
    bool ok = true;
    // Consecutive rendezvous complete consecutive phases of Bs.rv; a warp can
    // run at most one phase ahead of the slowest, and every wait is bounded
    // (an abort anywhere releases all of them).
    uint32_t rv_phase = 0;
    auto rendezvous = [&]() -> bool {
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(Bs.rv);
      const bool r2 = warp_wait_or_abort(Bs.rv, rv_phase, a.status, abort_flag);
      rv_phase ^= 1u;
      return r2;
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int sb = j & 1;
      if (!warp_wait_or_abort(&Bs.s_full[sb], (j >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t s0[32], s1[32];
      const uint32_t scol = tmem + lane_base + static_cast<uint32_t>(sb * BN + hf * 64);
      tmem_ld32_nowait(scol, s0);
      tmem_ld32_nowait(scol + 32, s1);
      tmem_wait_ld();

      // keys j BN + c with c <= lim are seen by this row (causal; rows past
      // the sequence see none).  Off the diagonal every key of every row of
      // the warp is seen: no masking there.
      // gate(beta (scale S - tau)) = 1/2 + t / 2 with t = tanh(cb S + ct),
      // x = cx S gate = u + u t with u = cx S / 2; the gate sum over a full
      // half is 32 + (sum t) / 2.
      const int lim = row_ok ? min(BN - 1, i - j * BN) - hf * 64 : -1;
      const bool full = __all_sync(0xffffffffu, lim >= 63);
      const float cb = 0.5f * beta * scale, ct = -0.5f * beta * tau, cx = scale * kLog2e, cu = 0.5f * cx;
      float pm = -INFINITY;
      if (full) {
        const float2 cb2 = make_float2(cb, cb), ct2 = make_float2(ct, ct), cu2 = make_float2(cu, cu);
        float2 ts2 = make_float2(0.f, 0.f);
        float pm1 = -INFINITY;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          uint32_t& sa = e < 16 ? s0[2 * e] : s1[2 * e - 32];
          uint32_t& sz = e < 16 ? s0[2 * e + 1] : s1[2 * e + 1 - 32];
          const float2 S2 = make_float2(__uint_as_float(sa), __uint_as_float(sz));
          const float2 a2 = ffma2(S2, cb2, ct2);
          const float2 t2 = make_float2(tanh_approx(a2.x), tanh_approx(a2.y));
          const float2 u2 = fmul2(S2, cu2);
          const float2 x2 = ffma2(u2, t2, u2);
          ts2 = fadd2(ts2, t2);
          if (e & 1) pm1 = max3f(pm1, x2.x, x2.y);
          else pm = max3f(pm, x2.x, x2.y);
          sa = __float_as_uint(x2.x);
          sz = __float_as_uint(x2.y);
        }
        pm = fmaxf(pm, pm1);
        r_part += fmaf(0.5f, ts2.x + ts2.y, 32.f);
      } else {
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          uint32_t& sv = c < 32 ? s0[c] : s1[c - 32];
          const float Sr = __uint_as_float(sv);
          const float sg = fmaf(0.5f, tanh_approx(fmaf(Sr, cb, ct)), 0.5f);
          const float x = Sr * cx * sg;
          const bool on = c <= lim;
          r_part += on ? sg : 0.f;
          pm = fmaxf(pm, on ? x : -INFINITY);
          sv = __float_as_uint(on ? x : -INFINITY);
        }
      }
      const float mt = pm;

      // A row whose max grew past the margin moves its reference; if it had
      // weights already, its O row is rescaled once P V of the previous tile
      // is done (P_j is not issued yet).  Tensor-memory loads and stores are
      // warp-wide, so the whole warp runs them (alpha = 1 for other rows).
      const bool grow = mt > m_run + kLazy;
      const bool rescale = grow && m_run != -INFINITY;
      if (__any_sync(0xffffffffu, rescale)) {
        if (!warp_wait_or_abort(Bs.o_done, static_cast<uint32_t>((j - 1) & 1), a.status, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const float alpha = rescale ? dev::fast_exp2(m_run - mt) : 1.f;
        const uint32_t ocol = tmem + lane_base + kOCol + static_cast<uint32_t>(hf * BN);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          uint32_t o[32];
          tmem_ld32_nowait(ocol + 32 * k, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
          tmem_st32(ocol + 32 * k, o);
        }
        tmem_wait_st();
        l_part *= alpha;
      }
      if (grow) m_run = mt;

      // P_j = 2^(x - m_run) as bf16 pairs over this half's S columns; l sums
      // the fp32 weights (their bf16 rounding is below the output's own)
      uint32_t pk[32];
      float lsum = 0.f;
      if (full) {
        const float2 nm2 = make_float2(-m_run, -m_run);
        float2 ls2 = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float2 x2 = make_float2(__uint_as_float(e < 16 ? s0[2 * e] : s1[2 * e - 32]),
                                        __uint_as_float(e < 16 ? s0[2 * e + 1] : s1[2 * e + 1 - 32]));
          const float2 y2 = fadd2(x2, nm2);
          // three pairs in eight on the FMA pipes, the rest on the
          // special-function unit (more shifts the bound to the issue rate)
          const float2 p2 = (e & 7) < 3 ? exp2_fma2(y2) : make_float2(dev::fast_exp2(y2.x), dev::fast_exp2(y2.y));
          pk[e] = pack_bf16(p2.x, p2.y);
          ls2 = fadd2(ls2, p2);
        }
        lsum = ls2.x + ls2.y;
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float x0 = __uint_as_float(e < 16 ? s0[2 * e] : s1[2 * e - 32]);
          const float x1 = __uint_as_float(e < 16 ? s0[2 * e + 1] : s1[2 * e + 1 - 32]);
          const float p0 = x0 == -INFINITY ? 0.f : dev::fast_exp2(x0 - m_run);
          const float p1 = x1 == -INFINITY ? 0.f : dev::fast_exp2(x1 - m_run);
          pk[e] = pack_bf16(p0, p1);
          lsum += p0 + p1;
        }
      }
      l_part += lsum;
      tmem_st32(scol, pk);
      tmem_wait_st();
      // V rows of this tile past the sequence end hold no key: zeroed so that
      // stale or non-finite bytes there cannot reach O (0 * inf)
      // (each half zeroes the rows its own P V reads, before it signals P)
      const int z0 = max(a.T - j * BN, hf * 64), z1 = hf * 64 + 64;
      if (z0 < z1) {
        // V_j has its own barrier: its copy lands before the zeroing
        if (!warp_wait_or_abort(&Bs.v_full[sb], static_cast<uint32_t>((j >> 1) & 1), a.status, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* vt = base + OFF_STAGE + sb * 2 * TILE + TILE;
        const int nz = (z1 - z0) * 8;  // 16-byte chunks per panel
        for (int c = st_id & 127; c < 2 * nz; c += kSoftThreads / 2) {
          const int pnl = c / nz, rem = c - pnl * nz;
          *reinterpret_cast<uint4*>(vt + pnl * PANEL + (z0 + (rem >> 3)) * 128 + (rem & 7) * 16) =
              make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&Bs.p_full[2 * sb + hf]);
    }
    if (ok) ok = warp_wait_or_abort(Bs.o_done, static_cast<uint32_t>((nt - 1) & 1), a.status, abort_flag);
    tc_fence_after();
    // the two halves of a row are merged: m* = max m_h, l = sum 2^(m_h - m*) l_h,
    // out = sum 2^(m_h - m*) O_h / l (every softmax thread reaches this point)
    float* mred = red;             // [2 halves][128]
    float* lred = red + 2 * BM;
    float* rred = red + 4 * BM;
    mred[hf * BM + r] = m_run;
    lred[hf * BM + r] = l_part;
    rred[hf * BM + r] = r_part;
    if (!rendezvous()) ok = false;
    if (ok) {
      const float m0 = mred[r], m1 = mred[BM + r];
      const float ms = fmaxf(m0, m1);
      const float f0 = m0 == -INFINITY ? 0.f : dev::fast_exp2(m0 - ms);
      const float f1 = m1 == -INFINITY ? 0.f : dev::fast_exp2(m1 - ms);
      const float l_run = f0 * lred[r] + f1 * lred[BM + r];
      const float inv = (row_ok && l_run > 0.f) ? 1.f / l_run : 0.f;
      const float g0 = f0 * inv, g1 = f1 * inv;
      uint4* orow = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.out) + row * D + hf * 64);
      const uint32_t ocol = tmem + lane_base + kOCol + static_cast<uint32_t>(hf * 64);
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        uint32_t o0[32], o1[32];
        tmem_ld32_nowait(ocol + 32 * k, o0);
        tmem_ld32_nowait(ocol + BN + 32 * k, o1);
        tmem_wait_ld();
        if (row_ok) {
#pragma unroll
          for (int c8 = 0; c8 < 4; ++c8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int c = 8 * c8 + 2 * e;
              w[e] = pack_bf16(fmaf(__uint_as_float(o0[c]), g0, __uint_as_float(o1[c]) * g1),
                               fmaf(__uint_as_float(o0[c + 1]), g0, __uint_as_float(o1[c + 1]) * g1));
            }
            orow[4 * k + c8] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
      if (row_ok && hf == 0) {
        if (a.lse) a.lse[row] = l_run > 0.f ? (ms + log2f(l_run)) * kLn2 : -INFINITY;
        if (a.gate_sum) a.gate_sum[row] = rred[r] + rred[BM + r];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a, cudaStream_t st) {
  CUtensorMap tq, tk, tv;
  const uint64_t qrows = static_cast<uint64_t>(a.B) * a.Hq * a.T;
  const uint64_t kvrows = static_cast<uint64_t>(a.B) * a.Hkv * a.kv_stride;
  if (!make_map(&tq, a.q, qrows, BM) || !make_map(&tk, a.k, kvrows, BN) || !make_map(&tv, a.v, kvrows, BN))
    return cudaErrorInvalidValue;
  static SmemLimit lim;
  const dim3 grid(a.Hq * a.B, (a.T + BM - 1) / BM);
  return launch_with_smem(reinterpret_cast<const void*>(prefill_tc_kernel), kSmemBytes, lim, [&] {
    prefill_tc_kernel<<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, a);
    return cudaGetLastError();
  });
}

}  // namespace eta
