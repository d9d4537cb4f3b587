/*
 * One ETA decode step through the C ABI alone (C99, CUDA runtime for device
 * memory, no Python): a bf16 cache of one sequence, 16 query / 4 KV heads,
 * d = 128, 4096 tokens in blocks of 64, calibrated thresholds.  Builds the
 * block metadata, sizes and runs the decode, checks the device status and
 * prints a checksum of the output.  Exit code 0 on success.
 *
 *   cc -std=c99 -I include -I <cuda>/include tests/c/decode_example.c \
 *      -L learned_threshold_sparse_b200 -leta -L <cuda>/lib64 -lcudart -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "eta.h"

enum { B = 1, HQ = 16, HKV = 4, D = 128, BS = 64, CTX = 4096 };

static uint16_t to_bf16(float x) {
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7fffu + ((u >> 16) & 1u); /* round to nearest even (finite inputs) */
  return (uint16_t)(u >> 16);
}

static float from_bf16(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

static float uniform(uint64_t* s) { /* splitmix64 -> [-1, 1) */
  uint64_t z = (*s += 0x9e3779b97f4a7c15ull);
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
  z ^= z >> 31;
  return (float)((double)(z >> 11) / 9007199254740992.0) * 2.0f - 1.0f;
}

#define CHECK(x)                                                         \
  do {                                                                   \
    if ((x) != cudaSuccess) {                                            \
      fprintf(stderr, "CUDA error at %s:%d\n", __FILE__, __LINE__);      \
      return 1;                                                          \
    }                                                                    \
  } while (0)

int main(void) {
  const size_t n_kv = (size_t)B * HKV * CTX * D, n_q = (size_t)B * HQ * D;
  const int nb = (CTX + BS - 1) / BS;
  uint16_t* h_kv = (uint16_t*)malloc(2 * n_kv * sizeof(uint16_t));
  uint16_t* h_q = (uint16_t*)malloc(n_q * sizeof(uint16_t));
  uint16_t* h_out = (uint16_t*)malloc(n_q * sizeof(uint16_t));
  float h_c[HQ];
  uint64_t seed = 1;
  if (!h_kv || !h_q || !h_out) return 1;
  for (size_t i = 0; i < 2 * n_kv; ++i) h_kv[i] = to_bf16(uniform(&seed));
  for (size_t i = 0; i < n_q; ++i) h_q[i] = to_bf16(uniform(&seed));
  for (int h = 0; h < HQ; ++h) h_c[h] = 0.6f;

  void *k, *v, *q, *out, *mu, *sigma, *ws;
  float *max_norm, *lse, *c_tau;
  int *seq, *first;
  const int h_seq = CTX, h_first = 0;
  CHECK(cudaMalloc(&k, n_kv * 2));
  CHECK(cudaMalloc(&v, n_kv * 2));
  CHECK(cudaMalloc(&q, n_q * 2));
  CHECK(cudaMalloc(&out, n_q * 2));
  CHECK(cudaMalloc(&mu, (size_t)B * HKV * nb * D * 2));
  CHECK(cudaMalloc(&sigma, (size_t)B * HKV * nb * D * 2));
  CHECK(cudaMalloc((void**)&max_norm, (size_t)B * HKV * nb * 4));
  CHECK(cudaMalloc((void**)&lse, (size_t)B * HQ * 4));
  CHECK(cudaMalloc((void**)&c_tau, HQ * 4));
  CHECK(cudaMalloc((void**)&seq, 4));
  CHECK(cudaMalloc((void**)&first, 4));
  CHECK(cudaMemcpy(k, h_kv, n_kv * 2, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(v, h_kv + n_kv, n_kv * 2, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(q, h_q, n_q * 2, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(c_tau, h_c, sizeof(h_c), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(seq, &h_seq, 4, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(first, &h_first, 4, cudaMemcpyHostToDevice));

  eta_decode_params p;
  memset(&p, 0, sizeof(p));
  p.cache.batch = B;
  p.cache.n_q_heads = HQ;
  p.cache.n_kv_heads = HKV;
  p.cache.head_dim = D;
  p.cache.block_size = BS;
  p.cache.max_ctx = CTX;
  p.cache.kv_dtype = ETA_BF16;
  p.cache.k_cache = k;
  p.cache.v_cache = v;
  p.cache.seq_lens = seq;
  p.summary.mu = mu;
  p.summary.sigma = sigma;
  p.summary.max_norm = max_norm;
  p.summary.format = ETA_META_FP16;
  p.q = q;
  p.tau_mode = ETA_TAU_CALIBRATED;
  p.c_tau = c_tau;
  p.scale = 1.0f / sqrtf((float)D);
  p.beta = 5.0f;
  p.z = 2.0f;
  p.n_local_blocks = 2;
  p.screen_enabled = 1;
  p.attend_impl = ETA_ATTEND_AUTO;
  p.out = out;
  p.lse = lse;

  eta_status st = eta_block_summary_update(&p.cache, &p.summary, first, nb, NULL);
  if (st != ETA_OK) {
    fprintf(stderr, "eta_block_summary_update: %s\n", eta_status_string(st));
    return 1;
  }
  st = eta_decode_workspace_size(&p, &p.workspace_bytes);
  if (st != ETA_OK) {
    fprintf(stderr, "eta_decode_workspace_size: %s\n", eta_status_string(st));
    return 1;
  }
  CHECK(cudaMalloc(&ws, p.workspace_bytes));
  CHECK(cudaMemset(ws, 0, p.workspace_bytes));
  p.workspace = ws;
  st = eta_decode(&p, NULL);
  if (st == ETA_OK) st = eta_read_device_status(ws, NULL);
  if (st != ETA_OK) {
    fprintf(stderr, "eta_decode: %s\n", eta_status_string(st));
    return 1;
  }
  CHECK(cudaMemcpy(h_out, out, n_q * 2, cudaMemcpyDeviceToHost));
  double sum = 0.0;
  for (size_t i = 0; i < n_q; ++i) sum += fabs((double)from_bf16(h_out[i]));
  printf("%s\ndecode ok: sum |out| = %.6f\n", eta_build_info(), sum);
  cudaFree(k); cudaFree(v); cudaFree(q); cudaFree(out); cudaFree(mu); cudaFree(sigma);
  cudaFree(max_norm); cudaFree(lse); cudaFree(c_tau); cudaFree(seq); cudaFree(first); cudaFree(ws);
  free(h_kv); free(h_q); free(h_out);
  return 0;
}
