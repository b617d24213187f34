/*
 * A plain C caller of libqsa.so (no Python, no torch): the way a serving runtime written in
 * C or C++ uses the boundary declared in include/qsa.h.  It builds a seeded random batch
 * on the host (bf16 Q, K and V; int32 slot lists with masked entries, a fully masked row
 * and rows of different widths), asks qsa_sparse_prefill_plan for the split plan and its
 * workspace, runs qsa_sparse_prefill on a stream of its own (the automatic plan and a
 * forced three-way split), copies the output back, and compares it element by element
 * with the CPU oracle (test infrastructure, linked in for the check) at the parity gates
 * of the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN
 * prefill PR", section "Nine tests that passed, and a speed number that did not come from
 * this branch" (atol 0.025, rtol 0.025, relative L2 below 0.008, masked rows exactly 0).
 * Exit status 0 when every check passes.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "qsa.h"

/* the CPU oracle (oracle/qsa_oracle.c) */
int qsa_oracle_forward(const uint16_t* q, int64_t q_stride_t, int64_t q_stride_h,
                       const uint16_t* k_cache, int64_t k_stride_s, int64_t k_stride_h,
                       const uint16_t* v_cache, int64_t v_stride_s, int64_t v_stride_h,
                       const int32_t* slot_idx, int64_t idx_stride_t, const int32_t* width,
                       int32_t Tq, int32_t Hq, int32_t Hkv, int32_t D, int64_t S, int32_t W,
                       float scale, const int64_t* rows, int64_t nrows, float* out,
                       uint32_t* err_bits);

enum { TQ = 160, HQ = 16, HKV = 2, D = 256, S = 4096, W = 700 };

static uint64_t g_state = 0x9e3779b97f4a7c15ull;
static uint32_t next_u32(void) { /* 64-bit LCG, high half */
  g_state = g_state * 6364136223846793005ull + 1442695040888963407ull;
  return (uint32_t)(g_state >> 32);
}
static float next_normal(void) { /* sum of four uniforms, centred and scaled to unit variance */
  float s = 0.f;
  for (int i = 0; i < 4; ++i) s += (float)next_u32() / 4294967296.0f;
  return (s - 2.0f) * 1.7320508f;
}
static uint16_t to_bf16(float x) { /* round to nearest even (finite inputs) */
  uint32_t u;
  memcpy(&u, &x, 4);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}
static float from_bf16(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float x;
  memcpy(&x, &u, 4);
  return x;
}

#define CHECK_CUDA(call)                                                    \
  do {                                                                      \
    cudaError_t e_ = (call);                                                \
    if (e_ != cudaSuccess) {                                                \
      fprintf(stderr, "%s: %s\n", #call, cudaGetErrorString(e_));           \
      return 2;                                                             \
    }                                                                       \
  } while (0)

int main(void) {
  const size_t nq = (size_t)TQ * HQ * D, nkv = (size_t)S * HKV * D, ni = (size_t)TQ * W;
  uint16_t* q = malloc(nq * 2);
  uint16_t* k = malloc(nkv * 2);
  uint16_t* v = malloc(nkv * 2);
  int32_t* idx = malloc(ni * 4);
  int32_t* width = malloc(TQ * 4);
  int32_t* perm = malloc(S * 4);
  uint16_t* got = malloc(nq * 2);
  float* ref = malloc(nq * 4);
  if (!q || !k || !v || !idx || !width || !perm || !got || !ref) return 2;
  for (size_t i = 0; i < nq; ++i) q[i] = to_bf16(next_normal());
  for (size_t i = 0; i < nkv; ++i) k[i] = to_bf16(next_normal());
  for (size_t i = 0; i < nkv; ++i) v[i] = to_bf16(next_normal());
  for (int t = 0; t < TQ; ++t) { /* W distinct slots: a partial Fisher-Yates shuffle */
    for (int s = 0; s < S; ++s) perm[s] = s;
    for (int w = 0; w < W; ++w) {
      const int j = w + (int)(next_u32() % (uint32_t)(S - w));
      const int tmp = perm[w];
      perm[w] = perm[j];
      perm[j] = tmp;
      idx[(size_t)t * W + w] = (next_u32() % 10u == 0u) ? -1 : perm[w];
    }
    width[t] = (int32_t)(next_u32() % (uint32_t)(W + 1));
  }
  for (int w = 0; w < W; ++w) idx[3 * W + w] = -1; /* row 3: every entry masked */
  width[3] = W;
  width[5] = 0; /* row 5: zero width */

  int dev = 0, num_sms = 0;
  CHECK_CUDA(cudaSetDevice(dev));
  CHECK_CUDA(cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev));
  void *dq, *dk, *dv, *didx, *dwidth, *dout, *dws = NULL;
  uint32_t* derr;
  CHECK_CUDA(cudaMalloc(&dq, nq * 2));
  CHECK_CUDA(cudaMalloc(&dk, nkv * 2));
  CHECK_CUDA(cudaMalloc(&dv, nkv * 2));
  CHECK_CUDA(cudaMalloc(&didx, ni * 4));
  CHECK_CUDA(cudaMalloc(&dwidth, TQ * 4));
  CHECK_CUDA(cudaMalloc(&dout, nq * 2));
  CHECK_CUDA(cudaMalloc((void**)&derr, 4));
  CHECK_CUDA(cudaMemcpy(dq, q, nq * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dk, k, nkv * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dv, v, nkv * 2, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(didx, idx, ni * 4, cudaMemcpyHostToDevice));
  CHECK_CUDA(cudaMemcpy(dwidth, width, TQ * 4, cudaMemcpyHostToDevice));
  cudaStream_t stream;
  CHECK_CUDA(cudaStreamCreateWithFlags(&stream, cudaStreamNonBlocking));

  uint32_t bits = 0;
  if (qsa_oracle_forward(q, HQ * D, D, k, HKV * D, D, v, HKV * D, D, idx, W, width, TQ, HQ, HKV,
                         D, S, W, 1.0f / 16.0f, NULL, 0, ref, &bits) != 0)
    return 3;

  int failures = 0;
  const int32_t requests[2] = {0, 3};
  for (int c = 0; c < 2; ++c) {
    size_t ws_bytes = 0;
    const int32_t nsplit = qsa_sparse_prefill_plan(TQ, HQ, HKV, D, W, num_sms, requests[c],
                                                   &ws_bytes);
    if (nsplit < 1) {
      fprintf(stderr, "plan: %s\n", qsa_last_error_detail());
      return 4;
    }
    if (ws_bytes > 0) CHECK_CUDA(cudaMalloc(&dws, ws_bytes));
    CHECK_CUDA(cudaMemsetAsync(derr, 0, 4, stream));
    CHECK_CUDA(cudaMemsetAsync(dout, 0xff, nq * 2, stream));
    const qsa_status_t st = qsa_sparse_prefill(
        dq, HQ * D, D, dk, HKV * D, D, dv, HKV * D, D, (const int32_t*)didx, W,
        (const int32_t*)dwidth, TQ, HQ, HKV, D, S, W, 1.0f / 16.0f, dout, HQ * D, D, nsplit, dws,
        ws_bytes, derr, (void*)stream);
    if (st != QSA_OK) {
      fprintf(stderr, "qsa_sparse_prefill: %s: %s\n", qsa_status_string(st), qsa_last_error_detail());
      return 5;
    }
    uint32_t err_word = 0;
    CHECK_CUDA(cudaMemcpyAsync(got, dout, nq * 2, cudaMemcpyDeviceToHost, stream));
    CHECK_CUDA(cudaMemcpyAsync(&err_word, derr, 4, cudaMemcpyDeviceToHost, stream));
    CHECK_CUDA(cudaStreamSynchronize(stream));
    if (dws) {
      CHECK_CUDA(cudaFree(dws));
      dws = NULL;
    }
    double num = 0.0, den = 0.0, max_err = 0.0;
    int bad = 0;
    for (size_t i = 0; i < nq; ++i) {
      const double g = from_bf16(got[i]), r = ref[i], e = fabs(g - r);
      if (!(e <= 0.025 + 0.025 * fabs(r))) ++bad;
      num += e * e;
      den += r * r;
      if (e > max_err) max_err = e;
    }
    for (int t = 3; t <= 5; t += 2) /* masked and zero-width rows: exact +0 bits */
      for (size_t i = (size_t)t * HQ * D; i < (size_t)(t + 1) * HQ * D; ++i) bad += got[i] != 0;
    const double rel = sqrt(num / (den > 0 ? den : 1));
    printf("nsplit=%d workspace=%zu max_abs_err=%.3e rel_l2=%.3e err_word=%u bad=%d\n", nsplit,
           ws_bytes, max_err, rel, err_word, bad);
    if (bad || !(rel < 0.008) || err_word != bits) ++failures;
  }
  printf(failures ? "FAILED\n" : "OK\n");
  return failures ? 1 : 0;
}
