/* Drives cvq_attend from C, with no Python in the loop: one decode step of a synthetic
 * layer per iteration.  Prints one JSON line with
 *   host_us_per_call   host time of one cvq_attend call (enqueue only: argument checks,
 *                      the cached tensor maps, the launch), measured over calls issued
 *                      back to back;
 *   device_us_per_step device time per step with the inputs resident on the device
 *                      (CUDA events around the back-to-back steps);
 *   e2e_us_per_step    device time per step when every step first copies its codes and
 *                      queries from pinned host memory and reads out and lse back.
 * The caller allocates every buffer (cudaMalloc / cudaMallocHost); the library allocates
 * nothing.  The values are synthetic (a fixed linear congruential stream): only the
 * timing is reported.
 *
 * usage: attend_loop B Hq Hkv R T steps
 * build: gcc -std=c99 -O2 -I include -I <cuda>/include tests/c_abi/attend_loop.c \
 *            -L compressed_attention_cvq_b200 -lcvq -L <cuda>/lib64 -lcudart -o attend_loop
 */
#define _POSIX_C_SOURCE 199309L
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#include "cvq.h"

#define CK(x)                                                                   \
  do {                                                                          \
    cudaError_t e_ = (x);                                                       \
    if (e_ != cudaSuccess) {                                                    \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x,                 \
              cudaGetErrorString(e_));                                          \
      return 2;                                                                 \
    }                                                                           \
  } while (0)
#define CV(x)                                                                   \
  do {                                                                          \
    int s_ = (int)(x);                                                          \
    if (s_ != CVQ_OK) {                                                         \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #x,                 \
              cvq_status_str(s_));                                              \
      return 3;                                                                 \
    }                                                                           \
  } while (0)

static uint32_t lcg_state = 12345u;
static uint32_t lcg(void) { lcg_state = lcg_state * 1664525u + 1013904223u; return lcg_state; }
static float unif(void) { return (float)(lcg() >> 8) / 16777216.0f - 0.5f; }

static double now_us(void) {
  struct timespec ts;
  clock_gettime(CLOCK_MONOTONIC, &ts);
  return ts.tv_sec * 1e6 + ts.tv_nsec * 1e-3;
}

int main(int argc, char** argv) {
  if (argc != 7) {
    fprintf(stderr, "usage: %s B Hq Hkv R T steps\n", argv[0]);
    return 1;
  }
  cvq_shape s;
  memset(&s, 0, sizeof s);
  s.batch = atoi(argv[1]);
  s.n_q_heads = atoi(argv[2]);
  s.n_kv_heads = atoi(argv[3]);
  s.head_dim = CVQ_HEAD_DIM;
  s.R = atoi(argv[4]);
  s.t_cap = atoi(argv[5]);
  s.rope_base = 500000.0f;
  s.group_dim = 8;
  const int steps = atoi(argv[6]);
  if (steps < 1) return 1;

  const size_t nq = (size_t)s.batch * s.n_q_heads * CVQ_HEAD_DIM;
  const size_t ncb = (size_t)s.n_kv_heads * CVQ_GROUPS * s.R * CVQ_CODES * 8;
  const size_t ncode = (size_t)s.batch * s.n_kv_heads * s.t_cap * s.R * 16;
  const size_t nout = nq, nlse = (size_t)s.batch * s.n_q_heads;

  float *hq, *hcb;
  uint8_t *hkc, *hvc;
  float *hout, *hlse;
  int32_t* hlen;
  CK(cudaMallocHost((void**)&hq, nq * 4));
  CK(cudaMallocHost((void**)&hcb, ncb * 4));
  CK(cudaMallocHost((void**)&hkc, ncode));
  CK(cudaMallocHost((void**)&hvc, ncode));
  CK(cudaMallocHost((void**)&hout, nout * 4));
  CK(cudaMallocHost((void**)&hlse, nlse * 4));
  CK(cudaMallocHost((void**)&hlen, s.batch * 4));
  for (size_t i = 0; i < nq; ++i) hq[i] = 2.0f * unif();
  for (size_t i = 0; i < ncb; ++i) hcb[i] = 2.0f * unif();
  for (size_t i = 0; i < ncode; ++i) { hkc[i] = (uint8_t)(lcg() >> 24); hvc[i] = (uint8_t)(lcg() >> 24); }
  for (int b = 0; b < s.batch; ++b) hlen[b] = s.t_cap;

  int dev = 0, sms = 0;
  CK(cudaGetDevice(&dev));
  CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  const int splits = cvq_suggest_splits(&s, sms);
  const size_t nws = cvq_attend_workspace_bytes(&s, splits);
  if (nws == 0) return 3;

  float *q, *kcb, *vcb, *out, *lse;
  uint8_t *kc, *vc;
  int32_t* len;
  void* ws;
  CK(cudaMalloc((void**)&q, nq * 4));
  CK(cudaMalloc((void**)&kcb, ncb * 4));
  CK(cudaMalloc((void**)&vcb, ncb * 4));
  CK(cudaMalloc((void**)&kc, ncode));
  CK(cudaMalloc((void**)&vc, ncode));
  CK(cudaMalloc((void**)&len, s.batch * 4));
  CK(cudaMalloc((void**)&out, nout * 4));
  CK(cudaMalloc((void**)&lse, nlse * 4));
  CK(cudaMalloc(&ws, nws));
  CK(cudaMemset(ws, 0, nws));
  CK(cudaMemcpy(q, hq, nq * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(kcb, hcb, ncb * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(vcb, hcb, ncb * 4, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(kc, hkc, ncode, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(vc, hvc, ncode, cudaMemcpyHostToDevice));
  CK(cudaMemcpy(len, hlen, s.batch * 4, cudaMemcpyHostToDevice));

  cudaStream_t st;
  CK(cudaStreamCreate(&st));
  const int64_t stride = (int64_t)(ncb / s.n_kv_heads);
#define ATTEND() cvq_attend(&s, q, CVQ_F32, kcb, stride, kc, vc, len, vcb, stride, splits, ws, out, lse, st)
  for (int i = 0; i < 5; ++i) CV(ATTEND());
  CK(cudaStreamSynchronize(st));

  /* host cost and device time of back-to-back steps on resident inputs */
  cudaEvent_t e0, e1;
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  CK(cudaEventRecord(e0, st));
  const double h0 = now_us();
  for (int i = 0; i < steps; ++i) CV(ATTEND());
  const double h1 = now_us();
  CK(cudaEventRecord(e1, st));
  CK(cudaEventSynchronize(e1));
  float dev_ms = 0.f;
  CK(cudaEventElapsedTime(&dev_ms, e0, e1));

  /* end to end: codes and queries up, the step, out and lse down, every step */
  CK(cudaEventRecord(e0, st));
  for (int i = 0; i < steps; ++i) {
    CK(cudaMemcpyAsync(kc, hkc, ncode, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(vc, hvc, ncode, cudaMemcpyHostToDevice, st));
    CK(cudaMemcpyAsync(q, hq, nq * 4, cudaMemcpyHostToDevice, st));
    CV(ATTEND());
    CK(cudaMemcpyAsync(hout, out, nout * 4, cudaMemcpyDeviceToHost, st));
    CK(cudaMemcpyAsync(hlse, lse, nlse * 4, cudaMemcpyDeviceToHost, st));
  }
  CK(cudaEventRecord(e1, st));
  CK(cudaEventSynchronize(e1));
  float e2e_ms = 0.f;
  CK(cudaEventElapsedTime(&e2e_ms, e0, e1));
  uint32_t fault = 0;
  CV(cvq_fault_status(&fault, 1));
  int finite = 1;
  for (size_t i = 0; i < nout; ++i) finite &= (hout[i] == hout[i]);

  printf("{\"caller\": \"C\", \"batch\": %d, \"n_q_heads\": %d, \"n_kv_heads\": %d, \"R\": %d, "
         "\"t_cap\": %d, \"n_splits\": %d, \"steps\": %d, \"host_us_per_call\": %.3f, "
         "\"device_us_per_step\": %.3f, \"e2e_us_per_step\": %.3f, \"h2d_bytes_per_step\": %zu, "
         "\"d2h_bytes_per_step\": %zu, \"fault\": %u, \"outputs_finite\": %d}\n",
         s.batch, s.n_q_heads, s.n_kv_heads, s.R, s.t_cap, splits, steps, (h1 - h0) / steps,
         1e3 * dev_ms / steps, 1e3 * e2e_ms / steps, 2 * ncode + nq * 4, (nout + nlse) * 4, fault,
         finite);
  return (fault == 0 && finite) ? 0 : 4;
}
