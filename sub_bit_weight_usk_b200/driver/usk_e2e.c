/*
 * usk_e2e.c -- end-to-end timing of usk_gemv through the C ABI alone (no
 * Python): per call, the activations go host -> device from pinned memory,
 * usk_gemv runs, and the result comes back device -> host, then the stream is
 * synchronised -- the round trip a C caller of libusk pays per product.
 *
 *   usk_e2e M K batch iters [warmup]
 *
 * Prints one JSON line: e2e_us (mean wall time per round trip, CLOCK_MONOTONIC),
 * kernel_loop_us (mean device time per call of a back-to-back loop of usk_gemv
 * with no copies, CUDA events), the bytes copied each way, and the CUDA /
 * library versions.  The weights are a deterministic pseudo-random bf16 fill
 * (their values do not change the decode work); the sketch is built with
 * usk_build first.  The program owns every buffer (the library allocates none).
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <time.h>

#include <cuda_runtime.h>

#include "usk.h"

#define CK(call)                                                                  \
  do {                                                                            \
    cudaError_t e_ = (call);                                                      \
    if (e_ != cudaSuccess) {                                                      \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #call, cudaGetErrorString(e_)); \
      return 2;                                                                   \
    }                                                                             \
  } while (0)

#define UK(call)                                                                  \
  do {                                                                            \
    usk_status s_ = (call);                                                       \
    if (s_ != USK_OK) {                                                           \
      fprintf(stderr, "%s:%d %s: %s\n", __FILE__, __LINE__, #call, usk_status_str(s_)); \
      return 3;                                                                   \
    }                                                                             \
  } while (0)

static double now_s(void) {
  struct timespec t;
  clock_gettime(CLOCK_MONOTONIC, &t);
  return (double)t.tv_sec + 1e-9 * (double)t.tv_nsec;
}

/* float -> bf16 bits, round to nearest even (finite inputs only) */
static uint16_t bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

/* xorshift64*: a deterministic fill, uniform in [-a, a) */
static float next_uniform(uint64_t* s, float a) {
  *s ^= *s >> 12;
  *s ^= *s << 25;
  *s ^= *s >> 27;
  uint64_t r = *s * 0x2545F4914F6CDD1Dull;
  return a * (2.0f * (float)((double)(r >> 11) * (1.0 / 9007199254740992.0)) - 1.0f);
}

int main(int argc, char** argv) {
  if (argc < 5) {
    fprintf(stderr, "usage: %s M K batch iters [warmup]\n", argv[0]);
    return 1;
  }
  const int64_t M = atoll(argv[1]), K = atoll(argv[2]), batch = atoll(argv[3]);
  const int iters = atoi(argv[4]), warmup = argc > 5 ? atoi(argv[5]) : 20;
  if (M <= 0 || K <= 0 || batch < 1 || batch > USK_GEMV_MAX_BATCH || iters < 1 || warmup < 0) {
    fprintf(stderr, "bad arguments\n");
    return 1;
  }
  size_t code_bytes = 0, scale_bytes = 0;
  UK(usk_sizes(M, K, &code_bytes, &scale_bytes));

  uint16_t* hW = (uint16_t*)malloc((size_t)(M * K) * 2);
  if (!hW) return 2;
  uint64_t st = 0x9E3779B97F4A7C15ull;
  for (int64_t q = 0; q < M * K; ++q) hW[q] = bf16_bits(next_uniform(&st, 0.05f));

  void *dW = NULL, *dx = NULL;
  int8_t* dcodes = NULL;
  uint16_t* dscales = NULL;
  float* dy = NULL;
  uint32_t* dstatus = NULL;
  CK(cudaMalloc(&dW, (size_t)(M * K) * 2));
  CK(cudaMalloc((void**)&dcodes, code_bytes));
  CK(cudaMalloc((void**)&dscales, scale_bytes));
  CK(cudaMalloc(&dx, (size_t)(batch * K) * 2));
  CK(cudaMalloc((void**)&dy, (size_t)(batch * M) * 4));
  CK(cudaMalloc((void**)&dstatus, 4));
  CK(cudaMemset(dstatus, 0, 4));
  CK(cudaMemcpy(dW, hW, (size_t)(M * K) * 2, cudaMemcpyHostToDevice));
  free(hW);

  cudaStream_t s;
  CK(cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking));
  usk_params p;
  memset(&p, 0, sizeof(p));
  p.version = USK_FORMAT_MAXKEY;
  p.seed = 1;
  UK(usk_build(dW, USK_BF16, M, K, K, NULL, &p, dcodes, dscales, dstatus, s));
  CK(cudaStreamSynchronize(s));
  CK(cudaFree(dW));

  usk_sketch sk;
  memset(&sk, 0, sizeof(sk));
  sk.M = M;
  sk.K = K;
  sk.seed = 1;
  sk.codes = dcodes;
  sk.scales = dscales;
  sk.version = USK_FORMAT_MAXKEY;

  uint16_t* hx = NULL;
  float* hy = NULL;
  const size_t xb = (size_t)(batch * K) * 2, yb = (size_t)(batch * M) * 4;
  CK(cudaMallocHost((void**)&hx, xb));
  CK(cudaMallocHost((void**)&hy, yb));
  for (int64_t q = 0; q < batch * K; ++q) hx[q] = bf16_bits(next_uniform(&st, 1.0f));

  /* end to end: H2D x, product, D2H y, synchronise -- per call */
  double t0 = 0.0;
  for (int i = 0; i < warmup + iters; ++i) {
    if (i == warmup) t0 = now_s();
    CK(cudaMemcpyAsync(dx, hx, xb, cudaMemcpyHostToDevice, s));
    UK(usk_gemv(&sk, dx, USK_BF16, batch, dy, dstatus, s));
    CK(cudaMemcpyAsync(hy, dy, yb, cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
  }
  const double e2e = (now_s() - t0) / iters;

  /* device time of back-to-back calls (no copies), for comparison */
  cudaEvent_t e0, e1;
  CK(cudaEventCreate(&e0));
  CK(cudaEventCreate(&e1));
  CK(cudaEventRecord(e0, s));
  for (int i = 0; i < iters; ++i) UK(usk_gemv(&sk, dx, USK_BF16, batch, dy, dstatus, s));
  CK(cudaEventRecord(e1, s));
  CK(cudaEventSynchronize(e1));
  float ms = 0.0f;
  CK(cudaEventElapsedTime(&ms, e0, e1));

  uint32_t flags = 0;
  CK(cudaMemcpy(&flags, dstatus, 4, cudaMemcpyDeviceToHost));
  if (flags) {
    fprintf(stderr, "device flags %#x\n", flags);
    return 4;
  }
  int rt = 0, drv = 0;
  cudaRuntimeGetVersion(&rt);
  cudaDriverGetVersion(&drv);
  printf("{\"M\": %lld, \"K\": %lld, \"batch\": %lld, \"iters\": %d, \"e2e_us\": %.4f, \"kernel_loop_us\": %.4f, "
         "\"h2d_bytes\": %zu, \"d2h_bytes\": %zu, \"cuda_runtime\": %d, \"cuda_driver\": %d, \"format\": %u}\n",
         (long long)M, (long long)K, (long long)batch, iters, e2e * 1e6, 1e3 * (double)ms / iters, xb, yb, rt, drv,
         usk_format_version());
  cudaFreeHost(hx);
  cudaFreeHost(hy);
  cudaFree(dcodes);
  cudaFree(dscales);
  cudaFree(dx);
  cudaFree(dy);
  cudaFree(dstatus);
  cudaStreamDestroy(s);
  return 0;
}
