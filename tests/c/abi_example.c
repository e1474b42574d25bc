/*
 * The C ABI used from plain C99: no Python, no torch.
 *
 * Eight virtual ranks hold x_p[i] = ((7p + i) mod 17) - 8, integers that every
 * element type carries exactly, so every rank's output must equal the exact
 * integer sum over ranks (|sum| <= 64). The program copies the inputs from host
 * memory, runs every all-reduce algorithm, the reduce-scatter and the
 * all-gather in bf16, fp16 and fp32 on the default stream, copies the outputs
 * back and compares them with the sums computed here. It prints "ok" and exits
 * 0, or names the first mismatch and exits 1; it exits 2 when no CUDA device
 * is present.
 *
 * Build (the tests do this): cc -std=c99 -I include -I <cuda>/include
 *   abi_example.c -L <lib dir> -lvrar -L <cuda>/lib64 -lcudart
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "vrar.h"

#define P 8
#define N 100003 /* ragged: not a multiple of any vector width */

static int value(int p, size_t i) { return (int)((7u * (unsigned)p + (unsigned)(i % 17u)) % 17u) - 8; }

static uint32_t f32_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  return u;
}

/* Small integers are exact in every type: bf16 keeps the top 16 bits of the
 * binary32 pattern; binary16 has a 10-bit fraction (|k| <= 64 needs 6 bits). */
static uint16_t int_to_bf16(int k) { return (uint16_t)(f32_bits((float)k) >> 16); }

static uint16_t int_to_f16(int k) {
  if (k == 0) return 0;
  uint16_t sign = k < 0 ? 0x8000u : 0u;
  unsigned a = (unsigned)(k < 0 ? -k : k);
  int e = 0;
  while ((a >> (e + 1)) != 0) ++e; /* a in [2^e, 2^(e+1)) */
  unsigned frac = (a << (10 - e)) & 0x3FFu;
  return (uint16_t)(sign | (unsigned)((e + 15) << 10) | frac);
}

static size_t esize(vrar_dtype_t dt) { return dt == VRAR_FP32 ? 4 : 2; }

static void encode(vrar_dtype_t dt, int k, void* dst, size_t i) {
  if (dt == VRAR_FP32) ((float*)dst)[i] = (float)k;
  else if (dt == VRAR_BF16) ((uint16_t*)dst)[i] = int_to_bf16(k);
  else ((uint16_t*)dst)[i] = int_to_f16(k);
}

static int same(vrar_dtype_t dt, const void* got, size_t i, int k) {
  if (dt == VRAR_FP32) return f32_bits(((const float*)got)[i]) == f32_bits((float)k);
  return ((const uint16_t*)got)[i] == (dt == VRAR_BF16 ? int_to_bf16(k) : int_to_f16(k));
}

static int check_cuda(cudaError_t e, const char* what) {
  if (e != cudaSuccess) {
    fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    return 0;
  }
  return 1;
}

static int sum_at(size_t i) {
  int s = 0;
  for (int p = 0; p < P; ++p) s += value(p, i);
  return s;
}

/* One all-reduce with algorithm `algo` (VRAR_ALGO_*), or the reduce-scatter
 * (kind 1) or all-gather (kind 2), checked element by element on every rank. */
static int run(vrar_dtype_t dt, int kind, vrar_algo_t algo) {
  const size_t es = esize(dt);
  const size_t n = kind == 0 ? N : (size_t)N - (size_t)N % P; /* RS / AG need n % P == 0 */
  const size_t m = n / P;
  const size_t in_len = kind == 2 ? m : n, out_len = kind == 1 ? m : n;
  void* host = malloc(n * es);
  void* din[P];
  void* dout[P];
  int ok = host != NULL;
  memset(din, 0, sizeof din);
  memset(dout, 0, sizeof dout);
  for (int p = 0; ok && p < P; ++p) {
    ok = check_cuda(cudaMalloc(&din[p], in_len * es), "cudaMalloc") &&
         check_cuda(cudaMalloc(&dout[p], out_len * es), "cudaMalloc");
    /* All-gather: rank p's slice holds the values of chunk p of the vector. */
    for (size_t i = 0; ok && i < in_len; ++i) encode(dt, value(p, kind == 2 ? (size_t)p * m + i : i), host, i);
    ok = ok && check_cuda(cudaMemcpy(din[p], host, in_len * es, cudaMemcpyHostToDevice), "H2D");
  }
  int rc = VRAR_OK;
  if (ok) {
    if (kind == 0) rc = vrar_allreduce((const void* const*)din, dout, P, n, dt, algo, NULL);
    else if (kind == 1) rc = vrar_reduce_scatter((const void* const*)din, dout, P, n, dt, NULL);
    else rc = vrar_all_gather((const void* const*)din, dout, P, n, dt, NULL);
    if (rc != VRAR_OK) {
      fprintf(stderr, "call failed: %s\n", vrar_strerror(rc));
      ok = 0;
    }
  }
  uint32_t info[4];
  if (ok && (rc = vrar_query_status(NULL, info)) != VRAR_OK) {
    fprintf(stderr, "device status: %s\n", vrar_strerror(rc));
    ok = 0;
  }
  for (int p = 0; ok && p < P; ++p) {
    ok = check_cuda(cudaMemcpy(host, dout[p], out_len * es, cudaMemcpyDeviceToHost), "D2H");
    for (size_t i = 0; ok && i < out_len; ++i) {
      const size_t g = kind == 1 ? (size_t)p * m + i : i; /* element of the full vector */
      const int want = kind == 2 ? value((int)(g / m), g) : sum_at(g);
      if (!same(dt, host, i, want)) {
        fprintf(stderr, "mismatch: dtype %d kind %d algo %d rank %d element %zu (want %d)\n", (int)dt, kind,
                (int)algo, p, i, want);
        ok = 0;
      }
    }
  }
  for (int p = 0; p < P; ++p) {
    cudaFree(din[p]);
    cudaFree(dout[p]);
  }
  free(host);
  return ok;
}

int main(void) {
  int count = 0;
  if (cudaGetDeviceCount(&count) != cudaSuccess || count < 1) {
    fprintf(stderr, "no CUDA device\n");
    return 2;
  }
  if (vrar_version() < 1) return 1;
  const vrar_dtype_t dts[3] = {VRAR_BF16, VRAR_FP16, VRAR_FP32};
  const vrar_algo_t algos[6] = {VRAR_ALGO_AUTO, VRAR_ALGO_ONESHOT, VRAR_ALGO_TWOSTAGE, VRAR_ALGO_TWOSTAGE_WRITE,
                                VRAR_ALGO_RD, VRAR_ALGO_HIER};
  if (vrar_set_group_size(4) != VRAR_OK) return 1; /* HIER: 2 groups of 4 */
  for (int d = 0; d < 3; ++d) {
    for (int a = 0; a < 6; ++a) {
      if (!run(dts[d], 0, algos[a])) return 1;
      printf("%s ok\n", vrar_kernel_name(P, N, dts[d], algos[a]));
    }
    if (!run(dts[d], 1, VRAR_ALGO_AUTO) || !run(dts[d], 2, VRAR_ALGO_AUTO)) return 1;
  }
  printf("ok\n");
  return 0;
}
