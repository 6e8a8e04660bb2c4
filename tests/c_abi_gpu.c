/* The C ABI used from plain C on the GPU (no C++, no torch): fa_build_basis, fa_compress and
 * fa_decode on device buffers from the CUDA runtime, checked against the fp64 oracle's
 * values stored in tests/golden/c_abi_gpu_case.txt (written by
 * tests/golden/make_c_abi_gpu_case.py, which calls only the oracle).
 *
 * Inputs come from SplitMix64 (Steele, Lea and Flood, OOPSLA 2014; 64-bit finaliser as in
 * Vigna's splitmix64.c), written here from that definition: element i of a tensor is the
 * signed top byte of output i (state seed + (i + 1) * gamma, then the finaliser) divided
 * by 64, a value bf16 holds exactly.
 *
 * Usage: c_abi_gpu <golden file>. Prints "ok" and exits 0 when every check holds. Built and
 * run by tests/test_gpu_c_program.py. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "fourier_attention.h"

#define CHECK(c)                                                        \
  do {                                                                  \
    if (!(c)) {                                                         \
      printf("check failed at line %d: %s (%s)\n", __LINE__, #c, fa_last_error()); \
      return 1;                                                         \
    }                                                                   \
  } while (0)
#define CUDA(c) CHECK((c) == cudaSuccess)

static const double TOL = 3e-3; /* max |err| <= TOL * max |ref|, as in the parity tests */

static uint64_t splitmix64_at(uint64_t seed, uint64_t i) {
  uint64_t z = seed + (i + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* bf16 bits of element i: the value is exact in bf16, so the bits are the top half of the
 * float's */
static uint16_t grid_bf16(uint64_t seed, uint64_t i) {
  const int v = (int)(int8_t)(uint8_t)(splitmix64_at(seed, i) >> 56);
  const float f = (float)v / 64.0f;
  uint32_t u;
  memcpy(&u, &f, 4);
  return (uint16_t)(u >> 16);
}

static uint16_t* draw(uint64_t seed, size_t n) {
  uint16_t* h = (uint16_t*)malloc(n * sizeof(uint16_t));
  for (size_t i = 0; i < n; ++i) h[i] = grid_bf16(seed, i);
  return h;
}

/* reads "count" doubles following a header line that starts with tag */
static int read_block(FILE* f, const char* tag, double* dst, int count) {
  char line[256];
  while (fgets(line, sizeof line, f))
    if (strncmp(line, tag, strlen(tag)) == 0) {
      for (int i = 0; i < count; ++i)
        if (fscanf(f, "%lf", &dst[i]) != 1) return 0;
      return 1;
    }
  return 0;
}

static int close_enough(const char* what, const double* ref, const float* got, int n) {
  double err = 0, scale = 0;
  for (int i = 0; i < n; ++i) {
    const double e = fabs((double)got[i] - ref[i]);
    err = e > err ? e : err;
    scale = fabs(ref[i]) > scale ? fabs(ref[i]) : scale;
  }
  if (!(err <= TOL * scale) || scale == 0) {
    printf("%s: max err %.3e > %.0e * %.3e\n", what, err, TOL, scale);
    return 0;
  }
  return 1;
}

int main(int argc, char** argv) {
  CHECK(argc == 2);
  FILE* gf = fopen(argv[1], "r");
  CHECK(gf != NULL);
  int B, Hq, Hkv, D, L, S, R, k;
  unsigned long long sk, sv, sq;
  char line[256];
  int have_shape = 0, have_seeds = 0;
  while ((!have_shape || !have_seeds) && fgets(line, sizeof line, gf)) {
    if (sscanf(line, "shape %d %d %d %d %d %d %d %d", &B, &Hq, &Hkv, &D, &L, &S, &R, &k) == 8)
      have_shape = 1;
    if (sscanf(line, "seeds %llu %llu %llu", &sk, &sv, &sq) == 3) have_seeds = 1;
  }
  CHECK(have_shape && have_seeds && D == 128 && Hkv == 2);

  fa_shape shape = {B, Hq, Hkv, D, L, S, R, k};
  static uint8_t mask[2 * 128];
  for (int d = 0; d < 128; ++d) {
    mask[d] = (uint8_t)(d % 4 != 0);     /* KV head 0: 96 compressed dims */
    mask[128 + d] = (uint8_t)(d < 64);   /* KV head 1: 64 compressed dims */
  }
  fa_plan plan;
  CHECK(fa_plan_init(&shape, mask, &plan) == FA_OK);
  CHECK(plan.M == L - S - R && plan.dc[0] == 96 && plan.dc[1] == 64);

  const size_t n_kv = (size_t)B * Hkv * L * D, n_q = (size_t)B * Hq * D;
  uint16_t* hK = draw(sk, n_kv);
  uint16_t* hV = draw(sv, n_kv);
  uint16_t* hq = draw(sq, n_q);

  void *dK, *dV, *dq, *dphi, *dout, *dws;
  fa_cache cache;
  CUDA(cudaMalloc(&dK, n_kv * 2));
  CUDA(cudaMalloc(&dV, n_kv * 2));
  CUDA(cudaMalloc(&dq, n_q * 2));
  CUDA(cudaMemcpy(dK, hK, n_kv * 2, cudaMemcpyHostToDevice));
  CUDA(cudaMemcpy(dV, hV, n_kv * 2, cudaMemcpyHostToDevice));
  CUDA(cudaMemcpy(dq, hq, n_q * 2, cudaMemcpyHostToDevice));
  CUDA(cudaMalloc(&cache.F_K, (size_t)plan.f_elems * 2));
  CUDA(cudaMalloc(&cache.F_V, (size_t)plan.f_elems * 2));
  CUDA(cudaMalloc(&cache.E_K, (size_t)plan.e_elems * 2 + 16));
  CUDA(cudaMalloc(&cache.E_V, (size_t)plan.e_elems * 2 + 16));
  CUDA(cudaMalloc(&cache.C_K, (size_t)plan.c_elems * 4));
  CUDA(cudaMalloc(&cache.C_V, (size_t)plan.c_elems * 4));
  CUDA(cudaMalloc(&dphi, (size_t)k * plan.phi_ld * 2));
  CUDA(cudaMalloc(&dout, n_q * 4));
  const size_t ws_bytes = fa_decode_workspace_size(&plan, 0);
  CHECK(ws_bytes > 0);
  CUDA(cudaMalloc(&dws, ws_bytes));

  /* the default stream (NULL) throughout */
  CHECK(fa_build_basis(plan.P, k, FA_BF16, 0, dphi, plan.phi_ld, NULL) == FA_OK);
  CHECK(fa_compress(&plan, dK, dV, dphi, &cache, NULL) == FA_OK);
  CHECK(fa_decode(&plan, dq, &cache, dout, FA_F32, dws, ws_bytes, 0, NULL) == FA_OK);
  CUDA(cudaDeviceSynchronize());
  CHECK(fa_device_status(NULL) == FA_OK);

  /* decode output of every query head */
  float* out = (float*)malloc(n_q * 4);
  double* ref = (double*)malloc(n_q * sizeof(double));
  CUDA(cudaMemcpy(out, dout, n_q * 4, cudaMemcpyDeviceToHost));
  CHECK(read_block(gf, "out ", ref, (int)n_q));
  CHECK(close_enough("decode output", ref, out, (int)n_q));

  /* coefficients of KV head 1 of batch row 1, compressed dims in ascending order */
  const int b = 1, g = 1, dc = plan.dc[g], dc_ld = plan.dc_ld[g];
  const size_t c_elems = (size_t)plan.c_elems;
  float* C = (float*)malloc(c_elems * 4);
  float* got = (float*)malloc((size_t)k * dc * 4);
  double* cref = (double*)malloc((size_t)k * dc * sizeof(double));
  for (int which = 0; which < 2; ++which) {
    CUDA(cudaMemcpy(C, which ? cache.C_V : cache.C_K, c_elems * 4, cudaMemcpyDeviceToHost));
    for (int j = 0; j < k; ++j)
      for (int i = 0; i < dc; ++i)
        got[j * dc + i] = C[b * plan.c_batch + plan.c_off[g] + (size_t)j * dc_ld + i];
    CHECK(read_block(gf, which ? "coef V 1 1" : "coef K 1 1", cref, k * dc));
    CHECK(close_enough(which ? "C_V" : "C_K", cref, got, k * dc));
  }
  fclose(gf);
  printf("ok\n");
  return 0;
}
