// fa_sensitivity.cu -- head-dimension sensitivity scores ([skill] Step 1: noise is added to
// one value dim at a time and the change of the attention output is measured).
//
// Only the values are perturbed, so the attention weights P stay the same and the output
// change of dim d is NOISE_SCALE * P n_d, n_d being the noise column of dim d. One exact
// attention pass over the keys with the noise in place of the values therefore gives every
// dim's change at once: it runs on the decode kernels with an all-exact plan (every token a
// sink row, F = the caller's K and noise buffers, no copy), and a small kernel reduces each
// dim's column to its norm over the batch rows and the query heads of each KV head.
#include <string.h>

#include "fa_host.h"
#include "fa_internal.cuh"

namespace fa {

// scores[g][d] = NOISE_SCALE * || out[b][g G + i][d] ||_2 over b < B, i < G.
__global__ void __launch_bounds__(FA_HEAD_DIM) sensitivity_norm_kernel(const float* __restrict__ out,
                                                                      float* __restrict__ scores,
                                                                      int B, int Hq, int G) {
  const int g = blockIdx.x, d = threadIdx.x;
  float acc = 0.0f;
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < G; ++i) {
      const float v = out[((long long)b * Hq + (long long)g * G + i) * FA_HEAD_DIM + d];
      acc = fmaf(v, v, acc);
    }
  scores[g * FA_HEAD_DIM + d] = FA_NOISE_SCALE * sqrtf(acc);
}

// The all-exact plan: every token is a sink row, nothing compressed (M = 0).
// Returns an fa_status code (fa_plan_init's, with its message).
int sensitivity_plan(const fa_shape* shape, fa_plan* plan) {
  fa_shape s = *shape;
  s.S = s.L;
  s.R = 0;
  s.k = 1;
  static const uint8_t zeros[FA_MAX_KV_HEADS * FA_HEAD_DIM] = {};
  return fa_plan_init(&s, zeros, plan);
}

size_t sensitivity_out_offset(const DecodeConfig& c) {
  return (c.qw_bytes + c.rec_bytes + 255) & ~size_t(255);
}

cudaError_t launch_sensitivity(const fa_plan* plan, const DecodeConfig& c, const void* q,
                               const void* K, const void* noise, float* scores, void* workspace,
                               cudaStream_t stream) {
  fa_cache cache;
  memset(&cache, 0, sizeof(cache));
  cache.F_K = const_cast<void*>(K);
  cache.F_V = const_cast<void*>(noise);
  float* out = reinterpret_cast<float*>(static_cast<char*>(workspace) + sensitivity_out_offset(c));
  cudaError_t e = launch_decode(plan, c, q, &cache, out, FA_F32, workspace, stream);
  if (e != cudaSuccess) return e;
  const fa_shape& sh = plan->shape;
  sensitivity_norm_kernel<<<sh.Hkv, FA_HEAD_DIM, 0, stream>>>(out, scores, sh.B, sh.Hq, plan->G);
  return cudaGetLastError();
}

}  // namespace fa
