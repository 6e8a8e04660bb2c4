// fa_decode_common.cuh -- parameters and helpers shared by the decode kernels
// (fa_decode.cu: prologue, CUDA-core split kernel, sink/recent, combine; fa_decode_tc.cu:
// tensor-core split kernel).
#pragma once

#include "fa_host.h"
#include "fa_internal.cuh"

namespace fa {

constexpr int DT = 64;    // tokens per tile
constexpr int DNT = 256;  // threads per CTA
constexpr int HL = 8;     // query heads per CTA (zero-padded)
constexpr int FT = 256;   // sink/recent rows per CTA

struct DecodeParams {
  int B, Hq, Hkv, G, M, k, F, F_pad, nF;
  int n_splits, split_len, n_fsplits, NKV, n_mid, n_rec;
  int rec_stride, qw_stride;
  int NTU, TG, DEC, TGE;
  int tc_F2, tc_tmem_cols;  // tensor-core split kernel: coefficient slots, TMEM columns
  float qscale, norm_single, norm_pair, two_over_M;
  long long e_batch, c_batch;
  long long e_off[FA_MAX_KV_HEADS], c_off[FA_MAX_KV_HEADS];
  int de[FA_MAX_KV_HEADS], de_ld[FA_MAX_KV_HEADS], dc[FA_MAX_KV_HEADS], dc_ld[FA_MAX_KV_HEADS];
  unsigned char perm[FA_MAX_KV_HEADS][FA_HEAD_DIM];
  const __nv_bfloat16 *q, *FK, *FV, *EK, *EV;
  const float *CK, *CV;
  void* out;
  int out_f32;
  float* qw;
  float* rec;
};

// cos / sin of 2 pi r / M for an exactly reduced integer phase 0 <= r < M.
__device__ __forceinline__ void phase_sincos(long long r, int M, float two_over_M, float* s,
                                             float* c) {
  const long long rr = (2 * r > M) ? r - M : r;  // (-M/2, M/2]
  sincospif((float)rr * two_over_M, s, c);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

cudaError_t launch_decode_tc(const DecodeParams& p, int de_max, cudaStream_t stream);
size_t decode_tc_smem_bytes(int F2);

}  // namespace fa
