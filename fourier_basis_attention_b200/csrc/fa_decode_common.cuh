// fa_decode_common.cuh -- parameters and helpers shared by the decode kernels
// (fa_decode.cu: prologue, CUDA-core split kernel, sink/recent, combine; fa_decode_tc.cu:
// tensor-core split kernel; fa_decode_hmma.cu: warp-MMA split kernel).
#pragma once

#include "fa_host.h"
#include "fa_internal.cuh"

namespace fa {

constexpr int DT = 64;    // tokens per tile
constexpr int DNT = 256;  // threads per CTA
constexpr int HL = 8;     // query heads per CTA (zero-padded)
constexpr int FT = 256;   // sink/recent rows per CTA

struct DecodeParams {
  int B, Hq, Hkv, G, M, P, k, F, F_pad, nF;  // M middle tokens, P basis period
  int n_splits, split_len, n_fsplits, NKV, n_mid, n_rec;
  int rec_stride, qw_stride;
  int NTU, TG, DEC, TGE;
  int tc_F2, tc_tmem_cols;  // tensor-core split kernel: coefficient slots, TMEM columns
  int e_row;                // token-major E: elements per token row of a batch
  int n_pro;                // prologue CTAs (the sink / recent CTAs of a prologue launch follow)
  int cl_C, cl_SL, cl_TB, cl_stages, cl_slot_bytes, cl_tmem_cols;  // cluster tensor-core kernel
  float qscale, norm_single, norm_pair, two_over_P;
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

// cos / sin of 2 pi r / P for an exactly reduced integer phase 0 <= r < P.
__device__ __forceinline__ void phase_sincos(long long r, int P, float two_over_P, float* s,
                                             float* c) {
  const long long rr = (2 * r > P) ? r - P : r;  // (-P/2, P/2]
  sincospif((float)rr * two_over_P, s, c);
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float (&x)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Sink / recent rows of one KV head, rows [fs * FT, fs * FT + FT) of its S + R exact rows
// (all 128 dims): scores, softmax statistics and values of the G query heads, written as
// split record n_splits + fs. All DNT threads of the CTA take part; `sm` holds
// sink_recent_smem_bytes() bytes. Run as extra CTAs of the CUDA-core split kernel, or of the
// prologue launch on the tensor-core and warp-MMA paths.
__device__ __forceinline__ void decode_sink_recent(const DecodeParams& p, float* sm, int fid) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = fid / p.n_fsplits, fs = fid - (fid / p.n_fsplits) * p.n_fsplits;
  const int b = kvh / p.Hkv, g = kvh - (kvh / p.Hkv) * p.Hkv;
  const int r0 = fs * FT, nr = min(FT, p.nF - r0);
  const int G = p.G;
  float* qs = sm;                       // [HL][128]
  float* sc = qs + HL * FA_HEAD_DIM;    // [FT][HL]
  float* mxs = sc + FT * HL;            // [8][HL]
  float* mh = mxs + 8 * HL;             // [HL]
  float* red = mh + HL;                 // [DNT][8]

  const __nv_bfloat16* FKh = p.FK + (long long)kvh * p.nF * FA_HEAD_DIM;
  const __nv_bfloat16* FVh = p.FV + (long long)kvh * p.nF * FA_HEAD_DIM;
  if (tid == 0) {  // this CTA's rows of both tensors into L2 while q is staged
    prefetch_l2_bulk(FKh + (long long)r0 * FA_HEAD_DIM, (uint32_t)(nr * FA_HEAD_DIM * 2));
    prefetch_l2_bulk(FVh + (long long)r0 * FA_HEAD_DIM, (uint32_t)(nr * FA_HEAD_DIM * 2));
  }
  for (int idx = tid; idx < HL * FA_HEAD_DIM; idx += DNT) {
    const int h = idx >> 7, d = idx & 127;
    qs[idx] = (h < G) ? __bfloat162float(p.q[((long long)b * p.Hq + g * G + h) * FA_HEAD_DIM + d]) *
                            p.qscale
                      : 0.0f;
  }
  __syncthreads();
  float s[HL];
#pragma unroll
  for (int h = 0; h < HL; ++h) s[h] = 0.0f;
  if (tid < nr) {
    const __nv_bfloat16* row = FKh + (long long)(r0 + tid) * FA_HEAD_DIM;
    for (int c = 0; c < FA_HEAD_DIM; c += 8) {
      float x[8];
      bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + c), x);
#pragma unroll
      for (int h = 0; h < HL; ++h) {
        if (h < G) {
          const float4 qa = *reinterpret_cast<const float4*>(qs + h * FA_HEAD_DIM + c);
          const float4 qb = *reinterpret_cast<const float4*>(qs + h * FA_HEAD_DIM + c + 4);
          s[h] += qa.x * x[0] + qa.y * x[1] + qa.z * x[2] + qa.w * x[3] + qb.x * x[4] +
                  qb.y * x[5] + qb.z * x[6] + qb.w * x[7];
        }
      }
    }
  }
#pragma unroll
  for (int h = 0; h < HL; ++h)
    if (tid >= nr || h >= G) s[h] = -INFINITY;
#pragma unroll
  for (int h = 0; h < HL; ++h) {
    float m = s[h];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) mxs[warp * HL + h] = m;
  }
  __syncthreads();
  if (tid < HL) {
    float m = mxs[tid];
#pragma unroll
    for (int w = 1; w < 8; ++w) m = fmaxf(m, mxs[w * HL + tid]);
    mh[tid] = m;
  }
  __syncthreads();
  float l[HL];
#pragma unroll
  for (int h = 0; h < HL; ++h) {
    const float pv = (h < G && tid < nr) ? exp2f(s[h] - mh[h]) : 0.0f;
    sc[tid * HL + h] = pv;
    l[h] = pv;
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < HL; ++h) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
    if (lane == 0) mxs[warp * HL + h] = l[h];
  }
  // values: item (head h, 8-dim chunk c), token group grp
  const int items = G * 16;
  const int it = tid % items, grp = tid / items, ngrp = DNT / items;
  const int h = it >> 4, c = it & 15;
  float acc[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
#pragma unroll 8  // independent row loads in flight
  for (int rr = grp; rr < nr; rr += ngrp) {
    const float pv = sc[rr * HL + h];
    float x[8];
    bf16x8_to_f32(*reinterpret_cast<const uint4*>(FVh + (long long)(r0 + rr) * FA_HEAD_DIM + c * 8), x);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] += pv * x[e];
  }
  {
    float4* dst = reinterpret_cast<float4*>(red + tid * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  __syncthreads();
  const long long bhq = (long long)p.B * p.Hq;
  const int rix = p.n_splits + fs;
  if (tid < G) {
    float ls = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) ls += mxs[w * HL + tid];
    float* rec = p.rec + ((long long)rix * bhq + (long long)b * p.Hq + g * G + tid) * p.rec_stride;
    rec[0] = mh[tid];
    rec[1] = ls;
  }
  if (grp == 0) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
    for (int q2 = 0; q2 < ngrp; ++q2) {
      const float* src = red + (q2 * items + it) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] += src[e];
    }
    float* rec = p.rec + ((long long)rix * bhq + (long long)b * p.Hq + g * G + h) * p.rec_stride +
                 4 + c * 8;
    reinterpret_cast<float4*>(rec)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(rec)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

__host__ __device__ constexpr size_t sink_recent_smem_bytes() {
  return (size_t)(HL * FA_HEAD_DIM + FT * HL + 8 * HL + HL + DNT * 8) * 4;
}

// Warp-MMA split kernel over per-KV-head E blocks, F2 = 512 or 1024 slots.
cudaError_t launch_decode_hmma(const DecodeParams& p, int F2, cudaStream_t stream);
size_t decode_hmma_smem_bytes(int F2);

// Tensor-core split kernel over token-major E with de_slot = 0, 8, 16 or 32 retained
// elements per KV head and token.
// bf16 x 8 -> 4 fp32 pairs (element 2i in .x, 2i + 1 in .y) for paired FMAs.
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4 v, float2 (&x)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

cudaError_t launch_decode_tc(const DecodeParams& p, int de_slot, cudaStream_t stream);

// Cluster tensor-core split kernel (fa_decode_cl.cu): per-KV-head E blocks, coefficient
// slots split over a cluster of C CTAs (C = 1, 2 or 4).
cudaError_t launch_decode_cl(const DecodeParams& p, cudaStream_t stream);
size_t decode_tc_smem_bytes(int F2, int de_slot, int G);

}  // namespace fa
