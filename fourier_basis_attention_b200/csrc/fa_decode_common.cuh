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

// bf16 x 8 -> 4 fp32 pairs (element 2i in .x, 2i + 1 in .y) for paired FMAs.
__device__ __forceinline__ void bf16x8_to_f32x2(const uint4 v, float2 (&x)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i)
    x[i] = make_float2(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}

// Sink / recent rows of one KV head, rows [fs * FT, fs * FT + FT) of its S + R exact rows
// (all 128 dims): scores, softmax statistics and values of the G query heads, written as
// split record n_splits + fs. All DNT threads of the CTA take part; `sm` holds
// sink_recent_smem_bytes() bytes. Run as extra CTAs of the CUDA-core split kernel, or of the
// prologue launch on the tensor-core and warp-MMA paths.
// NJ: query heads per block of the score and value passes (1, 2 or 4: G for G < 4), so that
// MHA and G = 2 plans do no arithmetic or shuffles for empty heads.
static_assert(HL == 8 && DNT == FT, "sink / recent pass: 8 heads per score row, one thread per row");

template <int NJ>
__device__ __forceinline__ void decode_sink_recent_t(const DecodeParams& p, float* sm, int fid) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int kvh = fid / p.n_fsplits, fs = fid - (fid / p.n_fsplits) * p.n_fsplits;
  const int b = kvh / p.Hkv, g = kvh - (kvh / p.Hkv) * p.Hkv;
  const int r0 = fs * FT, nr = min(FT, p.nF - r0);
  const int G = p.G;
  float* qs = sm;                       // [HL][128]
  float* sc = qs + HL * FA_HEAD_DIM;    // [FT][HL]
  float* mxs = sc + FT * HL;            // [8][HL]
  float* mh = mxs + 8 * HL;             // [HL]
  float* red = mh + HL;                 // [8 warps][16 chunks][4 heads][8]

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
  // scores: warp-cooperative, two rows per load instruction (lanes 0-15 and 16-31, one
  // 16-byte chunk each); each lane keeps its chunk of q for up to 4 query heads in
  // registers. A warp takes U = 16 / NJ row pairs at a time (all loads in flight), so each
  // lane holds 16 partial dot products (row pair u, head j); one reduce-scatter over the 16
  // lanes of each half-warp (15 shuffles) leaves lane c with the score of partial c, which
  // it writes to sc[row][head].
  {
    constexpr int U = 16 / NJ;
    const int ch = lane & 15, half = lane >> 4;
    const int npair = (nr + 1) >> 1;
    for (int hb = 0; hb < G; hb += NJ) {
      float2 qr[NJ][4];  // q pairs (dims 2e, 2e + 1 of the chunk)
#pragma unroll
      for (int j = 0; j < NJ; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          qr[j][e] = (hb + j < G)
                         ? *reinterpret_cast<const float2*>(qs + (hb + j) * FA_HEAD_DIM + ch * 8 + 2 * e)
                         : make_float2(0.0f, 0.0f);
      for (int i0 = warp; i0 < npair; i0 += 8 * U) {
        uint4 xr[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int row = 2 * (i0 + 8 * u) + half;
          xr[u] = row < nr ? *reinterpret_cast<const uint4*>(FKh + (long long)(r0 + row) * FA_HEAD_DIM + ch * 8)
                           : make_uint4(0, 0, 0, 0);
        }
        float v[16];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float2 x[4];
          bf16x8_to_f32x2(xr[u], x);
#pragma unroll
          for (int j = 0; j < NJ; ++j) {
            float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int e = 0; e < 4; ++e) a = __ffma2_rn(qr[j][e], x[e], a);
            v[u * NJ + j] = a.x + a.y;
          }
        }
        // reduce-scatter: at offset o the lanes with bit o set keep the upper half of the
        // remaining partials, the others the lower half, each adding its partner's copy
#pragma unroll
        for (int o = 8; o >= 1; o >>= 1) {
          const bool up = (ch & o) != 0;
#pragma unroll
          for (int t = 0; t < o; ++t) {
            const float send = up ? v[t] : v[t + o];
            const float keep = up ? v[t + o] : v[t];
            v[t] = keep + __shfl_xor_sync(0xffffffffu, send, o);
          }
        }
        const int u = ch / NJ, j = ch - (ch / NJ) * NJ;
        const int row = 2 * (i0 + 8 * u) + half;
        if (row < nr && hb + j < G) sc[row * HL + hb + j] = v[0];
      }
    }
  }
  __syncthreads();
  // row tid's scores (HL = 8 floats, two vector loads); absent rows and heads: -inf
  float s[HL];
  {
    const float4 lo = tid < nr ? *reinterpret_cast<const float4*>(sc + tid * HL) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 hi = (tid < nr && G > 4) ? *reinterpret_cast<const float4*>(sc + tid * HL + 4)
                                          : make_float4(0.f, 0.f, 0.f, 0.f);
    s[0] = lo.x; s[1] = lo.y; s[2] = lo.z; s[3] = lo.w;
    s[4] = hi.x; s[5] = hi.y; s[6] = hi.z; s[7] = hi.w;
  }
#pragma unroll
  for (int h = 0; h < HL; ++h)
    if (tid >= nr || h >= G) s[h] = -INFINITY;
#pragma unroll
  for (int h = 0; h < HL; ++h) {
    if (h >= G) break;  // uniform over the CTA
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
  for (int h = 0; h < HL; ++h) l[h] = (h < G && tid < nr) ? exp2f(s[h] - mh[h]) : 0.0f;
  if (tid < FT) {  // p of row tid (0 past the rows and heads), two vector stores
    *reinterpret_cast<float4*>(sc + tid * HL) = make_float4(l[0], l[1], l[2], l[3]);
    *reinterpret_cast<float4*>(sc + tid * HL + 4) = make_float4(l[4], l[5], l[6], l[7]);
  }
  __syncthreads();
#pragma unroll
  for (int h = 0; h < HL; ++h) {
    if (h >= G) break;  // uniform over the CTA
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) l[h] += __shfl_xor_sync(0xffffffffu, l[h], o);
    if (lane == 0) mxs[warp * HL + h] = l[h];
  }
  // values: thread = (16-byte chunk c of a row, row group grp): lanes 0-15 and 16-31 of a warp
  // read two whole rows per load, and each V row is read once for all G query heads (in
  // blocks of up to 4 heads). The two row groups of a warp are added by a shuffle, the 8
  // warps' partials in a fixed order through shared memory.
  const long long bhq = (long long)p.B * p.Hq;
  const int rix = p.n_splits + fs;
  const int c = tid & 15, grp = tid >> 4;
  constexpr int NGRP = DNT / 16;
  for (int hb = 0; hb < G; hb += NJ) {
    float2 acc[NJ][4];  // dims 2e, 2e + 1 of the chunk, per head of the block
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = make_float2(0.0f, 0.0f);
#pragma unroll 4  // independent row loads in flight
    for (int rr = grp; rr < nr; rr += NGRP) {
      float2 x[4];
      bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(FVh + (long long)(r0 + rr) * FA_HEAD_DIM + c * 8), x);
      // p of the block's heads for this row, one vector load (sc rows are HL = 8 floats,
      // hb a multiple of NJ: aligned; heads past G hold 0)
      float pj[NJ];
      if constexpr (NJ == 4) {
        const float4 t = *reinterpret_cast<const float4*>(sc + rr * HL + hb);
        pj[0] = t.x;
        pj[1] = t.y;
        pj[2] = t.z;
        pj[3] = t.w;
      } else if constexpr (NJ == 2) {
        const float2 t = *reinterpret_cast<const float2*>(sc + rr * HL + hb);
        pj[0] = t.x;
        pj[1] = t.y;
      } else {
        pj[0] = sc[rr * HL + hb];
      }
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        if (hb + j < G) {
          const float pv = pj[j];
          const float2 pv2 = make_float2(pv, pv);
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[j][e] = __ffma2_rn(pv2, x[e], acc[j][e]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < NJ; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[j][e].x += __shfl_xor_sync(0xffffffffu, acc[j][e].x, 16);
        acc[j][e].y += __shfl_xor_sync(0xffffffffu, acc[j][e].y, 16);
      }
    if (lane < 16) {
      float4* dst = reinterpret_cast<float4*>(red + (warp * 16 + lane) * 32);
#pragma unroll
      for (int j = 0; j < NJ; ++j) {
        dst[2 * j] = make_float4(acc[j][0].x, acc[j][0].y, acc[j][1].x, acc[j][1].y);
        dst[2 * j + 1] = make_float4(acc[j][2].x, acc[j][2].y, acc[j][3].x, acc[j][3].y);
      }
    }
    __syncthreads();
    const int nh = min(NJ, G - hb);
    for (int o = tid; o < 16 * nh * 8; o += DNT) {
      const int c2 = o / (nh * 8), j = (o / 8) % nh, e = o % 8;
      float v = 0.0f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += red[(w * 16 + c2) * 32 + j * 8 + e];
      p.rec[((long long)rix * bhq + (long long)b * p.Hq + g * G + hb + j) * p.rec_stride + 4 +
            c2 * 8 + e] = v;
    }
    __syncthreads();  // red is rewritten by the next head block
  }
  if (tid < G) {  // the warps' sums of p (mxs) are visible after the barriers above
    float ls = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) ls += mxs[w * HL + tid];
    float* rec = p.rec + ((long long)rix * bhq + (long long)b * p.Hq + g * G + tid) * p.rec_stride;
    rec[0] = mh[tid];
    rec[1] = ls;
  }
}

__device__ __forceinline__ void decode_sink_recent(const DecodeParams& p, float* sm, int fid) {
  if (p.G == 1)
    decode_sink_recent_t<1>(p, sm, fid);
  else if (p.G == 2)
    decode_sink_recent_t<2>(p, sm, fid);
  else
    decode_sink_recent_t<4>(p, sm, fid);
}

__host__ __device__ constexpr size_t sink_recent_smem_bytes() {
  return (size_t)(HL * FA_HEAD_DIM + FT * HL + 8 * HL + HL + 8 * 16 * 32) * 4;
}

// Warp-MMA split kernel over per-KV-head E blocks, F2 = 512 or 1024 slots.
cudaError_t launch_decode_hmma(const DecodeParams& p, int F2, cudaStream_t stream);
size_t decode_hmma_smem_bytes(int F2);

// Tensor-core split kernel over token-major E with de_slot = 0, 8, 16 or 32 retained
// elements per KV head and token.

cudaError_t launch_decode_tc(const DecodeParams& p, int de_slot, cudaStream_t stream);

// Cluster tensor-core split kernel (fa_decode_cl.cu): per-KV-head E blocks, coefficient
// slots split over a cluster of C CTAs (C = 1, 2 or 4).
cudaError_t launch_decode_cl(const DecodeParams& p, cudaStream_t stream);
size_t decode_tc_smem_bytes(int F2, int de_slot, int G);

}  // namespace fa
