// fa_decode.cu -- one decode step over the hybrid cache, in the coefficient domain.
//
// [skill] Step 4 restores the compressed dims during decoding; here the restoration is
// folded into the attention algebra instead of materialised. For query head h of batch
// row b (KV head g = h / G) and middle token t (basis row phi(t)):
//     score_t  = sigma * ( q_e . E_K[t]  +  phi(t) . w ),     w = C_K^T q_c   (k values)
//     out_c    = (Phi^T p) C_V  = u C_V,                      u = sum_t p_t phi(t)
//     out_e    = sum_t p_t E_V[t]
// and sink / recent tokens use all 128 dims exactly. By associativity this equals softmax
// attention over the reconstruction Phi C ([skill] Step 4), which the oracle computes.
//
// Three launches on the caller's stream:
//   prologue  per KV head: q_c / q_e gathered by the dim mask, w = C_K^T q_c, with the
//             softmax scale, log2(e) and the basis normalisation folded in. On the
//             tensor-core and warp-MMA paths the same launch runs the sink / recent rows.
//   split     the middle span, split-L: the tensor-core kernel (fa_decode_tc.cu, token-major
//             E, k <= 255), the warp-MMA kernel (fa_decode_hmma.cu, 256 <= k <= 1023) or the
//             CUDA-core kernel below: CTA (head set, split) streams its token range of
//             E_K / E_V in tiles of 64 tokens for 8 query heads at once, regenerating
//             cos/sin of the basis by a rotation recurrence (re-seeded from sincospif of the
//             exactly reduced phase), with an fp32 online softmax; its extra CTAs do the
//             sink / recent rows. Every CTA writes a partial record (running max, running
//             sum, value accumulator, u).
//   combine   per (KV head, group of its query heads): merges the records, out_c = u C_V,
//             scatters the dims back, normalises and stores fp32 or bf16.
#include "fa_decode_common.cuh"

namespace fa {

// ------------------------------------------------------------------------- prologue
// CTAs [0, n_pro): the prologue of one KV head each. CTAs past n_pro (tensor-core and
// warp-MMA paths): the sink / recent rows, which need only q, so they run beside the prologue
// instead of in a launch of their own.
__global__ void __launch_bounds__(DNT) decode_prologue_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(16) float qc_s[];  // [G][128] (sink / recent CTAs: their buffers)
  if ((int)blockIdx.x >= p.n_pro) {
    decode_sink_recent(p, qc_s, (int)blockIdx.x - p.n_pro);
    return;
  }
  const int kvh = blockIdx.x;
  const int b = kvh / p.Hkv, g = kvh - (kvh / p.Hkv) * p.Hkv;
  const int dc = p.dc[g], de = p.de[g], dc_ld = p.dc_ld[g];
  const int tid = threadIdx.x;
  for (int h = 0; h < p.G; ++h) {
    const long long gh = (long long)b * p.Hq + (long long)g * p.G + h;
    float* rec = p.qw + gh * p.qw_stride;
    if (tid < FA_HEAD_DIM) {
      const int d = p.perm[g][tid];
      const float v = __bfloat162float(p.q[gh * FA_HEAD_DIM + d]) * p.qscale;
      if (tid < dc) {
        qc_s[h * FA_HEAD_DIM + tid] = v;
        rec[de + tid] = 0.0f;  // q_e padding [de, 128)
      } else {
        qc_s[h * FA_HEAD_DIM + tid] = 0.0f;
        rec[tid - dc] = v;
      }
    }
    for (int i = tid; i < 2 * p.F_pad; i += DNT) rec[FA_HEAD_DIM + i] = 0.0f;
  }
  __syncthreads();
  const float* CK = p.CK + (long long)b * p.c_batch + p.c_off[g];
  for (int j = tid; j < p.k; j += DNT) {
    float acc[HL];
#pragma unroll
    for (int h = 0; h < HL; ++h) acc[h] = 0.0f;
    const float* row = CK + (long long)j * dc_ld;
    for (int c = 0; c < dc_ld; c += 4) {
      const float4 x = *reinterpret_cast<const float4*>(row + c);
#pragma unroll
      for (int h = 0; h < HL; ++h) {
        if (h < p.G) {
          const float4 q0 = *reinterpret_cast<const float4*>(qc_s + h * FA_HEAD_DIM + c);
          acc[h] += q0.x * x.x + q0.y * x.y + q0.z * x.z + q0.w * x.w;
        }
      }
    }
    const int f = (j + 1) >> 1;
    const int comp = (j > 0 && (j & 1) == 0) ? 1 : 0;
    const float nrm = (f == 0 || 2 * f == p.P) ? p.norm_single : p.norm_pair;
#pragma unroll
    for (int h = 0; h < HL; ++h) {
      if (h < p.G) {
        const long long gh = (long long)b * p.Hq + (long long)g * p.G + h;
        p.qw[gh * p.qw_stride + FA_HEAD_DIM + 2 * f + comp] = acc[h] * nrm;
      }
    }
  }
}

// ------------------------------------------------------------------------- main: middle
template <int SPT>
__device__ __forceinline__ void decode_middle(const DecodeParams& p, float* sm, int cta) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hs = cta / p.n_splits, sp = cta - (cta / p.n_splits) * p.n_splits;
  const int lo = sp * p.split_len;
  const int hi = min(p.M, lo + p.split_len);
  const int P = p.P;  // basis period

  float* Ws = sm;                           // [F_pad][cos | sin][HL]
  float* qes = Ws + p.F_pad * HL * 2;       // [HL][128]
  float* ps = qes + HL * FA_HEAD_DIM;       // [DT][HL]
  float* red = ps + DT * HL;                // [4][DT][HL]
  float* mx = red + 4 * DT * HL;            // [8][HL]
  float* alpha_s = mx + 8 * HL;             // [HL]
  float* mrun_s = alpha_s + HL;             // [HL]
  float* ured = mrun_s + HL;                // [DNT][16]
  long long* ebase_s = reinterpret_cast<long long*>(ured + DNT * 16);  // [HL]
  int* deld_s = reinterpret_cast<int*>(ebase_s + HL);                  // [HL]
  int* gh_s = deld_s + HL;                                             // [HL]

  if (tid < HL) {
    const int n = tid / p.G;
    const int kv = hs * p.NKV + n;
    const bool valid = (n < p.NKV) && (kv < p.B * p.Hkv);
    if (valid) {
      const int b = kv / p.Hkv, g = kv - (kv / p.Hkv) * p.Hkv;
      gh_s[tid] = b * p.Hq + g * p.G + (tid - n * p.G);
      ebase_s[tid] = (long long)b * p.e_batch + p.e_off[g];
      deld_s[tid] = p.de_ld[g];
    } else {
      gh_s[tid] = -1;
      ebase_s[tid] = 0;
      deld_s[tid] = 0;
    }
    mrun_s[tid] = -INFINITY;
  }
  __syncthreads();
  for (int idx = tid; idx < p.F_pad * HL * 2; idx += DNT) {
    const int f = idx >> 4, c = (idx >> 3) & 1, i = idx & 7;  // [f][cos | sin][head]
    const int gh = gh_s[i];
    Ws[idx] = (gh >= 0 && f < p.F) ? p.qw[(long long)gh * p.qw_stride + FA_HEAD_DIM + 2 * f + c]
                                   : 0.0f;
  }
  for (int idx = tid; idx < HL * FA_HEAD_DIM; idx += DNT) {
    const int i = idx >> 7, d = idx & 127;
    const int gh = gh_s[i];
    qes[idx] = gh >= 0 ? p.qw[(long long)gh * p.qw_stride + d] : 0.0f;
  }
  __syncthreads();

  // scores role: token tau, quarter qf of the frequency slots
  const int tau = ((warp & 1) << 5) | lane;
  const int qf = warp >> 1;
  const int FQ = (p.F + 3) >> 2;
  const int fb = qf * FQ, fe = min(p.F, fb + FQ);
  const int i0 = 2 * qf, i1 = 2 * qf + 1;
  const bool v0 = gh_s[i0] >= 0, v1 = gh_s[i1] >= 0;
  const long long eb0 = ebase_s[i0], eb1 = ebase_s[i1];
  const int dl0 = deld_s[i0], dl1 = deld_s[i1];
  // softmax role: token tau2, heads 2hp, 2hp+1
  const int tau2 = tid >> 2, hp = tid & 3;
  float l0 = 0.0f, l1 = 0.0f;
  // u role: slots ui + j * NTU, token group uq
  const int ui = tid % p.NTU, uq = tid / p.NTU;
  const int UT = DT / p.TG;
  // u accumulators, heads in pairs (paired fp32 FMA): ucs[j][hp] = cos sums of heads 2hp, 2hp+1,
  // uss[j][hp] = sin sums
  float2 ucs[SPT][HL / 2], uss[SPT][HL / 2];
  float cb[SPT], sb[SPT];
#pragma unroll
  for (int j = 0; j < SPT; ++j) {
    phase_sincos((long long)(ui + j * p.NTU) % P, P, p.two_over_P, &sb[j], &cb[j]);
#pragma unroll
    for (int pr2 = 0; pr2 < HL / 2; ++pr2) ucs[j][pr2] = uss[j][pr2] = make_float2(0.0f, 0.0f);
  }
  // exact-dim value role: head ie, 8-dim chunk ce, token group qg
  const int ei = tid % (HL * p.DEC), qg = tid / (HL * p.DEC);
  const int ie = ei / p.DEC, ce = ei - (ei / p.DEC) * p.DEC;
  const bool e_on = gh_s[ie] >= 0 && ce * 8 < deld_s[ie];
  const int dle = deld_s[ie];
  const int ET = DT / p.TGE;
  float acce[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acce[e] = 0.0f;
  const long long ebe = ebase_s[ie];

  for (int t0 = lo; t0 < hi; t0 += DT) {
    const int nt = min(DT, hi - t0);
    // prefetch the next tile's rows into L2
    if (tid < 2 * HL) {
      const int i = (tid & 7);
      const int tn = t0 + DT;
      if (gh_s[i] >= 0 && (i % p.G) == 0 && tn < hi && deld_s[i] > 0) {
        const int nb = min(DT, hi - tn);
        const __nv_bfloat16* base = (tid < HL ? p.EK : p.EV) + ebase_s[i] + (long long)tn * deld_s[i];
        prefetch_l2_bulk(base, (uint32_t)(nb * deld_s[i] * 2));
      }
    }
    // ---------------------------------------------------------------- scores
    float2 part2[HL / 2];
#pragma unroll
    for (int pr2 = 0; pr2 < HL / 2; ++pr2) part2[pr2] = make_float2(0.0f, 0.0f);
    const int tm = t0 + tau;
    if (tau < nt) {
      // the first 32 exact dims of both rows are loaded up front so that their latency
      // hides behind the basis loop
      uint4 ek0[4], ek1[4];
      const __nv_bfloat16* row0 = p.EK + eb0 + (long long)tm * dl0;
      const __nv_bfloat16* row1 = p.EK + eb1 + (long long)tm * dl1;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        ek0[c8] = (v0 && c8 * 8 < dl0) ? *reinterpret_cast<const uint4*>(row0 + c8 * 8) : make_uint4(0, 0, 0, 0);
        ek1[c8] = (v1 && c8 * 8 < dl1) ? *reinterpret_cast<const uint4*>(row1 + c8 * 8) : make_uint4(0, 0, 0, 0);
      }
      if (fb < fe) {
        float sa, ca;
        phase_sincos(tm, P, p.two_over_P, &sa, &ca);
        for (int f0 = fb; f0 < fe; f0 += 32) {
          float s, c;
          phase_sincos(((long long)f0 * tm) % P, P, p.two_over_P, &s, &c);
          const int f1 = min(fe, f0 + 32);
          for (int f = f0; f < f1; ++f) {
            const float4* w4 = reinterpret_cast<const float4*>(Ws + f * (HL * 2));
            const float4 wc0 = w4[0], wc1 = w4[1], ws0 = w4[2], ws1 = w4[3];
            const float2 cc = make_float2(c, c), ss = make_float2(s, s);
            part2[0] = __ffma2_rn(cc, make_float2(wc0.x, wc0.y), part2[0]);
            part2[1] = __ffma2_rn(cc, make_float2(wc0.z, wc0.w), part2[1]);
            part2[2] = __ffma2_rn(cc, make_float2(wc1.x, wc1.y), part2[2]);
            part2[3] = __ffma2_rn(cc, make_float2(wc1.z, wc1.w), part2[3]);
            part2[0] = __ffma2_rn(ss, make_float2(ws0.x, ws0.y), part2[0]);
            part2[1] = __ffma2_rn(ss, make_float2(ws0.z, ws0.w), part2[1]);
            part2[2] = __ffma2_rn(ss, make_float2(ws1.x, ws1.y), part2[2]);
            part2[3] = __ffma2_rn(ss, make_float2(ws1.z, ws1.w), part2[3]);
            const float cn = c * ca - s * sa;
            s = s * ca + c * sa;
            c = cn;
          }
        }
      }
      // exact dims of the middle tokens for heads i0, i1
      float e0 = 0.0f, e1 = 0.0f;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float x[8], y[8];
        bf16x8_to_f32(ek0[c8], x);
        bf16x8_to_f32(ek1[c8], y);
        const float4 qa = *reinterpret_cast<const float4*>(qes + i0 * FA_HEAD_DIM + c8 * 8);
        const float4 qb = *reinterpret_cast<const float4*>(qes + i0 * FA_HEAD_DIM + c8 * 8 + 4);
        const float4 ra = *reinterpret_cast<const float4*>(qes + i1 * FA_HEAD_DIM + c8 * 8);
        const float4 rb = *reinterpret_cast<const float4*>(qes + i1 * FA_HEAD_DIM + c8 * 8 + 4);
        e0 += qa.x * x[0] + qa.y * x[1] + qa.z * x[2] + qa.w * x[3] + qb.x * x[4] + qb.y * x[5] +
              qb.z * x[6] + qb.w * x[7];
        e1 += ra.x * y[0] + ra.y * y[1] + ra.z * y[2] + ra.w * y[3] + rb.x * y[4] + rb.y * y[5] +
              rb.z * y[6] + rb.w * y[7];
      }
      if (v0) {
        for (int c8 = 32; c8 < dl0; c8 += 8) {
          float x[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(row0 + c8), x);
          const float4 qa = *reinterpret_cast<const float4*>(qes + i0 * FA_HEAD_DIM + c8);
          const float4 qb = *reinterpret_cast<const float4*>(qes + i0 * FA_HEAD_DIM + c8 + 4);
          e0 += qa.x * x[0] + qa.y * x[1] + qa.z * x[2] + qa.w * x[3] + qb.x * x[4] +
                qb.y * x[5] + qb.z * x[6] + qb.w * x[7];
        }
      }
      if (v1) {
        for (int c8 = 32; c8 < dl1; c8 += 8) {
          float x[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(row1 + c8), x);
          const float4 qa = *reinterpret_cast<const float4*>(qes + i1 * FA_HEAD_DIM + c8);
          const float4 qb = *reinterpret_cast<const float4*>(qes + i1 * FA_HEAD_DIM + c8 + 4);
          e1 += qa.x * x[0] + qa.y * x[1] + qa.z * x[2] + qa.w * x[3] + qb.x * x[4] +
                qb.y * x[5] + qb.z * x[6] + qb.w * x[7];
        }
      }
      // heads i0 = 2 qf, i1 = 2 qf + 1 form pair qf
#pragma unroll
      for (int pr2 = 0; pr2 < HL / 2; ++pr2)
        if (pr2 == qf) {
          part2[pr2].x += e0;
          part2[pr2].y += e1;
        }
    }
    {
      float4* dst = reinterpret_cast<float4*>(red + (qf * DT + tau) * HL);
      dst[0] = make_float4(part2[0].x, part2[0].y, part2[1].x, part2[1].y);
      dst[1] = make_float4(part2[2].x, part2[2].y, part2[3].x, part2[3].y);
    }
    __syncthreads();
    // ---------------------------------------------------------------- online softmax
    float s0, s1;
    {
      const int h0 = 2 * hp;
      s0 = red[(0 * DT + tau2) * HL + h0] + red[(1 * DT + tau2) * HL + h0] +
           red[(2 * DT + tau2) * HL + h0] + red[(3 * DT + tau2) * HL + h0];
      s1 = red[(0 * DT + tau2) * HL + h0 + 1] + red[(1 * DT + tau2) * HL + h0 + 1] +
           red[(2 * DT + tau2) * HL + h0 + 1] + red[(3 * DT + tau2) * HL + h0 + 1];
      if (tau2 >= nt) s0 = s1 = -INFINITY;
      float m0 = s0, m1 = s1;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
        m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
      }
      if (lane < 4) {
        mx[warp * HL + 2 * lane] = m0;
        mx[warp * HL + 2 * lane + 1] = m1;
      }
    }
    __syncthreads();
    if (tid < HL) {
      float tmx = mx[tid];
#pragma unroll
      for (int w = 1; w < 8; ++w) tmx = fmaxf(tmx, mx[w * HL + tid]);
      const float mold = mrun_s[tid];
      const float mnew = fmaxf(mold, tmx);
      alpha_s[tid] = (mold == -INFINITY) ? 0.0f : exp2f(mold - mnew);
      mrun_s[tid] = mnew;
    }
    __syncthreads();
    {
      const int h0 = 2 * hp;
      const float pv0 = exp2f(s0 - mrun_s[h0]);
      const float pv1 = exp2f(s1 - mrun_s[h0 + 1]);
      *reinterpret_cast<float2*>(ps + tau2 * HL + h0) = make_float2(pv0, pv1);
      l0 = l0 * alpha_s[h0] + pv0;
      l1 = l1 * alpha_s[h0 + 1] + pv1;
    }
    __syncthreads();
    // ---------------------------------------------------------------- u += p phi
    {
      float2 al[HL / 2];
#pragma unroll
      for (int pr2 = 0; pr2 < HL / 2; ++pr2)
        al[pr2] = make_float2(alpha_s[2 * pr2], alpha_s[2 * pr2 + 1]);
#pragma unroll
      for (int j = 0; j < SPT; ++j)
#pragma unroll
        for (int pr2 = 0; pr2 < HL / 2; ++pr2) {
          ucs[j][pr2] = __fmul2_rn(ucs[j][pr2], al[pr2]);
          uss[j][pr2] = __fmul2_rn(uss[j][pr2], al[pr2]);
        }
      const int tb = uq * UT, te = min(nt, tb + UT);
      if (tb < te) {
        float c[SPT], s[SPT];
#pragma unroll
        for (int j = 0; j < SPT; ++j)
          phase_sincos(((long long)(ui + j * p.NTU) * (t0 + tb)) % P, P, p.two_over_P, &s[j],
                       &c[j]);
        for (int t = tb; t < te; ++t) {
          const float4 pa = *reinterpret_cast<const float4*>(ps + t * HL);
          const float4 pb = *reinterpret_cast<const float4*>(ps + t * HL + 4);
          const float2 pr[HL / 2] = {make_float2(pa.x, pa.y), make_float2(pa.z, pa.w),
                                     make_float2(pb.x, pb.y), make_float2(pb.z, pb.w)};
#pragma unroll
          for (int j = 0; j < SPT; ++j) {
            const float2 cc = make_float2(c[j], c[j]), ss = make_float2(s[j], s[j]);
#pragma unroll
            for (int pr2 = 0; pr2 < HL / 2; ++pr2) {
              ucs[j][pr2] = __ffma2_rn(pr[pr2], cc, ucs[j][pr2]);
              uss[j][pr2] = __ffma2_rn(pr[pr2], ss, uss[j][pr2]);
            }
            const float cn = c[j] * cb[j] - s[j] * sb[j];
            s[j] = s[j] * cb[j] + c[j] * sb[j];
            c[j] = cn;
          }
        }
      }
    }
    // ---------------------------------------------------------------- exact-dim values
    {
      const float ae = alpha_s[ie];
#pragma unroll
      for (int e = 0; e < 8; ++e) acce[e] *= ae;
      if (e_on) {
        const int tb = qg * ET, te = min(nt, tb + ET);
        for (int t = tb; t < te; ++t) {
          const float pv = ps[t * HL + ie];
          float x[8];
          bf16x8_to_f32(*reinterpret_cast<const uint4*>(p.EV + ebe + (long long)(t0 + t) * dle +
                                                        ce * 8),
                        x);
#pragma unroll
          for (int e = 0; e < 8; ++e) acce[e] += pv * x[e];
        }
      }
    }
    __syncthreads();
  }

  // ------------------------------------------------------------------ partial record
  const long long bhq = (long long)p.B * p.Hq;
#pragma unroll
  for (int o = 4; o < 32; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
  }
  if (lane < 4) {
    mx[warp * HL + 2 * lane] = l0;
    mx[warp * HL + 2 * lane + 1] = l1;
  }
  // exact-dim accumulators: reduce over token groups
  {
    float4* dst = reinterpret_cast<float4*>(red + (qg * (HL * p.DEC) + ei) * 8);
    dst[0] = make_float4(acce[0], acce[1], acce[2], acce[3]);
    dst[1] = make_float4(acce[4], acce[5], acce[6], acce[7]);
  }
  if (p.TG > 1) {
    // SPT == 1 whenever TG > 1; per thread [head][cos, sin]
    float4* dst = reinterpret_cast<float4*>(ured + tid * 16);
#pragma unroll
    for (int pr2 = 0; pr2 < HL / 2; ++pr2)
      dst[pr2] = make_float4(ucs[0][pr2].x, uss[0][pr2].x, ucs[0][pr2].y, uss[0][pr2].y);
  }
  __syncthreads();
  if (tid < HL && gh_s[tid] >= 0) {
    float l = 0.0f;
#pragma unroll
    for (int w = 0; w < 8; ++w) l += mx[w * HL + tid];
    float* rec = p.rec + ((long long)sp * bhq + gh_s[tid]) * p.rec_stride;
    rec[0] = mrun_s[tid];
    rec[1] = l;
  }
  if (qg == 0 && e_on) {
    float v[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = 0.0f;
    for (int q2 = 0; q2 < p.TGE; ++q2) {
      const float* src = red + (q2 * (HL * p.DEC) + ei) * 8;
#pragma unroll
      for (int e = 0; e < 8; ++e) v[e] += src[e];
    }
    float* rec = p.rec + ((long long)sp * bhq + gh_s[ie]) * p.rec_stride + 4 + ce * 8;
    reinterpret_cast<float4*>(rec)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(rec)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
  if (p.TG > 1) {
    if (uq == 0 && ui < p.F) {
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = 0.0f;
      for (int q2 = 0; q2 < p.TG; ++q2) {
        const float* src = ured + (q2 * p.NTU + ui) * 16;
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] += src[e];
      }
#pragma unroll
      for (int h = 0; h < HL; ++h) {
        if (gh_s[h] >= 0) {
          float* rec = p.rec + ((long long)sp * bhq + gh_s[h]) * p.rec_stride + 4 + FA_HEAD_DIM;
          *reinterpret_cast<float2*>(rec + 2 * ui) = make_float2(v[2 * h], v[2 * h + 1]);
        }
      }
    }
  } else {
#pragma unroll
    for (int j = 0; j < SPT; ++j) {
      const int f = ui + j * p.NTU;
      if (f < p.F) {
#pragma unroll
        for (int h = 0; h < HL; ++h) {
          if (gh_s[h] >= 0) {
            float* rec = p.rec + ((long long)sp * bhq + gh_s[h]) * p.rec_stride + 4 + FA_HEAD_DIM;
            const float uc = (h & 1) ? ucs[j][h >> 1].y : ucs[j][h >> 1].x;
            const float us = (h & 1) ? uss[j][h >> 1].y : uss[j][h >> 1].x;
            *reinterpret_cast<float2*>(rec + 2 * f) = make_float2(uc, us);
          }
        }
      }
    }
  }
}

template <int SPT>
__global__ void __launch_bounds__(DNT, SPT == 1 ? 2 : 1)
    decode_main_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ __align__(16) float sm[];
  const int cta = blockIdx.x;
  if (cta < p.n_mid)
    decode_middle<SPT>(p, sm, cta);
  else
    decode_sink_recent(p, sm, cta - p.n_mid);
}

// ------------------------------------------------------------------------- combine
// One CTA per (KV head, group of GT of its G query heads; the heads of a group share C_V),
// CB_THREADS threads = 8 warps. GT = G unless that leaves too few CTAs for the GPU.
//  1. warp h < GT: record weights w_r = 2^(m_r - m*) and the sum l of query head h;
//  2. the weighted sum over split records of their payload (retained-dim values, then u
//     slots), CB_PW(GT) columns per pass: warp w takes records w, w + 8, ... and reads each
//     record's columns as CB_NPW(GT) float4 per lane, CB_RB(GT) records per batch, so many
//     loads are in flight; the eight partial rows are then added in a fixed order
//     (deterministic);
//  3. out_c = u C_V with u_j = basis scale of function j x its slot sum, C_V staged
//     through shared memory in double-buffered CB_KC-row chunks (cp.async, started before
//     step 1: C_V does not depend on the records);
//  4. sink / recent records (all 128 dims in natural order) are added per dim, the dims
//     scattered back, normalised and stored.
constexpr int CB_THREADS = 256;
constexpr int CB_KC = 64;

__host__ __device__ constexpr int CB_NPW(int GT) { return GT >= 8 ? 2 : 4; }
__host__ __device__ constexpr int CB_PW(int GT) { return 128 * CB_NPW(GT); }
__host__ __device__ constexpr int CB_RB(int GT) {
  return 16 / (GT * CB_NPW(GT)) > 1 ? 16 / (GT * CB_NPW(GT)) : 1;
}

// Float offsets of the combine's shared arrays; every one a multiple of 4 (16 bytes), so
// the float4 accesses stay aligned.
__host__ __device__ inline int combine_wts_floats(int G, int nrec) { return (G * nrec + 3) & ~3; }

// Columns of one pass actually used: the pass width, or the whole payload if narrower.
__host__ __device__ inline int combine_pass_cols(int GT, int payload) {
  return payload < CB_PW(GT) ? ((payload + 3) & ~3) : CB_PW(GT);
}

__host__ __device__ inline size_t combine_smem_floats(int GT, int nrec, int payload) {
  return (size_t)combine_wts_floats(GT, nrec) + 16 + (size_t)GT * payload +
         (size_t)8 * GT * combine_pass_cols(GT, payload) + (size_t)2 * CB_KC * FA_HEAD_DIM +
         2 * (size_t)GT * FA_HEAD_DIM + FA_HEAD_DIM;
}

template <int GT>
__global__ void __launch_bounds__(CB_THREADS) decode_combine_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NPW = CB_NPW(GT), RB = CB_RB(GT);
  extern __shared__ __align__(16) float cs[];
  const int n_grp = p.G / GT;
  const int kvh = blockIdx.x / n_grp, hg = blockIdx.x - (blockIdx.x / n_grp) * n_grp;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int b = kvh / p.Hkv, g = kvh - (kvh / p.Hkv) * p.Hkv;
  const int dc = p.dc[g], dc_ld = p.dc_ld[g], nrec = p.n_rec, ns = p.n_splits;
  const int k = p.k;
  const int payload = p.rec_stride - 4;     // retained-dim values (128) + u slots (2 F_pad)
  const int PWc = combine_pass_cols(GT, payload);
  float* wts = cs;                          // [GT][nrec]
  float* mst = wts + combine_wts_floats(GT, nrec);  // [8]
  float* lsum = mst + 8;                    // [8]
  float* sum = lsum + 8;                    // [GT][payload] weighted sum of split payloads
  float* red = sum + GT * payload;          // [8 warps][GT][PWc] partial column sums
  float* cvs = red + 8 * GT * PWc;          // [2][CB_KC][128] chunks of C_V (double buffer)
  float* cpart = cvs + 2 * CB_KC * FA_HEAD_DIM;  // [2][GT][128] halves of u C_V
  int* inv = reinterpret_cast<int*>(cpart + 2 * GT * FA_HEAD_DIM);  // [128]
  const long long bhq = (long long)p.B * p.Hq;
  const long long gh0 = (long long)b * p.Hq + (long long)g * p.G + (long long)hg * GT;
  auto rec = [&](int r, int h) -> const float* {
    return p.rec + ((long long)r * bhq + gh0 + h) * p.rec_stride;
  };

  // C_V does not depend on the split records: its first two CB_KC-row chunks are copied
  // into shared memory (cp.async) while the records are merged. One commit group per chunk
  // (empty past the last), so waiting for all but the newest group completes chunk i.
  const float* CV = p.CV + (long long)b * p.c_batch + p.c_off[g];
  const bool do_cv = k > 0 && dc > 0 && ns > 0;
  auto load_cv_chunk = [&](int ci) {
    const int j0 = ci * CB_KC;
    if (do_cv && j0 < k) {
      const int nj = min(CB_KC, k - j0), nq = dc_ld / 4;
      float* buf = cvs + (ci & 1) * CB_KC * FA_HEAD_DIM;
      for (int e = tid; e < nj * nq; e += CB_THREADS) {
        const int jj = e / nq, c4 = e - jj * nq;
        cp_async16(buf + jj * FA_HEAD_DIM + 4 * c4, CV + (long long)(j0 + jj) * dc_ld + 4 * c4);
      }
    }
    cp_async_commit();
  };
  load_cv_chunk(0);
  load_cv_chunk(1);
  if (tid < FA_HEAD_DIM) inv[p.perm[g][tid]] = tid;
  if (warp < GT) {
    const int h = warp;
    float mx = -INFINITY;
    for (int r = lane; r < nrec; r += 32) mx = fmaxf(mx, rec(r, h)[0]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float ls = 0.0f;
    for (int r = lane; r < nrec; r += 32) {
      const float* rr = rec(r, h);
      const float w = exp2f(rr[0] - mx);
      wts[h * nrec + r] = w;
      ls += w * rr[1];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, o);
    if (lane == 0) {
      mst[h] = mx;
      lsum[h] = ls;
    }
  }
  __syncthreads();
  // weighted sum of the split records' payloads, PWc columns per pass; lane l, piece j
  // covers columns c0 + 128 j + 4 l .. + 3
  for (int c0 = 0; c0 < payload && ns > 0; c0 += PWc) {
    float4 a[GT][NPW];
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
      for (int j = 0; j < NPW; ++j) a[h][j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int r0 = warp; r0 < ns; r0 += 8 * RB) {
      float4 v[RB][GT][NPW];
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int r = r0 + 8 * u;
#pragma unroll
        for (int h = 0; h < GT; ++h)
#pragma unroll
          for (int j = 0; j < NPW; ++j) {
            const int col = c0 + 128 * j + 4 * lane;
            v[u][h][j] = (r < ns && col < payload && 128 * j + 4 * lane < PWc)
                             ? *reinterpret_cast<const float4*>(rec(r, h) + 4 + col)
                             : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          }
      }
#pragma unroll
      for (int u = 0; u < RB; ++u) {
        const int r = r0 + 8 * u;
#pragma unroll
        for (int h = 0; h < GT; ++h) {
          const float w = r < ns ? wts[h * nrec + r] : 0.0f;
#pragma unroll
          for (int j = 0; j < NPW; ++j) {
            a[h][j].x += w * v[u][h][j].x;
            a[h][j].y += w * v[u][h][j].y;
            a[h][j].z += w * v[u][h][j].z;
            a[h][j].w += w * v[u][h][j].w;
          }
        }
      }
    }
#pragma unroll
    for (int h = 0; h < GT; ++h)
#pragma unroll
      for (int j = 0; j < NPW; ++j)
        if (128 * j + 4 * lane < PWc)
          *reinterpret_cast<float4*>(red + (warp * GT + h) * PWc + 128 * j + 4 * lane) = a[h][j];
    __syncthreads();
    for (int idx = tid; idx < GT * PWc; idx += CB_THREADS) {
      const int h = idx / PWc, cc = idx - (idx / PWc) * PWc;
      if (c0 + cc < payload) {
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += red[(w * GT + h) * PWc + cc];
        sum[h * payload + c0 + cc] = v;
      }
    }
    __syncthreads();
  }
  // out_c = u C_V: C_V rows in double-buffered chunks; thread (half, column i) sums the rows
  // of its parity
  const int colc = tid & (FA_HEAD_DIM - 1), half = tid >> 7;
  float acc[GT];
#pragma unroll
  for (int h = 0; h < GT; ++h) acc[h] = 0.0f;
  for (int j0 = 0; j0 < k && do_cv; j0 += CB_KC) {
    const int nj = min(CB_KC, k - j0), ci = j0 / CB_KC;
    const float* cvb = cvs + (ci & 1) * CB_KC * FA_HEAD_DIM;
    cp_async_wait<1>();  // this thread's copies of chunk ci have landed
    __syncthreads();     // everyone's copies (first pass: sum written)
    if (colc < dc) {
      for (int jj = half; jj < nj; jj += 2) {
        const int j = j0 + jj, f = (j + 1) >> 1;
        const int slot = FA_HEAD_DIM + 2 * f + ((j > 0 && (j & 1) == 0) ? 1 : 0);
        const float cv = cvb[jj * FA_HEAD_DIM + colc] *
                         ((f == 0 || 2 * f == p.P) ? p.norm_single : p.norm_pair);
#pragma unroll
        for (int h = 0; h < GT; ++h) acc[h] += sum[h * payload + slot] * cv;
      }
    }
    __syncthreads();     // chunk ci consumed: its buffer takes chunk ci + 2
    load_cv_chunk(ci + 2);
  }
  cp_async_wait<0>();
  __syncthreads();
#pragma unroll
  for (int h = 0; h < GT; ++h) cpart[(half * GT + h) * FA_HEAD_DIM + colc] = acc[h];
  __syncthreads();
  for (int idx = tid; idx < GT * FA_HEAD_DIM; idx += CB_THREADS) {
    const int h = idx / FA_HEAD_DIM, d = idx - h * FA_HEAD_DIM;
    const int i = inv[d];
    float o = 0.0f;
    if (ns > 0) {
      if (i >= dc)
        o = sum[h * payload + (i - dc)];
      else
        o = cpart[h * FA_HEAD_DIM + i] + cpart[(GT + h) * FA_HEAD_DIM + i];
    }
    const float* wh = wts + h * nrec;
    for (int r = ns; r < nrec; ++r) o += wh[r] * rec(r, h)[4 + d];
    o /= lsum[h];
    const long long gh = gh0 + h;
    if (p.out_f32)
      static_cast<float*>(p.out)[gh * FA_HEAD_DIM + d] = o;
    else
      static_cast<__nv_bfloat16*>(p.out)[gh * FA_HEAD_DIM + d] = __float2bfloat16_rn(o);
  }
}

// ------------------------------------------------------------------------- host side
template <int GT>
static cudaError_t launch_combine_t(const DecodeParams& p, const DecodeConfig& c, int n_heads,
                                    cudaStream_t stream) {
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(decode_combine_kernel<GT>),
                                   (int)c.smem_combine);
  if (e != cudaSuccess) return e;
  decode_combine_kernel<GT><<<n_heads * (p.G / GT), CB_THREADS, c.smem_combine, stream>>>(p);
  return cudaGetLastError();
}

static cudaError_t launch_combine(const DecodeParams& p, const DecodeConfig& c, int n_heads,
                                  cudaStream_t stream) {
  switch (c.cb_gt) {
    case 1: return launch_combine_t<1>(p, c, n_heads, stream);
    case 2: return launch_combine_t<2>(p, c, n_heads, stream);
    case 4: return launch_combine_t<4>(p, c, n_heads, stream);
    case 8: return launch_combine_t<8>(p, c, n_heads, stream);
    default: return cudaErrorInvalidValue;
  }
}
static int next_pow2(int x) {
  int v = 1;
  while (v < x) v <<= 1;
  return v;
}

static size_t main_smem_bytes(int F_pad) {
  const size_t mid = (size_t)(F_pad * HL * 2 + HL * FA_HEAD_DIM + DT * HL + 4 * DT * HL + 8 * HL +
                              2 * HL + DNT * 16) * 4 +
                     HL * 8 + 2 * HL * 4;
  const size_t fpart = sink_recent_smem_bytes();
  return mid > fpart ? mid : fpart;
}

template <int SPT>
static cudaError_t occupancy(int* blocks, size_t smem) {
  return cached_occupancy(reinterpret_cast<const void*>(decode_main_kernel<SPT>), DNT, smem, blocks);
}

// Ring and buffer sizes of the cluster tensor-core kernel for a plan, cluster size C and
// 2 F_pad slots; leaves c->cl = 0 when its buffers do not fit in shared memory.
static void cl_configure(const fa_plan* plan, int C, int slots, DecodeConfig* c) {
  const fa_shape& sh = plan->shape;
  const int G = plan->G, nown = 4 / C, nkq = 32 / G;
  const int SL = ((slots + C - 1) / C + 63) / 64 * 64;
  // bytes one token of a ring slot takes for the worst CTA (sum of its exact KV heads'
  // row pitches) and the number of those heads with exact dims (each padded in a slot)
  long long worst_row = 0, worst_pad = 0;
  const long long bhq = (long long)sh.B * sh.Hq;
  const long long n_hs = (bhq + 127) / 128;
  for (long long hs = 0; hs < n_hs; ++hs)
    for (int r = 0; r < C; ++r) {
      long long row = 0, pad = 0;
      for (int li = 0; li < nown; ++li)
        for (int j = 0; j < nkq; ++j) {
          const long long gh = hs * 128 + 32 * (r * nown + li) + (long long)j * G;
          if (gh >= bhq) continue;
          const int g = (int)((gh % sh.Hq) / G);
          row += 2LL * plan->de_ld[g];
          pad += plan->de_ld[g] > 0 ? 64 : 0;
        }
      worst_row = row > worst_row ? row : worst_row;
      worst_pad = pad > worst_pad ? pad : worst_pad;
    }
  const size_t fixed = decode_cl_smem_bytes(C, SL, 0, 0);
  const size_t budget = 227 * 1024;
  if (fixed >= budget) return;
  int TB = 32;
  int slot = 0, stages = 0;
  for (; TB >= 8; TB >>= 1) {
    slot = (int)((TB * worst_row + worst_pad + 127) / 128 * 128);
    if (slot < 128) slot = 128;
    stages = (int)((budget - fixed) / (size_t)slot);
    if (stages > 8) stages = 8;
    if (stages >= 3 || (TB == 8 && stages >= 2)) break;
  }
  if (TB < 8 || stages < 2) return;
  int cols = 32;
  while (cols < SL + 64 + SL / 2) cols <<= 1;
  c->cl = 1;
  c->cl_C = C;
  c->cl_SL = SL;
  c->cl_TB = TB;
  c->cl_stages = stages;
  c->cl_slot_bytes = slot;
  c->cl_tmem_cols = cols;
  c->cl_smem = (int)decode_cl_smem_bytes(C, SL, slot, stages);
}

// Derive the launch configuration. `requested` <= 0 selects the split count from a
// wave-quantisation cost model for the current device. A plan the kernels cannot serve
// returns cudaErrorInvalidValue with *why naming the limit.
cudaError_t decode_configure(const fa_plan* plan, int requested, DecodeConfig* c,
                             const char** why) {
  memset(c, 0, sizeof(*c));
  const fa_shape& sh = plan->shape;
  const int M = plan->M;
  c->F = sh.k / 2 + 1;
  c->F_pad = (c->F + 3) & ~3;
  c->SPT = c->F <= 256 ? 1 : (c->F <= 512 ? 2 : 4);
  int ntu = next_pow2((c->F + c->SPT - 1) / c->SPT);
  if (ntu < 4) ntu = 4;
  if (ntu > DNT) ntu = DNT;
  c->NTU = ntu;
  c->TG = DNT / ntu;
  int de_ld_max = 8;
  for (int g = 0; g < sh.Hkv; ++g) de_ld_max = plan->de_ld[g] > de_ld_max ? plan->de_ld[g] : de_ld_max;
  c->DEC = next_pow2(de_ld_max / 8);
  c->TGE = DNT / (HL * c->DEC);
  c->NKV = HL / plan->G;
  const int n_heads = sh.B * sh.Hkv;
  c->smem_main = main_smem_bytes(c->F_pad);
  c->de_ld_max = de_ld_max;
  // The tensor-core split kernel runs exactly when the plan laid E out token-major (k <=
  // 255, so W and U of 128 heads x 2F <= 256 slots fit on chip; G in {1, 2, 4}; at most
  // 32 retained dims per KV head).
  c->tc_F2 = ((2 * c->F + 63) / 64) * 64;
  c->tc = (M > 0 && plan->e_token_major) ? 1 : 0;
  // The warp-MMA split kernel (16 query heads per CTA, U in registers) takes the other
  // plans with 256 <= k <= 1023 (2F rounded up to 512 or 1024 slots).
  c->hm_F2 = 2 * c->F <= 512 ? 512 : 1024;
  c->hm = (!c->tc && M > 0 && sh.k >= 256 && c->hm_F2 <= 1024) ? 1 : 0;
  int cols = 32;  // U (2F slots), S (2 x 32 tokens), W_lo (2F / 2 columns of slot pairs)
  while (cols < c->tc_F2 + 64 + c->tc_F2 / 2) cols <<= 1;
  c->tc_tmem_cols = cols;
  // The cluster tensor-core split kernel takes the plans with 256 <= k <= 1023 on
  // per-KV-head E blocks when G is 2, 4 or 8, its per-CTA buffers fit, and its 128-head
  // sets are at least three quarters full (it replaces the warp-MMA kernel there). A set's
  // cost hardly depends on how many of its heads are valid: with 32 query heads the
  // warp-MMA kernel (16 heads per CTA) decodes in 0.6-0.75 of its time, from 96 on the
  // cluster kernel wins (up to 1.6x at 128).
  c->cl = 0;
  const long long nq = (long long)sh.B * sh.Hq;
  const bool sets_full = 4 * nq >= 3 * 128 * ((nq + 127) / 128);
  if (!c->tc && M > 0 && sets_full && (plan->G == 2 || plan->G == 4 || plan->G == 8)) {
    const int slots = 2 * c->F_pad;
    const int C = slots <= 256 ? 1 : (slots <= 512 ? 2 : (slots <= 1024 ? 4 : 0));
    if (C >= 2 && de_ld_max <= 64) cl_configure(plan, C, slots, c);
    // a device on which no cluster of it can be resident keeps the warp-MMA kernel (with no
    // device to ask, the plan's choice stands)
    int nclu = 0;
    if (c->cl && decode_cl_max_clusters(c->cl_C, c->cl_smem, &nclu) == cudaSuccess && nclu < 1)
      c->cl = 0;
  }
  if (c->cl) c->hm = 0;
  const int unit_tokens = (c->tc || c->cl) ? 32 : DT;  // tokens per tile (64: warp-MMA, CUDA cores)
  const int n_headsets = (c->tc || c->cl) ? (sh.B * sh.Hq + 127) / 128
                               : (c->hm ? (sh.B * sh.Hq + 15) / 16 : (n_heads + c->NKV - 1) / c->NKV);
  const int ntiles = (M + unit_tokens - 1) / unit_tokens;
  if (M == 0) {
    c->n_splits = 0;
    c->split_len = 0;
  } else {
    int ns;
    if (requested > 0) {
      ns = requested < ntiles ? requested : ntiles;
    } else {
      int sms = 148, occ = 1;
      cudaError_t e = device_sm_count(&sms);
      if (e != cudaSuccess) return e;
      if (c->cl) {
        // slots = resident clusters (each cluster serves one head set and split)
        int nclu = 0;
        e = decode_cl_max_clusters(c->cl_C, c->cl_smem, &nclu);
        if (e != cudaSuccess) return e;
        sms = nclu > 0 ? nclu : 1;
        occ = 1;
      } else if (c->tc || c->hm) {
        occ = 1;  // one CTA per SM (shared memory)
      } else {
        e = c->SPT == 1 ? occupancy<1>(&occ, c->smem_main)
                        : (c->SPT == 2 ? occupancy<2>(&occ, c->smem_main) : occupancy<4>(&occ, c->smem_main));
        if (e != cudaSuccess) return e;
      }
      if (occ < 1) occ = 1;
      const long long slots = (long long)sms * occ;
      // cost = waves x tiles per CTA, plus a small per-split charge for the record
      // traffic and the combine work
      double best = 1e300;
      ns = 1;
      for (int cand = 1; cand <= ntiles && cand <= 4096; ++cand) {
        const int per = (ntiles + cand - 1) / cand;
        const int eff = (ntiles + per - 1) / per;
        if (eff != cand) continue;
        const long long ctas = (long long)n_headsets * cand;
        const long long waves = (ctas + slots - 1) / slots;
        const double cost = (double)waves * (per + 1.0) + 0.02 * cand;
        if (cost < best) {
          best = cost;
          ns = cand;
        }
      }
    }
    // the combine keeps the G x n_rec record weights in shared memory: at most as many
    // splits as fit (thousands; only an explicit request can reach the bound)
    const long long nfs = (plan->S + plan->R + FT - 1) / FT;
    const long long fixed = (long long)combine_smem_floats(plan->G, 0, FA_HEAD_DIM + 2 * c->F_pad) + 4;
    const long long ns_max = ((227 * 1024) / 4 - fixed) / plan->G - nfs;
    if (ns_max < 1) {
      // the sink / recent records alone fill the combine's shared memory
      if (why) *why = "too many sink + recent rows for the combine (S + R too large for this k and G)";
      return cudaErrorInvalidValue;
    }
    if (ns > ns_max) ns = (int)ns_max;
    const int per = (ntiles + ns - 1) / ns;
    c->n_splits = (ntiles + per - 1) / per;
    c->split_len = per * unit_tokens;
  }
  const int nF = plan->S + plan->R;
  c->n_fsplits = (nF + FT - 1) / FT;
  c->n_rec = c->n_splits + c->n_fsplits;
  c->rec_stride = 4 + FA_HEAD_DIM + 2 * c->F_pad;
  c->qw_stride = FA_HEAD_DIM + 2 * c->F_pad;
  const long long bhq = (long long)sh.B * sh.Hq;
  c->qw_bytes = (size_t)(bhq * c->qw_stride * 4);
  c->rec_bytes = (size_t)((long long)c->n_rec * bhq * c->rec_stride * 4);
  // query heads per combine CTA: all G of a KV head (they share C_V) unless that leaves
  // fewer than two CTAs per SM, then halved (each CTA re-reads C_V)
  {
    int sms = 148;
    if (device_sm_count(&sms) != cudaSuccess) sms = 148;  // no device: sizes only
    int gt = plan->G;
    while (gt > 1 && (long long)n_heads * (plan->G / gt) < 2LL * sms) gt >>= 1;
    c->cb_gt = gt;
  }
  c->smem_combine = combine_smem_floats(c->cb_gt, c->n_rec, c->rec_stride - 4) * 4;
  if (c->smem_combine > 227 * 1024) {
    if (why) *why = "the combine's shared memory would exceed 227 KB (too many split records)";
    return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

cudaError_t launch_decode(const fa_plan* plan, const DecodeConfig& c, const void* q,
                          const fa_cache* cache, void* out, int out_dtype, void* workspace,
                          cudaStream_t stream) {
  const fa_shape& sh = plan->shape;
  DecodeParams p;
  memset(&p, 0, sizeof(p));
  p.B = sh.B;
  p.Hq = sh.Hq;
  p.Hkv = sh.Hkv;
  p.G = plan->G;
  p.M = plan->M;
  p.k = plan->M > 0 ? sh.k : 0;
  p.F = c.F;
  p.F_pad = c.F_pad;
  p.nF = plan->S + plan->R;
  p.n_splits = c.n_splits;
  p.split_len = c.split_len;
  p.n_fsplits = c.n_fsplits;
  p.NKV = c.NKV;
  const int n_heads = sh.B * sh.Hkv;
  const int n_headsets = (n_heads + c.NKV - 1) / c.NKV;
  p.n_mid = n_headsets * c.n_splits;
  p.n_rec = c.n_rec;
  p.rec_stride = c.rec_stride;
  p.qw_stride = c.qw_stride;
  p.NTU = c.NTU;
  p.TG = c.TG;
  p.tc_F2 = c.tc_F2;
  p.tc_tmem_cols = c.tc_tmem_cols;
  p.cl_C = c.cl_C;
  p.cl_SL = c.cl_SL;
  p.cl_TB = c.cl_TB;
  p.cl_stages = c.cl_stages;
  p.cl_slot_bytes = c.cl_slot_bytes;
  p.cl_tmem_cols = c.cl_tmem_cols;
  p.DEC = c.DEC;
  p.TGE = c.TGE;
  p.qscale = (float)(1.4426950408889634 / sqrt((double)FA_HEAD_DIM));
  const int Pq = plan->P > 0 ? plan->P : 1;  // basis period
  p.P = Pq;
  p.norm_single = (float)(1.0 / sqrt((double)Pq));
  p.norm_pair = (float)sqrt(2.0 / (double)Pq);
  p.two_over_P = (float)(2.0 / (double)Pq);
  p.e_batch = plan->e_batch;
  p.c_batch = plan->c_batch;
  for (int g = 0; g < sh.Hkv; ++g) {
    p.e_off[g] = plan->e_off[g];
    p.c_off[g] = plan->c_off[g];
    p.de[g] = plan->de[g];
    p.de_ld[g] = plan->de_ld[g];
    p.dc[g] = plan->dc[g];
    p.dc_ld[g] = plan->dc_ld[g];
    memcpy(p.perm[g], plan->perm[g], FA_HEAD_DIM);
  }
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.FK = static_cast<const __nv_bfloat16*>(cache->F_K);
  p.FV = static_cast<const __nv_bfloat16*>(cache->F_V);
  p.EK = static_cast<const __nv_bfloat16*>(cache->E_K);
  p.EV = static_cast<const __nv_bfloat16*>(cache->E_V);
  p.CK = static_cast<const float*>(cache->C_K);
  p.CV = static_cast<const float*>(cache->C_V);
  p.out = out;
  p.out_f32 = out_dtype == FA_F32 ? 1 : 0;
  p.qw = static_cast<float*>(workspace);
  p.rec = reinterpret_cast<float*>(static_cast<char*>(workspace) + c.qw_bytes);

  cudaError_t e;
  // On the tensor-core and warp-MMA paths the sink / recent rows run as extra CTAs of the
  // prologue launch (small CTAs that need only q; the split kernels hold whole SMs).
  const bool sr_with_prologue = p.M > 0 && (c.tc || c.hm || c.cl);
  if (p.M > 0) {
    p.n_pro = n_heads;
    const int pro_grid = n_heads + (sr_with_prologue ? n_heads * c.n_fsplits : 0);
    size_t pro_smem = (size_t)plan->G * FA_HEAD_DIM * 4;
    if (sr_with_prologue && sink_recent_smem_bytes() > pro_smem) pro_smem = sink_recent_smem_bytes();
    decode_prologue_kernel<<<pro_grid, DNT, pro_smem, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (c.tc) {
    p.e_row = plan->e_pitch[0];
    if ((e = launch_decode_tc(p, plan->de_ld[0], stream)) != cudaSuccess) return e;
  } else if (plan->e_token_major && plan->M > 0) {
    return cudaErrorInvalidValue;  // the CUDA-core kernel reads per-KV-head E blocks only
  } else if (c.cl) {
    if ((e = launch_decode_cl(p, stream)) != cudaSuccess) return e;
  } else if (c.hm) {
    if ((e = launch_decode_hmma(p, c.hm_F2, stream)) != cudaSuccess) return e;
  }
  const int grid = sr_with_prologue ? 0 : p.n_mid + n_heads * c.n_fsplits;
  if (grid > 0) {
    int occ = 0;
    if (c.SPT == 1) {
      if ((e = occupancy<1>(&occ, c.smem_main)) != cudaSuccess) return e;
      decode_main_kernel<1><<<grid, DNT, c.smem_main, stream>>>(p);
    } else if (c.SPT == 2) {
      if ((e = occupancy<2>(&occ, c.smem_main)) != cudaSuccess) return e;
      decode_main_kernel<2><<<grid, DNT, c.smem_main, stream>>>(p);
    } else {
      if ((e = occupancy<4>(&occ, c.smem_main)) != cudaSuccess) return e;
      decode_main_kernel<4><<<grid, DNT, c.smem_main, stream>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return launch_combine(p, c, n_heads, stream);
}

}  // namespace fa
