// fa_decode_tc.cu -- split-L decode of the middle span with the k-length contractions on
// the tcgen05 tensor cores (fp16 operands, fp32 accumulators in tensor memory).
//
// Same mathematics as the CUDA-core split kernel ([skill] Step 4, in the coefficient
// domain): for a tile of TC_T middle tokens and the CTA's 128 query heads,
//     S^T[heads x tokens]  = W[heads x slots] . Phi_t^T        (MMA 1, slots = 2F cos/sin)
//     p = online softmax of (S + exact-dim scores)              (CUDA cores, one thread per head)
//     U^T[heads x slots]  += P^T[heads x tokens] . Phi_t        (MMA 2, accumulates over tiles)
// where W holds sigma log2(e) s_f (C_K^T q_c) per slot and Phi_t the unit-amplitude
// cos / sin of the tile's tokens. Operands are fp16: Phi_t lies in [-1, 1]; P is stored as
// 2^12 p, so probabilities down to 2^-26 stay normal (U carries the 2^12 until the record
// is written); W is scaled per head by a power of two to at most 1 in magnitude and split
// into hi + lo (lo = W - hi), so S takes two MMAs (W_hi . Phi^T + W_lo . Phi^T). The score
// error is then ~2^-22 relative and the value error ~2^-12 per term, far inside the 3e-3
// output bar (one plain fp16 or tf32 pass for S would leave only a 5x margin). One buffer per
// tile holds Phi_t as [token][slot] with 128-byte swizzle: MMA 1 reads it as its K-major B
// operand, MMA 2 as its MN-major B operand (the layout compress uses for the cache rows).
//
// Warp roles: warp 0 = TMEM owner and MMA issuer (one thread); warps 1-4 = head threads
// (thread = TMEM lane = query head): exact-dim dot products, online softmax, P rows,
// U rescaling, the split record; warps 5-7 = basis generators (thread = token and a third
// of the frequencies; rotation recurrence over the frequencies, re-seeded every 32 of them
// from the exactly reduced phase). Tiles are double-buffered (Phi, P, S); every wait is
// bounded.
#include "fa_decode_common.cuh"

namespace fa {

constexpr int TC_NH = 128;      // query heads per CTA = MMA M = TMEM lanes
constexpr int TC_T = 32;        // tokens per tile
constexpr int TC_THREADS = 256; // 8 warps
constexpr int TC_GEN = 96;      // generator threads (warps 5-7)

struct TcLayout {
  int w, phi, p, misc, total;  // byte offsets from the 1024-aligned base
};

// W: hi then lo, each [F2/64 atoms][128 heads][64 fp16] (K-major, 128-byte swizzle)
// Phi: 2 buffers of [F2/64 atoms][32 tokens][64 fp16] (128-byte swizzle)
// P: 2 buffers of [128 heads][32 fp16] (K-major, 64-byte swizzle)
__host__ __device__ inline TcLayout tc_layout(int F2) {
  TcLayout L;
  L.w = 0;
  L.phi = L.w + 2 * TC_NH * F2 * 2;
  L.p = L.phi + 2 * TC_T * F2 * 2;
  L.misc = L.p + 2 * TC_NH * TC_T * 2;
  L.total = L.misc + 256 + 1024;  // + alignment slack
  return L;
}

constexpr float TC_P_SCALE = 4096.0f;          // P is stored as 2^12 p
constexpr float TC_P_UNSCALE = 1.0f / 4096.0f;

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

size_t decode_tc_smem_bytes(int F2) { return (size_t)tc_layout(F2).total; }

template <int DE>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int F2 = p.tc_F2;
  const TcLayout Ly = tc_layout(F2);
  uint8_t* Ws = smem + Ly.w;      // hi at Ws, lo at Ws + w_half
  uint8_t* PHI = smem + Ly.phi;   // buffer b at PHI + b * phi_bytes
  uint8_t* PS = smem + Ly.p;      // buffer b at PS + b * p_bytes
  const int w_half = TC_NH * F2 * 2;
  const int phi_bytes = TC_T * F2 * 2;
  const int p_bytes = TC_NH * TC_T * 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.misc);
  uint64_t* phi_full = bars;      // [2] generators -> MMA (count 3)
  uint64_t* phi_free = bars + 2;  // [2] MMA 2 done: Phi and P buffers reusable (commit)
  uint64_t* s_full = bars + 4;    // [2] MMA 1 done (commit)
  uint64_t* p_full = bars + 6;    // [2] head threads -> MMA (count 4)
  uint64_t* u_done = bars + 8;    // last MMA 2 done (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = blockIdx.x / p.n_splits;
  const int sp = blockIdx.x - hg * p.n_splits;
  const int lo = sp * p.split_len;
  const int hi = min(p.M, lo + p.split_len);
  const int ntiles = (hi - lo + TC_T - 1) / TC_T;
  const int M = p.M;
  const long long bhq = (long long)p.B * p.Hq;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&phi_full[b], TC_GEN / 32);
      mbar_init(&phi_free[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 4);
    }
    mbar_init(u_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, p.tc_tmem_cols);
    tmem_relinquish();
  }
  // head threads: W rows, scaled by 2^-e to at most 1 in magnitude, split into fp16 hi / lo
  // and written into the K-major swizzled operand; S is scaled back by 2^e on readout
  const int h = (warp & 3) * 32 + lane;  // TMEM lane of a head thread
  const long long gh = (long long)hg * TC_NH + h;
  const bool is_head = warp >= 1 && warp <= 4;
  const bool hvalid = is_head && gh < bhq;
  float w_unscale = 1.0f;
  if (is_head) {
    const float* wsrc = p.qw + gh * p.qw_stride + FA_HEAD_DIM;
    const int nslot = hvalid ? 2 * p.F_pad : 0;
    float wmax = 0.0f;
    for (int slot = 0; slot < nslot; ++slot) wmax = fmaxf(wmax, fabsf(wsrc[slot]));
    int ex = 0;
    if (wmax > 0.0f) frexpf(wmax, &ex);  // wmax < 2^ex
    const float w_scale = ldexpf(1.0f, -ex);
    w_unscale = ldexpf(1.0f, ex);
    for (int c8 = 0; c8 < F2 / 8; ++c8) {
      uint32_t hv[4], lv[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int slot = c8 * 8 + 2 * e;
        const float a = slot < nslot ? wsrc[slot] * w_scale : 0.0f;
        const float b = slot + 1 < nslot ? wsrc[slot + 1] * w_scale : 0.0f;
        hv[e] = pack_half2(a, b);
        const __half2 hh = *reinterpret_cast<const __half2*>(&hv[e]);
        lv[e] = pack_half2(a - __low2float(hh), b - __high2float(hh));
      }
      const int atom = c8 >> 3, chunk = c8 & 7;
      const int off = atom * (TC_NH * 128) + h * 128 + ((chunk ^ (h & 7)) << 4);
      *reinterpret_cast<uint4*>(Ws + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      *reinterpret_cast<uint4*>(Ws + w_half + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_u = tmem;              // U^T: columns [0, F2)
  const uint32_t tmem_s = tmem + F2;         // S^T buffer b: columns F2 + 32 b

  if (warp == 0) {
    // -------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_f16_f32(TC_NH, TC_T, /*b_mn_major=*/false);
      const uint32_t idesc2 = idesc_f16_f32(TC_NH, F2, /*b_mn_major=*/true);
      const uint32_t w_addr = smem_u32(Ws);
      bool ok = true;
      auto mma1 = [&](int i) {
        const int b = i & 1;
        if (!mbar_wait(&phi_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 2u)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t phi_addr = smem_u32(PHI + b * phi_bytes);
        for (int ks = 0; ks < F2 / 16; ++ks) {
          // 16 slots = 32 bytes further along a swizzled 128-byte row; 64-slot atoms
          const uint32_t koff = (uint32_t)((ks & 3) * 32);
          const uint32_t wa = w_addr + (ks >> 2) * (TC_NH * 128) + koff;
          const uint32_t pa = phi_addr + (ks >> 2) * (TC_T * 128) + koff;
          const uint64_t bd = smem_desc_sw128(pa, 16, 1024);
          mma_f16(tmem_s + 32 * b, smem_desc_sw128(wa, 16, 1024), bd, idesc1, ks > 0 ? 1u : 0u);
          mma_f16(tmem_s + 32 * b, smem_desc_sw128(wa + w_half, 16, 1024), bd, idesc1, 1u);
        }
        mma_commit(&s_full[b]);
      };
      if (ntiles > 0) mma1(0);
      for (int i = 0; i < ntiles && ok; ++i) {
        if (i + 1 < ntiles) {
          mma1(i + 1);
          if (!ok) break;
        }
        const int b = i & 1;
        if (!mbar_wait(&p_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 3u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t p_addr = smem_u32(PS + b * p_bytes);
        const uint32_t phi_addr = smem_u32(PHI + b * phi_bytes);
        for (int ks = 0; ks < TC_T / 16; ++ks) {
          // P: 64-byte rows (32 tokens), 8-row groups 512 bytes apart; 16 tokens = 32 bytes
          const uint32_t pa = p_addr + ks * 32;
          // Phi as MN-major B: 64-slot atoms TC_T * 128 bytes apart (leading), 8-token
          // groups 1024 bytes apart; 16 tokens = two groups
          mma_f16(tmem_u, smem_desc_sw64(pa, 16, 512),
                   smem_desc_sw128(phi_addr + ks * 2048, TC_T * 128, 1024), idesc2,
                   (i > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&phi_free[b]);
      }
      // TMEM is released only after every MMA of this CTA has completed
      mma_commit(u_done);
      const unsigned long long w0 = globaltimer_ns();
      while (!mbar_try_wait(u_done, 0) && globaltimer_ns() - w0 < 2000000000ull) {
      }
    }
  } else if (warp >= 5) {
    // -------------------------------------------------------------------- basis generators
    // thread: token tau of the tile and one third of the frequencies, two per 16-byte store
    const int gt = threadIdx.x - 160;
    const int tau = gt & 31, part = gt >> 5;  // part 0..2
    const int npair = F2 / 4;                 // frequency pairs (f, f+1), f even
    const int per = (npair + 2) / 3;
    const int pa = part * per, pb = min(npair, pa + per);
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      if (i >= 2 &&
          !mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag, WD_DECODE | 4u))
        break;
      const long long tm = (long long)lo + i * TC_T + tau;  // middle-relative token
      uint8_t* base = PHI + b * phi_bytes + tau * 128;
      if (pa < pb) {
        float sa, ca;  // rotation by 2 pi tm / M per frequency step
        phase_sincos(tm % M, M, p.two_over_M, &sa, &ca);
        for (int q0 = pa; q0 < pb; q0 += 16) {
          float s, c;
          phase_sincos(((long long)(2 * q0) * tm) % M, M, p.two_over_M, &s, &c);
          const int q1 = min(pb, q0 + 16);
          for (int q = q0; q < q1; ++q) {
            const float c0 = c, s0 = s;
            float cn = c * ca - s * sa;
            s = s * ca + c * sa;
            c = cn;
            const float c1 = c, s1 = s;
            cn = c * ca - s * sa;
            s = s * ca + c * sa;
            c = cn;
            // slots 4q .. 4q+3: atom 4q / 64, 16-byte chunk (4q % 64) / 8 swizzled by token
            const int atom = q >> 4, chunk = (q & 15) >> 1;
            const int off = atom * (TC_T * 128) + ((chunk ^ (tau & 7)) << 4) + (q & 1) * 8;
            *reinterpret_cast<uint2*>(base + off) = make_uint2(pack_half2(c0, s0), pack_half2(c1, s1));
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_full[b]);
    }
  } else {
    // -------------------------------------------------------------------- head threads
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    const int bi = hvalid ? (int)(gh / p.Hq) : 0;
    const int hq = hvalid ? (int)(gh - (long long)bi * p.Hq) : 0;
    const int g = hq / p.G;
    const long long ebase = (long long)bi * p.e_batch + p.e_off[g];
    const int dle = hvalid ? p.de_ld[g] : 0;
    const bool leader = hvalid && (hq % p.G) == 0;  // prefetches the group's rows
    float qe[DE], acc[DE];
#pragma unroll
    for (int d = 0; d < DE; ++d) {
      qe[d] = (d < dle) ? p.qw[gh * p.qw_stride + d] : 0.0f;
      acc[d] = 0.0f;
    }
    float m = -INFINITY, l = 0.0f;
    constexpr int UT = DE <= 32 ? 2 : 1;  // tokens whose rows are in flight together
    bool ok = true;
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      const int t0 = lo + i * TC_T;
      const int nt = min(TC_T, hi - t0);
      if (leader && i + 1 < ntiles && dle > 0) {
        const int tn = t0 + TC_T;
        const int nb = min(TC_T, hi - tn);
        prefetch_l2_bulk(p.EK + ebase + (long long)tn * dle, (uint32_t)(nb * dle * 2));
        prefetch_l2_bulk(p.EV + ebase + (long long)tn * dle, (uint32_t)(nb * dle * 2));
      }
      ok = mbar_wait(&s_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 5u) && ok;
      __syncwarp();  // tcgen05.ld is warp-collective
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_32x32b_x32(tmem_s + lanebase + 32 * b, sr);
      tmem_ld_wait();
      float sc[TC_T];
#pragma unroll
      for (int t = 0; t < TC_T; ++t) sc[t] = __uint_as_float(sr[t]) * w_unscale;
      // exact dims of the middle tokens
      const __nv_bfloat16* ek = p.EK + ebase + (long long)t0 * dle;
#pragma unroll 1  // bounded loads in flight (register budget)
      for (int t8 = 0; t8 < TC_T; t8 += UT) {
        uint4 rows[UT][DE / 8];
#pragma unroll
        for (int u = 0; u < UT; ++u)
#pragma unroll
          for (int c8 = 0; c8 < DE / 8; ++c8)
            rows[u][c8] = (t8 + u < nt && c8 * 8 < dle)
                              ? *reinterpret_cast<const uint4*>(ek + (long long)(t8 + u) * dle + c8 * 8)
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < UT; ++u) {
          float e = 0.0f;
#pragma unroll
          for (int c8 = 0; c8 < DE / 8; ++c8) {
            float x[8];
            bf16x8_to_f32(rows[u][c8], x);
#pragma unroll
            for (int j = 0; j < 8; ++j) e += qe[c8 * 8 + j] * x[j];
          }
          sc[t8 + u] += e;
        }
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int t = 0; t < TC_T; ++t) {
        if (t >= nt) sc[t] = -INFINITY;
        tmax = fmaxf(tmax, sc[t]);
      }
      const float m_new = fmaxf(m, tmax);
      const float alpha = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
      float psum = 0.0f;
#pragma unroll
      for (int t = 0; t < TC_T; ++t) {
        sc[t] = exp2f(sc[t] - m_new);  // -inf -> 0
        psum += sc[t];
      }
      l = l * alpha + psum;
      m = m_new;
      // U^T rows of heads whose running max rose are rescaled before MMA 2 of this tile
      const bool need = i > 0 && alpha < 1.0f;
      if (__any_sync(0xffffffffu, need)) {
        const bool w_ok = mbar_wait(&phi_free[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u,
                                    abort_flag, WD_DECODE | 6u);
        ok = ok && w_ok;
        __syncwarp();
        tc_fence_after();
        const float a = need ? alpha : 1.0f;
#pragma unroll 1
        for (int c = 0; c < F2 / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
          tmem_st_32x32b_x32(tmem_u + lanebase + c * 32, r);
        }
        tmem_st_wait();
      }
      // exact-dim values
      const __nv_bfloat16* ev = p.EV + ebase + (long long)t0 * dle;
#pragma unroll
      for (int d = 0; d < DE; ++d) acc[d] *= alpha;
#pragma unroll 1  // bounded loads in flight (register budget)
      for (int t8 = 0; t8 < TC_T; t8 += UT) {
        uint4 rows[UT][DE / 8];
#pragma unroll
        for (int u = 0; u < UT; ++u)
#pragma unroll
          for (int c8 = 0; c8 < DE / 8; ++c8)
            rows[u][c8] = (t8 + u < nt && c8 * 8 < dle)
                              ? *reinterpret_cast<const uint4*>(ev + (long long)(t8 + u) * dle + c8 * 8)
                              : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < UT; ++u) {
          const float pv = sc[t8 + u];
#pragma unroll
          for (int c8 = 0; c8 < DE / 8; ++c8) {
            float x[8];
            bf16x8_to_f32(rows[u][c8], x);
#pragma unroll
            for (int j = 0; j < 8; ++j) acc[c8 * 8 + j] += pv * x[j];
          }
        }
      }
      // P^T row of this head (fp16, 2^12 p) into buffer b, once MMA 2 of tile i-2 released it
      if (i >= 2) {
        const bool w_ok = mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag,
                                    WD_DECODE | 7u);
        ok = ok && w_ok;
      }
      // row h: 64 bytes, 16-byte chunk c (tokens 8c .. 8c+7) swizzled by (h >> 1) & 3
      uint8_t* prow = PS + b * p_bytes + h * 64;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t pv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          pv[e] = pack_half2(sc[8 * c + 2 * e] * TC_P_SCALE, sc[8 * c + 2 * e + 1] * TC_P_SCALE);
        *reinterpret_cast<uint4*>(prow + ((c ^ ((h >> 1) & 3)) << 4)) =
            make_uint4(pv[0], pv[1], pv[2], pv[3]);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
    }
    // split record: running max, sum, exact-dim values, U
    const bool done = ntiles == 0 || mbar_wait(u_done, 0, abort_flag, WD_DECODE | 8u);
    __syncwarp();
    tc_fence_after();
    float* rec = p.rec + ((long long)sp * bhq + gh) * p.rec_stride;
    if (hvalid && ok && done) {
      rec[0] = m;
      rec[1] = l;
#pragma unroll
      for (int d = 0; d < DE; ++d)
        if (d < dle) rec[4 + d] = acc[d];
    }
    const int nslot = 2 * p.F_pad;
#pragma unroll 1
    for (int c = 0; c < F2 / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
      tmem_ld_wait();
      if (hvalid && ok && done) {
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int slot = c * 32 + j;
          if (slot < nslot)
            *reinterpret_cast<float4*>(rec + 4 + FA_HEAD_DIM + slot) =
                make_float4(__uint_as_float(r[j]) * TC_P_UNSCALE,
                            __uint_as_float(r[j + 1]) * TC_P_UNSCALE,
                            __uint_as_float(r[j + 2]) * TC_P_UNSCALE,
                            __uint_as_float(r[j + 3]) * TC_P_UNSCALE);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tc_tmem_cols);
  }
}

cudaError_t launch_decode_tc(const DecodeParams& p, int de_max, cudaStream_t stream) {
  const int smem = (int)decode_tc_smem_bytes(p.tc_F2);
  const int heads = p.B * p.Hq;
  const int grid = ((heads + TC_NH - 1) / TC_NH) * p.n_splits;
  cudaError_t e;
  if (de_max <= 32) {
    e = cudaFuncSetAttribute(decode_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<32><<<grid, TC_THREADS, smem, stream>>>(p);
  } else {
    e = cudaFuncSetAttribute(decode_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    decode_tc_kernel<64><<<grid, TC_THREADS, smem, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace fa
