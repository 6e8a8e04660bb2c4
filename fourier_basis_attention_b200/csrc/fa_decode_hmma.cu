// fa_decode_hmma.cu -- split-L decode of the middle span for large k (2F up to 1024 slots)
// with the k-length contractions on warp-level tensor-core MMAs (mma.sync m16n8k16, fp16
// operands, fp32 accumulation); per-KV-head E blocks.
//
// Same mathematics as the other split kernels ([skill] Step 4, in the coefficient domain).
// CTA = 16 query heads (the MMA's M) x a token range, 8 warps, tiles of HM_T = 64 tokens:
//   A. the basis tile Phi_t [64 tokens][F2 slots] (fp16 cos / sin pairs, unit amplitude) is
//      generated in shared memory: thread = frequency, rotation along the tokens, started
//      each tile from the exactly reduced phase; 16-byte chunks swizzled by token so that
//      ldmatrix reads of 8 token rows hit 8 different banks;
//   B. exact-dim scores q_e . E_K[t] on the CUDA cores;
//   C. S = W . Phi_t^T: warp w owns slots [w F2 / 8, (w + 1) F2 / 8) and multiplies its W
//      fragments (registers, fp16 hi + lo: the per-head W is scaled by a power of two to at
//      most 1 and split, so the score keeps ~2^-22 relative precision) with Phi rows loaded
//      by ldmatrix; the eight partial S are summed through shared memory;
//   D. online softmax per head with a lazily raised reference max (only when a tile exceeds
//      it by more than 2^8), P = 2^7 p in fp16;
//   E. U += P . Phi_t: warp w keeps U for its slots in registers (16 heads x F2 / 8 slots);
//   F. exact-dim values acc += p E_V[t] on the CUDA cores; when a tile's E_V rows of the
//      CTA's KV heads fit in HM_EV_BYTES they are staged into shared memory with cp.async
//      at the start of the tile, so their loads overlap phases A-E.
// The split record (m, l, exact-dim values, U) has the layout of the other split kernels,
// so the same combine merges it. The sink / recent rows run in the prologue launch.
#include "fa_decode_common.cuh"

namespace fa {

constexpr int HM_NH = 16;          // query heads per CTA = MMA M
constexpr int HM_T = 64;           // tokens per tile
constexpr int HM_THREADS = 256;    // 8 warps
constexpr int HM_LD = HM_T + 4;    // fp32 row pitch of the [head][token] buffers
constexpr float HM_LAZY = 8.0f;
constexpr float HM_P_SCALE = 128.0f;
constexpr float HM_P_UNSCALE = 1.0f / 128.0f;
constexpr int HM_EV_BYTES = 32768;  // staged E_V rows of one tile

struct HmLayout {
  int phi, red, esc, ph, qe, ev, misc, total;  // byte offsets
};

// phi: [64 tokens][F2] fp16; red: [8 warps][16 heads][HM_LD] fp32 partial scores;
// esc: [16][HM_LD] fp32 exact-dim scores, then p; ph: [16 heads][64 tokens] fp16 (2^7 p,
// chunks swizzled by head); qe: [16][128] fp32 q_e; misc: scales, alpha
__host__ __device__ inline HmLayout hm_layout(int F2) {
  HmLayout L;
  L.phi = 0;
  L.red = L.phi + HM_T * F2 * 2;
  L.esc = L.red + 8 * HM_NH * HM_LD * 4;
  L.ph = L.esc + HM_NH * HM_LD * 4;
  L.qe = L.ph + HM_NH * HM_T * 2;
  L.ev = L.qe + HM_NH * FA_HEAD_DIM * 4;
  L.misc = L.ev + HM_EV_BYTES;
  L.total = L.misc + 4 * HM_NH * 4 + HM_NH * 16;
  return L;
}

size_t decode_hmma_smem_bytes(int F2) { return (size_t)hm_layout(F2).total; }

__device__ __forceinline__ uint32_t hm_pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row)));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(row)));
}

// Byte offset of 16-byte chunk `chunk` of token row `tok` of the Phi tile (F2 slots).
__device__ __forceinline__ int phi_off(int tok, int chunk, int F2) {
  return tok * F2 * 2 + ((chunk ^ (tok & 7)) << 4);
}

template <int KW>  // 16-slot k-steps per warp: F2 = 128 KW
__global__ void __launch_bounds__(HM_THREADS, 1)
    decode_hmma_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int F2 = 128 * KW;
  constexpr int WS = F2 / 8;   // slots per warp
  constexpr int NU = WS / 8;   // 8-slot n-tiles of U per warp
  extern __shared__ __align__(16) uint8_t smem[];
  const HmLayout Ly = hm_layout(F2);
  uint8_t* phi = smem + Ly.phi;
  float* red = reinterpret_cast<float*>(smem + Ly.red);
  float* esc = reinterpret_cast<float*>(smem + Ly.esc);
  uint8_t* ph = smem + Ly.ph;
  float* qe = reinterpret_cast<float*>(smem + Ly.qe);
  float* wsc = reinterpret_cast<float*>(smem + Ly.misc);  // [16] 2^-e (W scale)
  float* wun = wsc + HM_NH;                               // [16] 2^e
  float* alph = wun + HM_NH;                              // [16] alpha of the tile
  uint8_t* ev = smem + Ly.ev;                             // [KV head][64 tokens][evld] bf16
  long long* kvb = reinterpret_cast<long long*>(alph + HM_NH);  // [16 / G] E offsets
  int* kvd = reinterpret_cast<int*>(kvb + HM_NH);               // [16 / G] de_ld

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int hs = blockIdx.x / p.n_splits, sp = blockIdx.x - (blockIdx.x / p.n_splits) * p.n_splits;
  const int lo = sp * p.split_len;
  const int hi = min(p.M, lo + p.split_len);
  const int ntiles = (hi - lo + HM_T - 1) / HM_T;
  const int P = p.P;  // basis period
  const long long bhq = (long long)p.B * p.Hq;
  const long long gh0 = (long long)hs * HM_NH;  // first query head of the CTA
  const int nvh = (int)max(0LL, min((long long)HM_NH, bhq - gh0));
  const int nslot = 2 * p.F_pad;

  // q_e of the 16 heads and the per-head W scale
  for (int idx = tid; idx < HM_NH * FA_HEAD_DIM; idx += HM_THREADS) {
    const int h = idx >> 7, d = idx & 127;
    qe[idx] = h < nvh ? p.qw[(gh0 + h) * p.qw_stride + d] : 0.0f;
  }
  const int nkv = HM_NH / p.G;  // KV heads of the CTA (G divides 16)
  if (tid < nkv) {
    const long long gh = gh0 + (long long)tid * p.G;
    if (gh < bhq) {
      const int bb = (int)(gh / p.Hq), gg = (int)(gh - (long long)bb * p.Hq) / p.G;
      kvb[tid] = (long long)bb * p.e_batch + p.e_off[gg];
      kvd[tid] = p.de_ld[gg];
    } else {
      kvb[tid] = 0;
      kvd[tid] = 0;
    }
  }
  // E_V rows of a tile staged in shared memory when they fit (row pitch evld elements)
  int evld = 8;
  for (int g2 = 0; g2 < nkv; ++g2) {
    const long long gh = gh0 + (long long)g2 * p.G;
    if (gh < bhq) {
      const int bb = (int)(gh / p.Hq), gg = (int)(gh - (long long)bb * p.Hq) / p.G;
      evld = max(evld, p.de_ld[gg]);
    }
  }
  const bool stage = nkv * HM_T * evld * 2 <= HM_EV_BYTES;
  if (tid < HM_NH) {
    float wmax = 0.0f;
    if (tid < nvh) {
      const float* w = p.qw + (gh0 + tid) * p.qw_stride + FA_HEAD_DIM;
      for (int s = 0; s < nslot; ++s) wmax = fmaxf(wmax, fabsf(w[s]));
    }
    int ex = 0;
    if (wmax > 0.0f) frexpf(wmax, &ex);
    wsc[tid] = ldexpf(1.0f, -ex);
    wun[tid] = ldexpf(1.0f, ex);
  }
  __syncthreads();

  // W fragments of this warp's slots: A[row = head][k = slot], a0 (row g, k 2t..2t+1),
  // a1 (row g + 8), a2 (row g, k + 8), a3 (row g + 8, k + 8); fp16 hi and lo
  const int g = lane >> 2, t4 = lane & 3;
  const int wbase = warp * WS;
  uint32_t ahi[KW][4], alo[KW][4];
#pragma unroll
  for (int ks = 0; ks < KW; ++ks)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = g + ((i & 1) ? 8 : 0);
      const int s0 = wbase + ks * 16 + ((i & 2) ? 8 : 0) + 2 * t4;
      float a = 0.0f, b = 0.0f;
      if (row < nvh) {
        const float* w = p.qw + (gh0 + row) * p.qw_stride + FA_HEAD_DIM;
        a = s0 < nslot ? w[s0] * wsc[row] : 0.0f;
        b = s0 + 1 < nslot ? w[s0 + 1] * wsc[row] : 0.0f;
      }
      ahi[ks][i] = hm_pack_half2(a, b);
      const __half2 hh = *reinterpret_cast<const __half2*>(&ahi[ks][i]);
      alo[ks][i] = hm_pack_half2(a - __low2float(hh), b - __high2float(hh));
    }
  float uacc[NU][4];
#pragma unroll
  for (int n = 0; n < NU; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) uacc[n][e] = 0.0f;

  // softmax state: thread (head sh, quarter-lane sq) of phase D
  const int sh = tid >> 4, sq = tid & 15;
  float m = -INFINITY, l = 0.0f;
  // exact-dim values: thread (head vh, 8-dim chunk vc) of phase F
  const int vh = tid >> 4, vc = tid & 15;
  float acc8[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) acc8[e] = 0.0f;
  int v_de = 0, v_ld = 0;
  long long v_base = 0;
  if (vh < nvh) {
    const long long gh = gh0 + vh;
    const int bb = (int)(gh / p.Hq), gg = (int)(gh - (long long)bb * p.Hq) / p.G;
    v_de = p.de[gg];
    v_ld = p.de_ld[gg];
    v_base = (long long)bb * p.e_batch + p.e_off[gg];
  }

  // phase-A rotation of this thread's frequencies (f = tid, tid + 256, ...)
  constexpr int NFT = (F2 / 2 + HM_THREADS - 1) / HM_THREADS;
  float ra[NFT], rb[NFT];
#pragma unroll
  for (int u = 0; u < NFT; ++u) {
    const int f = tid + HM_THREADS * u;
    ra[u] = 1.0f;
    rb[u] = 0.0f;
    if (f < F2 / 2) phase_sincos(f % P, P, p.two_over_P, &rb[u], &ra[u]);
  }

  for (int i = 0; i < ntiles; ++i) {
    const int t0 = lo + i * HM_T;
    const int nt = min(HM_T, hi - t0);
    if (stage) {  // this tile's E_V rows -> shared memory, landing while A-E run
      const int cpr = evld / 8;  // 16-byte chunks per staged row
      for (int idx = tid; idx < nkv * HM_T * cpr; idx += HM_THREADS) {
        const int kv = idx / (HM_T * cpr), rem = idx - kv * (HM_T * cpr);
        const int t = rem / cpr, c = rem - (rem / cpr) * cpr;
        const int dle = kvd[kv];
        if (t < nt && 8 * c < dle)
          cp_async16(ev + ((kv * HM_T + t) * evld + 8 * c) * 2,
                     p.EV + kvb[kv] + (long long)(t0 + t) * dle + 8 * c);
      }
      cp_async_commit();
    }
    // ---- A: basis tile
#pragma unroll
    for (int u = 0; u < NFT; ++u) {
      const int f = tid + HM_THREADS * u;
      if (f < F2 / 2) {
        float s, c;
        phase_sincos(((long long)f * t0) % P, P, p.two_over_P, &s, &c);
        const int chunk = f >> 2, within = (f & 3) * 4;
#pragma unroll 8
        for (int tau = 0; tau < HM_T; ++tau) {
          *reinterpret_cast<uint32_t*>(phi + phi_off(tau, chunk, F2) + within) = hm_pack_half2(c, s);
          const float cn = c * ra[u] - s * rb[u];
          s = s * ra[u] + c * rb[u];
          c = cn;
        }
      }
    }
    // ---- B: exact-dim scores, thread = (token, 4 heads)
    {
      const int t = tid & (HM_T - 1), hg = tid >> 6;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int h = hg * 4 + j;
        float e = 0.0f;
        if (h < nvh && t < nt) {
          const long long gh = gh0 + h;
          const int bb = (int)(gh / p.Hq), gg = (int)(gh - (long long)bb * p.Hq) / p.G;
          const int dle = p.de_ld[gg];
          const __nv_bfloat16* row = p.EK + (long long)bb * p.e_batch + p.e_off[gg] +
                                     (long long)(t0 + t) * dle;
          const float* qh = qe + h * FA_HEAD_DIM;
          for (int c8 = 0; c8 < dle; c8 += 8) {
            float x[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(row + c8), x);
#pragma unroll
            for (int u = 0; u < 8; ++u) e += qh[c8 + u] * x[u];
          }
        }
        esc[h * HM_LD + t] = e;
      }
    }
    __syncthreads();
    // ---- C: partial S of this warp's slots
#pragma unroll 1
    for (int j = 0; j < HM_T / 8; ++j) {  // 8-token n-tiles
      float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      const int tok = 8 * j + (lane & 7);
#pragma unroll
      for (int ks = 0; ks < KW; ks += 2) {
        // matrices: (k-step ks: slots +0..7, +8..15), (k-step ks + 1: +16..23, +24..31)
        const int chunk = (wbase + ks * 16) / 8 + (lane >> 3);
        uint32_t bq[4];
        ldsm_x4(bq, phi + phi_off(tok, chunk, F2));
        mma_f16_16816(d, ahi[ks], bq[0], bq[1]);
        mma_f16_16816(d, alo[ks], bq[0], bq[1]);
        if (ks + 1 < KW) {
          mma_f16_16816(d, ahi[ks + 1], bq[2], bq[3]);
          mma_f16_16816(d, alo[ks + 1], bq[2], bq[3]);
        }
      }
      float* r0 = red + (warp * HM_NH + g) * HM_LD + 8 * j + 2 * t4;
      r0[0] = d[0];
      r0[1] = d[1];
      r0[8 * HM_LD] = d[2];
      r0[8 * HM_LD + 1] = d[3];
    }
    __syncthreads();
    // ---- D: softmax, thread (head sh, tokens 4 sq .. 4 sq + 3)
    {
      float s4[4];
      float tmax = -INFINITY;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int t = 4 * sq + u;
        float v = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) v += red[(w * HM_NH + sh) * HM_LD + t];
        v = sh < nvh ? v * wun[sh] + esc[sh * HM_LD + t] : 0.0f;
        s4[u] = t < nt ? v : -INFINITY;
        tmax = fmaxf(tmax, s4[u]);
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, o));
      const float m_new = (tmax > m + HM_LAZY) ? tmax : m;
      const float alpha = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
      float psum = 0.0f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        s4[u] = exp2f(s4[u] - m_new);
        psum += s4[u];
      }
#pragma unroll
      for (int o = 8; o > 0; o >>= 1) psum += __shfl_xor_sync(0xffffffffu, psum, o);
      l = l * alpha + psum;
      m = m_new;
      // P row sh: 128 bytes, 16-byte chunk (tokens 8c .. 8c+7) swizzled by the head
      const int c = sq >> 1;
      *reinterpret_cast<uint2*>(ph + sh * 128 + ((c ^ (sh & 7)) << 4) + (sq & 1) * 8) =
          make_uint2(hm_pack_half2(s4[0] * HM_P_SCALE, s4[1] * HM_P_SCALE),
                     hm_pack_half2(s4[2] * HM_P_SCALE, s4[3] * HM_P_SCALE));
#pragma unroll
      for (int u = 0; u < 4; ++u) esc[sh * HM_LD + 4 * sq + u] = s4[u];
      if (sq == 0) alph[sh] = alpha;
    }
    if (stage) cp_async_wait<0>();  // this thread's staged rows landed
    __syncthreads();
    // ---- E: U += P . Phi over this warp's slots
    {
      const float a_lo = alph[g], a_hi = alph[g + 8];
#pragma unroll
      for (int n = 0; n < NU; ++n) {
        uacc[n][0] *= a_lo;
        uacc[n][1] *= a_lo;
        uacc[n][2] *= a_hi;
        uacc[n][3] *= a_hi;
      }
#pragma unroll
      for (int kk = 0; kk < HM_T / 16; ++kk) {
        // A = P: matrices (heads 0-7 | 8-15) x (tokens 16 kk + 0..7 | + 8..15)
        const int mi = lane >> 3;
        const int head = (lane & 7) + ((mi & 1) ? 8 : 0);
        const int pchunk = 2 * kk + (mi >> 1);
        uint32_t a[4];
        ldsm_x4(a, ph + head * 128 + ((pchunk ^ (head & 7)) << 4));
        // B = Phi rows (tokens) 16 kk + 0..15 of this warp's slots, transposed on load
        const int tok = 16 * kk + (lane & 7) + ((mi & 1) ? 8 : 0);
#pragma unroll
        for (int n = 0; n < NU; n += 2) {
          const int chunk = (wbase + 8 * n) / 8 + (mi >> 1);
          uint32_t bq[4];
          ldsm_x4_trans(bq, phi + phi_off(tok, chunk, F2));
          mma_f16_16816(uacc[n], a, bq[0], bq[1]);
          mma_f16_16816(uacc[n + 1], a, bq[2], bq[3]);
        }
      }
    }
    // ---- F: exact-dim values, thread (head vh, dims 8 vc .. 8 vc + 7)
    {
      const float a = alph[vh];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc8[e] *= a;
      if (vh < nvh && 8 * vc < v_de) {
        const float* pv = esc + vh * HM_LD;
        if (stage) {
          const uint8_t* col = ev + ((vh / p.G) * HM_T * evld + 8 * vc) * 2;
#pragma unroll 8
          for (int t = 0; t < nt; ++t) {
            float x[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(col + t * evld * 2), x);
            const float pt = pv[t];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] += pt * x[e];
          }
        } else {
          const __nv_bfloat16* col = p.EV + v_base + (long long)t0 * v_ld + 8 * vc;
#pragma unroll 8
          for (int t = 0; t < nt; ++t) {
            float x[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4*>(col + (long long)t * v_ld), x);
            const float pt = pv[t];
#pragma unroll
            for (int e = 0; e < 8; ++e) acc8[e] += pt * x[e];
          }
        }
      }
    }
    __syncthreads();  // Phi, P, p and the partial scores are rewritten by the next tile
  }

  // ---- split record: m, l, exact-dim values, U (unscaled from 2^7 p)
  float* rec_base = p.rec + ((long long)sp * bhq + gh0) * p.rec_stride;
  if (sq == 0 && sh < nvh) {
    rec_base[(long long)sh * p.rec_stride + 0] = m;
    rec_base[(long long)sh * p.rec_stride + 1] = l;
  }
  if (vh < nvh) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
      if (8 * vc + e < v_de) rec_base[(long long)vh * p.rec_stride + 4 + 8 * vc + e] = acc8[e];
  }
#pragma unroll
  for (int n = 0; n < NU; ++n) {
    const int s0 = wbase + 8 * n + 2 * t4;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int row = g + 8 * half;
      if (row < nvh) {
        float* r = rec_base + (long long)row * p.rec_stride + 4 + FA_HEAD_DIM;
        if (s0 < nslot) r[s0] = uacc[n][2 * half] * HM_P_UNSCALE;
        if (s0 + 1 < nslot) r[s0 + 1] = uacc[n][2 * half + 1] * HM_P_UNSCALE;
      }
    }
  }
}

template <int KW>
static cudaError_t launch_hm(const DecodeParams& p, int grid, cudaStream_t stream) {
  const int smem = (int)decode_hmma_smem_bytes(128 * KW);
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(decode_hmma_kernel<KW>), smem);
  if (e != cudaSuccess) return e;
  decode_hmma_kernel<KW><<<grid, HM_THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode_hmma(const DecodeParams& p, int F2, cudaStream_t stream) {
  const int heads = p.B * p.Hq;
  const int grid = ((heads + HM_NH - 1) / HM_NH) * p.n_splits;
  switch (F2) {  // the plans sent here have 256 <= k <= 1023
    case 512: return launch_hm<4>(p, grid, stream);
    case 1024: return launch_hm<8>(p, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace fa
