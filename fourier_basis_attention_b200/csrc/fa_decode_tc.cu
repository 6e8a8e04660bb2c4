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
// 2^7 p with p <= 2^8 (lazy max below), so it stays normal down to p = 2^-21 (U carries
// the 2^7 until the record is written); W is scaled per head by a power of two to at most
// 1 in magnitude and split into hi + lo (lo = W - hi), so S takes two MMAs
// (W_hi . Phi^T with W_hi in shared memory + W_lo . Phi^T with W_lo in tensor memory). The score error is then ~2^-22 relative and the value
// error ~2^-12 per term, far inside the 3e-3 output bar (one plain fp16 or tf32 pass for S
// would leave only a 5x margin). One buffer per tile holds Phi_t as [token][slot] with
// 128-byte swizzle: MMA 1 reads it as its K-major B operand, MMA 2 as its MN-major B
// operand (the layout compress uses for the cache rows).
//
// Warp roles: warp 0 = TMEM owner and MMA issuer (one thread); warps 1-8 = head warps, two
// per TMEM lane quadrant (warps w and w + 4 share quadrant w & 3, each taking 16 of its 32
// query heads; the pair exchanges its rescale factors through shared memory and one of them
// rescales the quadrant's U rows); warps 9-11 = basis generators
// (thread = frequency; rotation recurrence along the tile's tokens, started each tile from
// the exactly reduced phase). Tiles are double-buffered (Phi, P, S); every wait is bounded.
//
// Exact dims: this kernel runs on token-major E (the plan lays E out so that token t of a
// batch is one row holding every KV head's retained dims, w = 8, 16 or 32 per head). Per
// token a head warp needs the w-element slices of its 32 / G KV heads, lane = (KV head,
// 16-byte chunk): coalesced row segments. Each lane streams its chunks, step after step
// (K phase, V phase, next tile), into its own slots of a per-warp shared-memory ring with
// 16-byte asynchronous copies, TC_RING steps ahead of use (one commit group per step), and
// reads them back; the G query heads of a KV head share each chunk.
// Dot products are reduced over a KV head's chunk lanes with shuffles and handed to the
// head lanes through a per-warp [head][token] buffer, which then carries p back; the value
// accumulator stays distributed (lane = KV head, chunk, query head) until the record is
// written. Softmax, P rows, U rescaling and (m, l) are per head lane.
//
// The sink / recent rows run on the CUDA cores as extra CTAs of the prologue launch.
#include "fa_decode_common.cuh"

namespace fa {

constexpr int TC_NH = 128;      // query heads per CTA = MMA M = TMEM lanes
constexpr int TC_T = 32;        // tokens per tile
constexpr int TC_THREADS = 384; // 12 warps
constexpr int TC_GEN = 96;      // generator threads (warps 9-11)

// The reference max is raised lazily: only when a tile's max exceeds it by more than
// TC_LAZY (log2 units) are U, the value accumulator and the sum rescaled, so the head
// warps rarely wait for the previous tile's MMA 2. p = 2^(s - m_ref) <= 2^8, stored as
// 2^7 p <= 2^15 in fp16.
constexpr float TC_LAZY = 8.0f;
constexpr float TC_P_SCALE = 128.0f;
constexpr float TC_P_UNSCALE = 1.0f / 128.0f;

constexpr int TC_XS_LD = 33;    // row pitch (floats) of the per-warp [head][token] buffer
constexpr int TC_RING_BYTES = 24576;       // exact-dim ring per head warp
constexpr int TC_RING_BYTES_WIDE = 32768;  // the same with up to 128 basis slots (room to spare)

// Ring bytes per head warp for F2 basis slots: the deeper ring where W and Phi leave room
// (measured: 12% faster at G = 4 with 16 instead of 12 KB-scale steps in flight).
__host__ __device__ constexpr int tc_ring_bytes(int F2) {
  return F2 <= 128 ? TC_RING_BYTES_WIDE : TC_RING_BYTES;
}

struct TcLayout {
  int w, phi, p, xs, ring, misc, total;  // byte offsets from the 1024-aligned base
};

// W_hi: [F2/64 atoms][128 heads][64 fp16] (K-major, 128-byte swizzle); W_lo lives in TMEM
// Phi: 2 buffers of [F2/64 atoms][32 tokens][64 fp16] (128-byte swizzle)
// P: 2 buffers of [128 heads][32 fp16] (K-major, 64-byte swizzle)
// xs: per head warp [32 heads][TC_XS_LD] fp32: exact-dim scores, then p, of the tile
// ring: per head warp tc_ring_bytes(F2): steps of 512 NI bytes (one 16-byte chunk per lane
//   and load)
// misc: pipeline mbarriers, TMEM slot, abort flag
__host__ __device__ inline TcLayout tc_layout(int F2) {
  TcLayout L;
  L.w = 0;
  L.phi = L.w + TC_NH * F2 * 2;
  L.p = L.phi + 2 * TC_T * F2 * 2;
  L.xs = L.p + 2 * TC_NH * TC_T * 2;
  L.ring = L.xs + 4 * 32 * TC_XS_LD * 4;
  L.misc = L.ring + 4 * tc_ring_bytes(F2);
  L.total = L.misc + 256 + 2 * 4 * 32 * 4 + 1024;  // + rescale factors + alignment slack
  return L;
}

size_t decode_tc_smem_bytes(int F2, int de_slot, int G) {
  (void)de_slot;
  (void)G;
  return (size_t)tc_layout(F2).total;
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Lane layout of a head warp's exact-dim work. CPS = 16-byte chunks per KV-head slice of
// a token row (w / 8), G = query heads per KV head. Per step the warp covers TT tokens;
// lane l, load r handles chunk (32 r + l) % CH: KV head / CPS, chunk % CPS, and token
// l / CH of the step (all warp-local).
template <int CPS, int G, int RB>
struct EMap {
  static constexpr int NK = 16 / G;                                  // KV heads per warp
  static constexpr int CH = CPS > 0 ? NK * CPS : 32;                 // chunks per token
  static constexpr int TT = CH >= 32 ? 1 : 32 / CH;                  // tokens per step
  static constexpr int NI = CH >= 32 ? CH / 32 : 1;                  // loads per lane per step
  static constexpr int NS = TC_T / TT;                               // steps per tile
  static constexpr int CPS1 = CPS > 0 ? CPS : 1;
  static constexpr int RING = RB / (512 * NI);                      // steps in flight
  // exact-dim scores on the warp-level bf16 MMA: one load per lane and step, 8 tokens per MMA
  static constexpr bool KMMA = CPS > 0 && NI == 1 && RING >= 2 * (8 / TT);
  static constexpr int SPG = 8 / TT;                                 // steps per 8 tokens
  static constexpr int KS = CPS >= 2 ? CPS / 2 : 1;                  // 16-dim k-steps
};

template <int CPS, int G, int RB>
__global__ void __launch_bounds__(TC_THREADS, 1)
    decode_tc_kernel(const __grid_constant__ DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, formed by pointer arithmetic on smem_raw so that the compiler
  // keeps it (and everything derived from it) in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int cta = blockIdx.x;
  const int F2 = p.tc_F2;
  const TcLayout Ly = tc_layout(F2);
  uint8_t* Ws = smem + Ly.w;      // W_hi
  uint8_t* PHI = smem + Ly.phi;   // buffer b at PHI + b * phi_bytes
  uint8_t* PS = smem + Ly.p;      // buffer b at PS + b * p_bytes
  const int phi_bytes = TC_T * F2 * 2;
  const int p_bytes = TC_NH * TC_T * 2;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.misc);
  uint64_t* phi_full = bars;      // [2] generators -> MMA (count 3)
  uint64_t* phi_free = bars + 2;  // [2] MMA 2 done: Phi and P buffers reusable (commit)
  uint64_t* s_full = bars + 4;    // [2] MMA 1 done (commit)
  uint64_t* p_full = bars + 6;    // [2] head warps -> MMA (count 4)
  uint64_t* u_done = bars + 8;    // last MMA 2 done (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 9);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hg = cta / p.n_splits;
  const int sp = cta - hg * p.n_splits;
  const int lo = sp * p.split_len;
  const int hi = min(p.M, lo + p.split_len);
  const int ntiles = (hi - lo + TC_T - 1) / TC_T;
  const int P = p.P;  // basis period
  const long long bhq = (long long)p.B * p.Hq;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&phi_full[b], TC_GEN / 32);
      mbar_init(&phi_free[b], 1);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 8);
    }
    mbar_init(u_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, p.tc_tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_u = tmem;              // U^T: columns [0, F2)
  const uint32_t tmem_s = tmem + F2;         // S^T buffer b: columns F2 + 32 b
  const uint32_t tmem_wlo = tmem + F2 + 64;  // W_lo: columns [F2 + 64, F2 + 64 + F2 / 2)
  // head warps: W rows, scaled by 2^-e to at most 1 in magnitude, split into fp16 hi (the
  // K-major swizzled shared operand) and lo (TMEM row = this head's lane, two slots per
  // column); S is scaled back by 2^e on readout
  const int h = (warp & 3) * 32 + lane;  // TMEM lane of a head thread
  const long long gh = (long long)hg * TC_NH + h;
  // two head warps per TMEM lane quadrant: warps 1-4 (half 0) and 5-8 (half 1) both serve
  // quadrant warp & 3; warps 1-4 also write W
  const bool any_head = warp >= 1 && warp <= 8;
  const bool is_head = warp >= 1 && warp <= 4;
  const bool qvalid = any_head && gh < bhq;  // the quadrant row of this lane is a query head
  float w_unscale = 1.0f;
  if (any_head) {
    const float* wsrc = p.qw + gh * p.qw_stride + FA_HEAD_DIM;
    const int nslot = qvalid ? 2 * p.F_pad : 0;
    float wmax = 0.0f;
    for (int slot = 0; slot < nslot; ++slot) wmax = fmaxf(wmax, fabsf(wsrc[slot]));
    int ex = 0;
    if (wmax > 0.0f) frexpf(wmax, &ex);  // wmax < 2^ex
    const float w_scale = ldexpf(1.0f, -ex);
    w_unscale = ldexpf(1.0f, ex);
    if (is_head) {
    const uint32_t lanebase_w = (uint32_t)((warp & 3) * 32) << 16;
    for (int c64 = 0; c64 < F2 / 64; ++c64) {  // 64 slots: one swizzle atom, 32 TMEM columns
      uint32_t lo32[32];
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t hv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int slot = c64 * 64 + c8 * 8 + 2 * e;
          const float a = slot < nslot ? wsrc[slot] * w_scale : 0.0f;
          const float b = slot + 1 < nslot ? wsrc[slot + 1] * w_scale : 0.0f;
          hv[e] = pack_half2(a, b);
          const __half2 hh = *reinterpret_cast<const __half2*>(&hv[e]);
          lo32[c8 * 4 + e] = pack_half2(a - __low2float(hh), b - __high2float(hh));
        }
        const int off = c64 * (TC_NH * 128) + h * 128 + ((c8 ^ (h & 7)) << 4);
        *reinterpret_cast<uint4*>(Ws + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      tmem_st_32x32b_x32(tmem_wlo + lanebase_w + c64 * 32, lo32);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // -------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_f16_f32(TC_NH, TC_T, /*b_mn_major=*/false);
      const uint32_t idesc2 = idesc_f16_f32(TC_NH, F2, /*b_mn_major=*/true);
      // descriptors of buffer 0; a byte offset x inside the (< 256 KB) shared window adds
      // x >> 4 to the start-address field
      const uint64_t d_w = smem_desc_sw128(smem_u32(Ws), 16, 1024);
      // Phi as K-major B of MMA 1: 8-token groups 1024 bytes apart, 64-slot atoms
      const uint64_t d_phik = smem_desc_sw128(smem_u32(PHI), 16, 1024);
      // Phi as MN-major B of MMA 2: 64-slot atoms TC_T * 128 bytes apart (leading), 8-token
      // groups 1024 bytes apart
      const uint64_t d_phin = smem_desc_sw128(smem_u32(PHI), TC_T * 128, 1024);
      // P: 64-byte rows (32 tokens), 8-row groups 512 bytes apart
      const uint64_t d_p = smem_desc_sw64(smem_u32(PS), 16, 512);
      const int nks = F2 / 16;
      bool ok = true;
      auto mma1 = [&](int i) {
        const int b = i & 1;
        if (!mbar_wait(&phi_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 2u)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t dphi = d_phik + (uint64_t)((b * phi_bytes) >> 4);
        const uint32_t ts = tmem_s + 32 * b;
#pragma unroll 4
        for (int ks = 0; ks < nks; ++ks) {
          // 16 slots = 32 bytes further along a swizzled 128-byte row; 64-slot atoms
          const uint32_t ow = (uint32_t)(((ks >> 2) * (TC_NH * 128) + (ks & 3) * 32) >> 4);
          const uint32_t op = (uint32_t)(((ks >> 2) * (TC_T * 128) + (ks & 3) * 32) >> 4);
          mma_f16(ts, d_w + ow, dphi + op, idesc1, ks > 0 ? 1u : 0u);
          mma_f16_ta(ts, tmem_wlo + 8 * ks, dphi + op, idesc1, 1u);  // 16 slots = 8 columns
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
        // 16 tokens per MMA: 32 bytes along the P rows, two 8-token groups of Phi
#pragma unroll
        for (int ks = 0; ks < TC_T / 16; ++ks)
          mma_f16(tmem_u, d_p + (uint64_t)((b * p_bytes + ks * 32) >> 4),
                  d_phin + (uint64_t)((b * phi_bytes + ks * 2048) >> 4), idesc2,
                  (i > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&phi_free[b]);
      }
      // TMEM is released only after every MMA of this CTA has completed
      mma_commit(u_done);
      const unsigned long long w0 = globaltimer_ns();
      while (!mbar_try_wait(u_done, 0) && globaltimer_ns() - w0 < 2000000000ull) {
      }
    }
  } else if (warp >= 9) {
    // -------------------------------------------------------------------- basis generators
    // thread gt: frequencies gt and gt + 96; per tile the unit phasor of f (t0 + tau) / M
    // for tau = 0 .. 31 by rotation, started from the exactly reduced phase f t0 mod M.
    // Slots 2f (cos) and 2f + 1 (sin) are one fp16 pair: atom f / 32, byte 4 (f % 32) of
    // the token's 128-byte row, 16-byte chunk swizzled by the token.
    const int gt = threadIdx.x - 288;
    const int nf = F2 / 2;
    float ra[2], rb[2];  // cos, sin of 2 pi f / P
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = gt + TC_GEN * u;
      ra[u] = 1.0f;
      rb[u] = 0.0f;
      if (f < nf) phase_sincos(f % P, P, p.two_over_P, &rb[u], &ra[u]);
    }
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      if (i >= 2 &&
          !mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag, WD_DECODE | 4u))
        break;
      const long long tm0 = (long long)lo + i * TC_T;  // middle-relative first token
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int f = gt + TC_GEN * u;
        if (f < nf) {
          float s, c;
          phase_sincos(((long long)f * tm0) % P, P, p.two_over_P, &s, &c);
          uint8_t* base = PHI + b * phi_bytes + (f >> 5) * (TC_T * 128) + 4 * (f & 3);
          const int chunk = (f & 31) >> 2;
#pragma unroll 8
          for (int tau = 0; tau < TC_T; ++tau) {
            *reinterpret_cast<uint32_t*>(base + tau * 128 + ((chunk ^ (tau & 7)) << 4)) =
                pack_half2(c, s);
            const float cn = c * ra[u] - s * rb[u];
            s = s * ra[u] + c * rb[u];
            c = cn;
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&phi_full[b]);
    }
  } else {
    // -------------------------------------------------------------------- head warps
    // this warp: query heads [16 hf, 16 hf + 16) of TMEM lane quadrant warp & 3, half of the
    // quadrant's ring space; its softmax lanes are lanes 16 hf .. 16 hf + 15 (`mine`)
    using EM = EMap<CPS, G, RB / 2>;
    constexpr int NI = EM::NI;
    const int hf = (warp - 1) >> 2;
    const int pair = (warp - 1) & 3;
    const bool mine = (lane >> 4) == hf;
    const bool hvalid = mine && qvalid;
    const uint32_t lanebase = (uint32_t)((warp & 3) * 32) << 16;
    const long long gbase = (long long)hg * TC_NH + (warp & 3) * 32 + 16 * hf;  // warp's first head
    const int nvalid = (int)max(0LL, min(16LL, bhq - gbase));
    // rescale factors of the pair's 32 heads, by tile parity (half 1 -> half 0)
    float* al_s = reinterpret_cast<float*>(smem + Ly.misc + 256);
    const int tau_l = EM::TT > 1 ? lane / EM::CH : 0;  // token of this lane within a step
    // per load r: the lane's KV head (warp-local), its element offset, q_e, accumulator
    int kap[NI], c8r[NI], de_r[NI];
    bool ev[NI];
    long long eoff[NI];
    float2 qv[NI][G][4];    // q_e (scaled by sigma log2 e) of the lane's chunk, in pairs
    float2 accv[NI][G][4];  // value accumulator of the lane's chunk, in pairs
#pragma unroll
    for (int r = 0; r < NI; ++r) {
      const int q = (32 * r + lane) % EM::CH;
      const int k_ = q / EM::CPS1;
      const int c_ = q % EM::CPS1;
      kap[r] = k_;
      c8r[r] = c_ * 8;
      ev[r] = CPS > 0 && k_ * G < nvalid;
      const long long gh0 = gbase + (long long)k_ * G;
      const int bb = ev[r] ? (int)(gh0 / p.Hq) : 0;
      const int gg = ev[r] ? (int)(gh0 - (long long)bb * p.Hq) / G : 0;
      eoff[r] = (long long)bb * p.e_batch + p.e_off[gg] + c_ * 8;
      de_r[r] = ev[r] ? p.de[gg] - c_ * 8 : 0;  // valid dims of this chunk (may be <= 0)
#pragma unroll
      for (int hq = 0; hq < G; ++hq)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float* qe = p.qw + (gh0 + hq) * p.qw_stride + c_ * 8 + 2 * e;  // zero past de
          qv[r][hq][e] = ev[r] ? make_float2(qe[0], qe[1]) : make_float2(0.0f, 0.0f);
          accv[r][hq][e] = make_float2(0.0f, 0.0f);
        }
    }
    // bf16 query rows for the MMA scores: A[row][k] = q (unscaled, exact in bf16) of query
    // head `row` of KV head kv at retained dim k (rows >= G zero); this lane holds row
    // lane / 4, dims 2 (lane % 4) + {0, 1} and + {8, 9} of each 16-dim k-step
    uint32_t aq[EM::KMMA ? EM::NK : 1][EM::KS][2];
    if constexpr (EM::KMMA) {
      const int ar = lane >> 2, ac = (lane & 3) * 2;
#pragma unroll
      for (int kv = 0; kv < EM::NK; ++kv) {
        const long long gh0 = gbase + (long long)kv * G;
        const bool av = kv * G < nvalid && ar < G;
        const int bb = av ? (int)(gh0 / p.Hq) : 0;
        const int gg = av ? (int)(gh0 - (long long)bb * p.Hq) / G : 0;
#pragma unroll
        for (int ks = 0; ks < EM::KS; ++ks)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t pr = 0;
#pragma unroll
            for (int u2 = 0; u2 < 2; ++u2) {
              const int d = ks * 16 + hh * 8 + ac + u2;  // retained-dim index
              if (av && d < p.de[gg])
                pr |= (uint32_t)__bfloat16_as_ushort(
                          p.q[(gh0 + ar) * FA_HEAD_DIM + p.perm[gg][p.dc[gg] + d]])
                      << (16 * u2);
            }
            aq[kv][ks][hh] = pr;
          }
      }
    }
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    // the quadrant's [32 heads][token] buffer; this warp's rows start at row 16 hf
    float* xsq = reinterpret_cast<float*>(smem + Ly.xs) + pair * 32 * TC_XS_LD;
    float* xs = xsq + 16 * hf * TC_XS_LD;
    const int c_first = ((lane % EM::CH) % EM::CPS1) == 0;  // first chunk lane of its KV head

    // exact-dim ring: global step gs = (tile, phase K / V, step) uses slot gs % RING; chunk c
    // of a slot (lane l's load r: c = 32 r + l) sits at 16-byte position c ^ (token & 7),
    // so the 8 token rows an ldmatrix reads from 8 slots fall in 8 different banks
    constexpr int RING = EM::RING;
    constexpr int STEP = 512 * NI;
    // steps per pass of the CUDA-core exact-dim loops (independent chains in flight)
    constexpr int SB = (EM::NS % 2 == 0 && RING >= 2 && NI <= 4) ? 2 : 1;
    uint8_t* ring = smem + Ly.ring + (warp - 1) * (RB / 2);
    const int nkv = nvalid / G;
    // this lane's chunks of global step gs, then one commit group (empty past the end)
    auto issue = [&](int gs) {
      const int ti = gs / (2 * EM::NS);
      if (CPS > 0 && ti < ntiles) {
        const int ph = (gs / EM::NS) & 1;
        const int st = gs % EM::NS;
        const int t0 = lo + ti * TC_T;
        const int tok = st * EM::TT + tau_l;
        if (tok < min(TC_T, hi - t0)) {
          const __nv_bfloat16* E = ph ? p.EV : p.EK;
          const unsigned trow = (unsigned)(t0 + tok) * (unsigned)p.e_row;  // < M e_row < 2^32
#pragma unroll
          for (int r = 0; r < NI; ++r)
            if (ev[r])
              cp_async16(ring + (gs % RING) * STEP + (((32 * r + lane) ^ (tok & 7)) * 16),
                         E + eoff[r] + trow);
        }
      }
      cp_async_commit();
    };
    // chunks of the SB consecutive global steps gs .. gs + SB - 1 (tile steps s .. s + SB - 1)
    // once this lane's copies landed; every later step's group may still be in flight
    auto take_batch = [&](int gs, int s, int nt, uint4 (&x)[SB][NI]) {
      cp_async_wait<RING - SB>();
#pragma unroll
      for (int u = 0; u < SB; ++u) {
        const int tok = (s + u) * EM::TT + tau_l;
#pragma unroll
        for (int r = 0; r < NI; ++r)
          x[u][r] = (ev[r] && tok < nt)
                        ? *reinterpret_cast<const uint4*>(ring + ((gs + u) % RING) * STEP +
                                                          (((32 * r + lane) ^ (tok & 7)) * 16))
                        : make_uint4(0, 0, 0, 0);
      }
    };
    if constexpr (CPS > 0) {
      // rows that are never copied (tokens past the split) are read by the MMA path: they
      // must hold finite values
      for (int o = lane * 16; o < RB / 2; o += 32 * 16)
        *reinterpret_cast<uint4*>(ring + o) = make_uint4(0, 0, 0, 0);
      __syncwarp();
      if (nkv > 0)
        for (int gs = 0; gs < RING; ++gs) issue(gs);
    }

    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      const int t0 = lo + i * TC_T;
      const int nt = min(TC_T, hi - t0);
      if constexpr (CPS > 0) {
        // (no separate L2 prefetch: the ring's own copies run far enough ahead, and an
        // extra bulk prefetch of the next tile measured slower)
        if (EM::KMMA && nkv > 0) {
          // exact-dim scores on the warp-level MMA: per 8 tokens and KV head, B = the 8
          // token rows of the KV head's slice (ldmatrix from the ring), A = its query rows
          const int gs0 = i * 2 * EM::NS;
#pragma unroll 1
          for (int tg = 0; tg < TC_T / 8; ++tg) {
            cp_async_wait<RING - EM::SPG>();  // this lane's copies of the 8 tokens landed
            __syncwarp();                     // and every other lane's
            const int tok = tg * 8 + (lane & 7);  // ldmatrix row supplied by this lane
            const int st = tok / EM::TT, tt = tok - (tok / EM::TT) * EM::TT;
            const uint8_t* slotp = ring + ((gs0 + st) % RING) * STEP;
            const int cbase = tt * EM::CH + (lane >> 3);  // chunk of matrix lane / 8 of KV 0
#pragma unroll
            for (int kv = 0; kv < (EM::KMMA ? EM::NK : 1); ++kv) {
              if (kv < nkv) {
                uint32_t bq[4];
                const uint8_t* rowp = slotp + (((cbase + kv * EM::CPS1) ^ (lane & 7)) * 16);
                if constexpr (CPS >= 4)
                  ldmatrix_x4(bq, rowp);
                else if constexpr (CPS == 2)
                  ldmatrix_x2(bq, rowp);
                else
                  ldmatrix_x1(bq, rowp);
                float dq[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                mma_bf16_16816_rows8(dq, aq[kv][0][0], aq[kv][0][1], bq[0], bq[1]);
                if constexpr (EM::KS == 2)
                  mma_bf16_16816_rows8(dq, aq[kv][EM::KS - 1][0], aq[kv][EM::KS - 1][1], bq[2], bq[3]);
                if ((lane >> 2) < G) {
                  float* xr = xs + (kv * G + (lane >> 2)) * TC_XS_LD + tg * 8 + 2 * (lane & 3);
                  xr[0] = dq[0] * p.qscale;
                  xr[1] = dq[1] * p.qscale;
                }
              }
            }
            __syncwarp();  // every lane has read the slots of these 8 tokens
#pragma unroll
            for (int u2 = 0; u2 < EM::SPG; ++u2) issue(gs0 + tg * EM::SPG + u2 + RING);
          }
        } else if (nkv > 0) {
          // exact-dim scores: per step, dot products of the lane's chunks with q_e, summed
          // over the KV head's CPS chunk lanes, into xs[query head][token]. SB steps per
          // pass: one wait, then SB independent load / multiply / shuffle chains.
#pragma unroll 1
          for (int s1 = 0; s1 < EM::NS; s1 += SB) {
            const int gs = i * 2 * EM::NS + s1;
            uint4 x[SB][NI];
            take_batch(gs, s1, nt, x);
            float part[SB][NI][G];
#pragma unroll
            for (int u = 0; u < SB; ++u)
#pragma unroll
              for (int r = 0; r < NI; ++r) {
                float2 x2[4];
                bf16x8_to_f32x2(x[u][r], x2);
#pragma unroll
                for (int hq = 0; hq < G; ++hq) {
                  float2 a = make_float2(0.0f, 0.0f);
#pragma unroll
                  for (int e = 0; e < 4; ++e) a = __ffma2_rn(qv[r][hq][e], x2[e], a);
                  part[u][r][hq] = a.x + a.y;
                }
              }
#pragma unroll
            for (int o = 1; o < CPS; o <<= 1)
#pragma unroll
              for (int u = 0; u < SB; ++u)
#pragma unroll
                for (int r = 0; r < NI; ++r)
#pragma unroll
                  for (int hq = 0; hq < G; ++hq)
                    part[u][r][hq] += __shfl_xor_sync(0xffffffffu, part[u][r][hq], o);
            if (c_first) {
#pragma unroll
              for (int u = 0; u < SB; ++u) {
                const int tok = (s1 + u) * EM::TT + tau_l;
#pragma unroll
                for (int r = 0; r < NI; ++r)
#pragma unroll
                  for (int hq = 0; hq < G; ++hq)
                    xs[(kap[r] * G + hq) * TC_XS_LD + tok] = part[u][r][hq];
              }
            }
            // into the slots just read (their values are consumed above)
#pragma unroll
            for (int u = 0; u < SB; ++u) issue(gs + u + RING);
          }
        } else {
          for (int t = lane; t < 16 * TC_XS_LD; t += 32) xs[t] = 0.0f;
        }
        __syncwarp();
      }
      float sc[TC_T];
#pragma unroll
      for (int t = 0; t < TC_T; ++t) sc[t] = (CPS > 0 && mine) ? xsq[lane * TC_XS_LD + t] : 0.0f;
      ok = mbar_wait(&s_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 5u) && ok;
      __syncwarp();  // tcgen05.ld is warp-collective
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_32x32b_x32(tmem_s + lanebase + 32 * b, sr);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < TC_T; ++t)
        sc[t] = hvalid ? __uint_as_float(sr[t]) * w_unscale + sc[t] : 0.0f;
#pragma unroll
      for (int t = 0; t < TC_T; ++t)
        if (t >= nt) sc[t] = -INFINITY;
      // max and sum over the tile as pairwise trees (short dependency chains)
      float red[TC_T / 2];
#pragma unroll
      for (int t = 0; t < TC_T / 2; ++t) red[t] = fmaxf(sc[2 * t], sc[2 * t + 1]);
#pragma unroll
      for (int w2 = TC_T / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int t = 0; t < w2; ++t) red[t] = fmaxf(red[t], red[t + w2]);
      const float tmax = red[0];
      const float m_new = (tmax > m + TC_LAZY) ? tmax : m;  // m = -inf: the first tile's max
      const float alpha = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
#pragma unroll
      for (int t = 0; t < TC_T; ++t) sc[t] = exp2f(sc[t] - m_new);  // -inf -> 0
#pragma unroll
      for (int t = 0; t < TC_T / 2; ++t) red[t] = sc[2 * t] + sc[2 * t + 1];
#pragma unroll
      for (int w2 = TC_T / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
        for (int t = 0; t < w2; ++t) red[t] += red[t + w2];
      const float psum = red[0];
      l = l * alpha + psum;
      m = m_new;
      // a head whose reference max rose rescales its U^T row (after the previous tile's
      // MMA 2; half 0 of the pair does the quadrant's 32 rows, with half 1's factors passed
      // through shared memory) and its value accumulators
      const float a_own = (mine && i > 0 && alpha < 1.0f) ? alpha : 1.0f;
      if (hf == 1 && mine) al_s[(b * 4 + pair) * 32 + lane] = a_own;
      asm volatile("bar.sync %0, 64;" ::"r"(2 + pair) : "memory");  // the pair's factors
      const float a_row = mine ? a_own : al_s[(b * 4 + pair) * 32 + lane];
      if (hf == 0 && __any_sync(0xffffffffu, a_row < 1.0f)) {
        const bool w_ok = mbar_wait(&phi_free[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u,
                                    abort_flag, WD_DECODE | 6u);
        ok = ok && w_ok;
        __syncwarp();
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < F2 / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a_row);
          tmem_st_32x32b_x32(tmem_u + lanebase + c * 32, r);
        }
        tmem_st_wait();
      }
      if (__any_sync(0xffffffffu, a_own < 1.0f)) {
#pragma unroll
        for (int r = 0; r < NI; ++r)
#pragma unroll
          for (int hq = 0; hq < G; ++hq) {
            const float ah = __shfl_sync(0xffffffffu, a_own, 16 * hf + kap[r] * G + hq);
#pragma unroll
            for (int e = 0; e < 4; ++e) accv[r][hq][e] = __fmul2_rn(accv[r][hq][e], make_float2(ah, ah));
          }
      }
      // P^T row of this head (fp16, 2^7 p) into buffer b, once MMA 2 of tile i-2 released it
      if (i >= 2) {
        const bool w_ok = mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag,
                                    WD_DECODE | 7u);
        ok = ok && w_ok;
      }
      // row h: 64 bytes, 16-byte chunk c (tokens 8c .. 8c+7) swizzled by (h >> 1) & 3
      uint8_t* prow = PS + b * p_bytes + h * 64;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if (!mine) break;  // the other half of the pair writes these rows
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
      if constexpr (CPS > 0) {
        // p of this head for the exact-dim values
#pragma unroll
        for (int t = 0; t < TC_T; ++t)
          if (mine) xsq[lane * TC_XS_LD + t] = sc[t];
        __syncwarp();
        // exact-dim values: accv[r][hq] += p(head kap G + hq, token) E_V chunk
        if (nkv > 0) {
#pragma unroll 1
          for (int s1 = 0; s1 < EM::NS; s1 += SB) {
            const int gs = i * 2 * EM::NS + EM::NS + s1;
            uint4 x[SB][NI];
            take_batch(gs, s1, nt, x);
#pragma unroll
            for (int u = 0; u < SB; ++u) {
              const int tok = (s1 + u) * EM::TT + tau_l;
#pragma unroll
              for (int r = 0; r < NI; ++r) {
                float2 x2[4];
                bf16x8_to_f32x2(x[u][r], x2);
#pragma unroll
                for (int hq = 0; hq < G; ++hq) {
                  const float pv = xs[(kap[r] * G + hq) * TC_XS_LD + tok];
                  const float2 pv2 = make_float2(pv, pv);
#pragma unroll
                  for (int e = 0; e < 4; ++e)
                    accv[r][hq][e] = __ffma2_rn(pv2, x2[e], accv[r][hq][e]);
                }
              }
            }
#pragma unroll
            for (int u = 0; u < SB; ++u) issue(gs + u + RING);
          }
        }
        __syncwarp();  // xs is rewritten by the next tile's scores
      }
    }
    cp_async_wait<0>();  // no copy of this thread is left in flight
    // split record: running max, sum, exact-dim values, U
    const bool done = ntiles == 0 || mbar_wait(u_done, 0, abort_flag, WD_DECODE | 8u);
    const bool all_ok = __all_sync(0xffffffffu, ok && done);
    __syncwarp();
    tc_fence_after();
    if (hvalid && all_ok) {
      float* rec = p.rec + ((long long)sp * bhq + gh) * p.rec_stride;
      rec[0] = m;
      rec[1] = l;
    }
    if constexpr (CPS > 0) {
#pragma unroll
      for (int o = EM::CH; o < 32; o <<= 1)  // sum over the step's token lanes
#pragma unroll
        for (int r = 0; r < NI; ++r)
#pragma unroll
          for (int hq = 0; hq < G; ++hq)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              accv[r][hq][e].x += __shfl_xor_sync(0xffffffffu, accv[r][hq][e].x, o);
              accv[r][hq][e].y += __shfl_xor_sync(0xffffffffu, accv[r][hq][e].y, o);
            }
      if (tau_l == 0 && all_ok) {
#pragma unroll
        for (int r = 0; r < NI; ++r) {
          if (!ev[r]) continue;
#pragma unroll
          for (int hq = 0; hq < G; ++hq) {
            float* rec = p.rec + ((long long)sp * bhq + gbase + kap[r] * G + hq) * p.rec_stride;
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (e < de_r[r]) rec[4 + c8r[r] + e] = (e & 1) ? accv[r][hq][e >> 1].y : accv[r][hq][e >> 1].x;
          }
        }
      }
    }
    const int nslot = 2 * p.F_pad;
#pragma unroll 1
    for (int c = 0; c < F2 / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
      tmem_ld_wait();
      if (hvalid && all_ok) {
        float* rec = p.rec + ((long long)sp * bhq + gh) * p.rec_stride;
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

template <int CPS, int G, int RB>
static cudaError_t launch_tc_rb(const DecodeParams& p, int grid, int smem, cudaStream_t stream) {
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(decode_tc_kernel<CPS, G, RB>), smem);
  if (e != cudaSuccess) return e;
  decode_tc_kernel<CPS, G, RB><<<grid, TC_THREADS, smem, stream>>>(p);
  return cudaGetLastError();
}

template <int CPS, int G>
static cudaError_t launch_tc(const DecodeParams& p, int grid, int smem, cudaStream_t stream) {
  return tc_ring_bytes(p.tc_F2) == TC_RING_BYTES_WIDE
             ? launch_tc_rb<CPS, G, TC_RING_BYTES_WIDE>(p, grid, smem, stream)
             : launch_tc_rb<CPS, G, TC_RING_BYTES>(p, grid, smem, stream);
}

template <int CPS>
static cudaError_t launch_tc_g(const DecodeParams& p, int grid, int smem, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_tc<CPS, 1>(p, grid, smem, stream);
    case 2: return launch_tc<CPS, 2>(p, grid, smem, stream);
    case 4: return launch_tc<CPS, 4>(p, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_decode_tc(const DecodeParams& p, int de_slot, cudaStream_t stream) {
  const int smem = (int)decode_tc_smem_bytes(p.tc_F2, de_slot, p.G);
  const int heads = p.B * p.Hq;
  const int grid = ((heads + TC_NH - 1) / TC_NH) * p.n_splits;
  switch (de_slot) {
    case 0: return launch_tc_g<0>(p, grid, smem, stream);
    case 8: return launch_tc_g<1>(p, grid, smem, stream);
    case 16: return launch_tc_g<2>(p, grid, smem, stream);
    case 32: return launch_tc_g<4>(p, grid, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

FA_WATCHDOG_READER(read_watchdog_decode_tc)

}  // namespace fa
