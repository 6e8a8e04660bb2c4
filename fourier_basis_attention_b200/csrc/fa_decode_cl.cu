// fa_decode_cl.cu -- split-L decode of the middle span on the tcgen05 tensor cores for
// large k, with the coefficient slots split over a thread-block cluster.
//
// Same mathematics as the other split kernels ([skill] Step 4, in the coefficient domain).
// For a tile of CL_T = 32 middle tokens and a set of 128 query heads:
//     S^T[heads x tokens] = W[heads x slots] . Phi_t^T      (MMA 1; slots = cos / sin pairs)
//     p = online softmax of (S + exact-dim scores)
//     U^T[heads x slots] += P^T[heads x tokens] . Phi_t    (MMA 2, accumulated over tiles)
// For k up to 1023 there are 2F = 1024 slots: U^T alone would need 1024 fp32 columns of
// tensor memory (an SM has 512) and W (fp16 hi + lo) 512 KB. So a cluster of C CTAs
// (C = 2 or 4; C = 1 for k <= 255) splits the slots: CTA r of the cluster keeps slots
// [r SL, (r + 1) SL) (SL <= 256): its W_hi in shared memory, W_lo and its U^T slice in
// tensor memory, and it generates only its frequencies of Phi_t. Its MMA 1 then gives a
// partial S over its slots. The 128 heads form four quadrants of 32 (the TMEM lane
// quarters); quadrant q is owned by CTA q C / 4. For each tile:
//   1. every CTA reads its partial S of each quadrant out of tensor memory, stages the
//      quadrants it does not own in its shared memory and sends each to its owner as one
//      bulk shared-to-shared copy across the cluster (counted on the owner's mbarrier);
//   2. the owner adds the C partials and the exact-dim scores, runs the online softmax
//      (fp32, lazily raised reference max) and sends the P rows (fp16, 2^7 p) and the
//      rescale factors of its heads to every CTA of the cluster by bulk copies;
//   3. each CTA rescales its U^T rows where the reference max rose and issues MMA 2 on its
//      slots. MMA 2's commit arrives on the same barrier in every CTA of the cluster, which
//      tells the owners when P buffers may be rewritten.
// The exact (retained) dims of the owned quadrants' KV heads are streamed by TMA bulk
// copies (one per KV head and token block, per-KV-head E blocks as stored) into a ring of
// shared-memory slots fed by one producer thread. Exact-dim scores run on the CUDA cores
// (each lane holds its query head's retained q values in registers and serves a group of
// tokens), values on the CUDA cores with fp32 accumulators. The head warps are software-
// pipelined: while the partial scores of tile i cross the cluster, they accumulate the
// values of tile i - 1 and, after the softmax, compute the exact-dim scores of tile i + 1.
//
// Warp roles (8 warps): 0 = TMEM owner and MMA issuer; 1 = exact-dim producer; 2-3 = basis
// generators (thread = frequency, rotation along the tile's tokens from the exactly
// reduced phase); 4-7 = head warps, warp 4 + q serving TMEM lane quarter q. Every wait is
// bounded; the CTAs of a cluster leave together through a final cluster barrier.
#include "fa_decode_common.cuh"

namespace fa {

constexpr int CL_NH = 128;       // query heads per cluster = MMA M = TMEM lanes
constexpr int CL_T = 32;         // tokens per tile
constexpr int CL_THREADS = 256;  // 8 warps
constexpr int CL_GEN = 64;       // generator threads (warps 2-3)
constexpr float CL_LAZY = 8.0f;
constexpr float CL_P_SCALE = 128.0f;
constexpr float CL_P_UNSCALE = 1.0f / 128.0f;
constexpr int CL_XS_LD = 33;     // fp32 row pitch of the [head][token] score / p buffers
constexpr int CL_XB = 32 * CL_T * 4;  // bytes of one quadrant's partial-score block (4 KB):
                                 // row = head, 16-byte chunk j of row h at (j ^ (h & 7))
constexpr int CL_MAX_EXACT = 32; // exact KV heads per CTA (owned query heads / G)
constexpr int CL_MAX_STAGES = 8;
constexpr int CL_EPAD = 64;      // bytes between two KV heads' blocks in a ring slot
constexpr int CL_MAX_IPL = 4;    // exact-dim value items (query head, 8 dims) per lane

struct ClExact {   // one exact KV head of the CTA (32 bytes)
  long long gbase; // element offset of its E block (b e_batch + e_off[g])
  int off;         // byte offset of its rows inside a ring slot
  int de_ld, de;   // row pitch and retained dims
  int row0;        // quadrant-local row of its first query head (j G)
  int li;          // index of its quadrant among the CTA's owned quadrants
  int valid;
};

struct ClLayout {
  int w, phi, ps, ring, xr, xsend, xs, al, meta, bars, total;  // byte offsets
};

__host__ __device__ inline ClLayout cl_layout(int C, int SL, int slot_bytes, int stages) {
  const int nown = 4 / C;
  ClLayout L;
  L.w = 0;                                          // [SL/64][128 heads][64 fp16] SW128
  L.phi = L.w + CL_NH * SL * 2;                     // 2 x [SL/64][32 tokens][64 fp16] SW128
  L.ps = L.phi + 2 * CL_T * SL * 2;                 // 2 x [128 heads][32 fp16] SW64
  L.ring = L.ps + 2 * CL_NH * CL_T * 2;             // stages x slot_bytes
  L.xr = L.ring + stages * slot_bytes;              // [2][nown][C-1] partial-score blocks
  L.xsend = L.xr + 2 * nown * (C - 1) * CL_XB;      // [4 - nown] outgoing blocks
  L.xs = L.xsend + (4 - nown) * CL_XB;              // [2][nown][32][CL_XS_LD] fp32
  L.al = L.xs + 2 * nown * 32 * CL_XS_LD * 4;             // [2][128] fp32 rescale factors
  L.meta = L.al + 2 * CL_NH * 4;                          // [CL_MAX_EXACT] ClExact
  L.bars = L.meta + CL_MAX_EXACT * (int)sizeof(ClExact);  // mbarriers, TMEM slot, flags
  L.total = L.bars + 64 * 8 + 64 + 1024;                  // + alignment slack
  return L;
}

__device__ __forceinline__ uint32_t cl_pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int C>
__global__ void __launch_bounds__(CL_THREADS, 1)
    decode_cl_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NOWN = 4 / C;  // quadrants owned by each CTA
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned base, formed by pointer arithmetic on smem_raw so that the compiler
  // keeps it (and everything derived from it) in the shared address space
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int SL = p.cl_SL;
  const int stages = p.cl_stages, slot_bytes = p.cl_slot_bytes, TB = p.cl_TB;
  const ClLayout Ly = cl_layout(C, SL, slot_bytes, stages);
  uint8_t* Ws = smem + Ly.w;
  uint8_t* PHI = smem + Ly.phi;
  uint8_t* PS = smem + Ly.ps;
  uint8_t* ring = smem + Ly.ring;
  uint8_t* xr = smem + Ly.xr;
  uint8_t* xsend = smem + Ly.xsend;
  float* xs = reinterpret_cast<float*>(smem + Ly.xs);
  float* al = reinterpret_cast<float*>(smem + Ly.al);
  ClExact* meta = reinterpret_cast<ClExact*>(smem + Ly.meta);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* phi_full = bars;        // [2] generators -> MMA (count 2 warps)
  uint64_t* phi_free = bars + 2;    // [2] MMA 2 of every CTA of the cluster done (count C)
  uint64_t* s_full = bars + 4;      // [2] MMA 1 done (commit)
  uint64_t* p_full = bars + 6;      // [2] head warps -> MMA (count 4)
  uint64_t* u_done = bars + 8;      // every MMA of this CTA done
  uint64_t* r_full = bars + 9;      // [stages] producer -> head warps (expect_tx)
  uint64_t* r_empty = r_full + CL_MAX_STAGES;  // [stages] head warps -> producer (count 4)
  uint64_t* xr_full = r_empty + CL_MAX_STAGES; // [2][NOWN] partial scores received
  uint64_t* pr_full = xr_full + 2 * 4;         // [2][4 - NOWN] P rows + factors received
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pr_full + 2 * 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* n_exact_s = const_cast<int*>(abort_flag) + 1;
  int* has_exact_s = n_exact_s + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = C > 1 ? cluster_ctarank() : 0u;
  const int cid = blockIdx.x / C;
  const int hs = cid / p.n_splits;
  const int sp = cid - hs * p.n_splits;
  const int lo = sp * p.split_len;
  const int hi = min(p.M, lo + p.split_len);
  const int ntiles = (hi - lo + CL_T - 1) / CL_T;
  const int P = p.P;  // basis period
  const long long bhq = (long long)p.B * p.Hq;
  const int G = p.G;
  const int slot0 = (int)rank * SL;  // first global coefficient slot of this CTA
  const int nslot = 2 * p.F_pad;
  const int nsb = CL_T / TB;         // ring slots (token blocks) per tile and phase
  const int q_first = (int)rank * NOWN;  // first owned quadrant

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&phi_full[b], CL_GEN / 32);
      mbar_init(&phi_free[b], C);
      mbar_init(&s_full[b], 1);
      mbar_init(&p_full[b], 4);
      for (int l = 0; l < NOWN; ++l) mbar_init(&xr_full[b * 4 + l], 1);
      for (int l = 0; l < 4 - NOWN; ++l) mbar_init(&pr_full[b * 4 + l], 1);
    }
    mbar_init(u_done, 1);
    for (int s = 0; s < stages; ++s) {
      mbar_init(&r_full[s], 1);
      mbar_init(&r_empty[s], 4);
    }
    *abort_flag = 0;
    // exact KV heads of the owned quadrants and their places in a ring slot
    int off = 0, n = 0, any = 0;
    const int nkq = 32 / G;
    for (int li = 0; li < NOWN; ++li)
      for (int j = 0; j < nkq; ++j) {
        ClExact e;
        const long long gh = (long long)hs * CL_NH + 32 * (q_first + li) + j * G;
        e.valid = gh < bhq;
        const int bb = e.valid ? (int)(gh / p.Hq) : 0;
        const int gg = e.valid ? (int)(gh - (long long)bb * p.Hq) / G : 0;
        e.gbase = (long long)bb * p.e_batch + p.e_off[gg];
        e.de_ld = e.valid ? p.de_ld[gg] : 0;
        e.de = e.valid ? p.de[gg] : 0;
        e.row0 = j * G;
        e.li = li;
        e.off = off;
        off += TB * e.de_ld * 2 + (e.de_ld > 0 ? CL_EPAD : 0);
        any |= e.de_ld > 0;
        meta[n++] = e;
      }
    *n_exact_s = n;
    *has_exact_s = any;
    fence_barrier_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, p.cl_tmem_cols);
    tmem_relinquish();
  }
  // (The exact-dim ring is not cleared: rows past a split's end are never copied, but their
  // tokens' scores are replaced by -inf before use and the value loops stop at the last
  // token.)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if constexpr (C > 1) cluster_sync_all();  // peers' barriers exist before any remote op
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_u = tmem;              // U^T slice: columns [0, SL)
  const uint32_t tmem_s = tmem + SL;         // S^T buffer b: columns SL + 32 b
  const uint32_t tmem_wlo = tmem + SL + 64;  // W_lo: SL / 2 columns (slot pairs)
  const int n_exact = *n_exact_s;
  const bool has_exact = *has_exact_s != 0;
  const uint16_t cta_mask = (uint16_t)((1u << C) - 1u);

  // head warps: W rows of this CTA's slots, scaled by 2^-e to at most 1, split into fp16
  // hi (shared, K-major, 128-byte swizzle) and lo (tensor memory, row = this head's lane)
  const int quad = warp & 3;                 // TMEM lane quarter of a head warp
  const int h = quad * 32 + lane;
  const long long gh = (long long)hs * CL_NH + h;
  const bool is_head = warp >= 4;
  const bool hvalid = is_head && gh < bhq;
  float w_unscale = 1.0f;
  if (is_head) {
    const float* wsrc = p.qw + gh * p.qw_stride + FA_HEAD_DIM + slot0;
    const int ns_here = hvalid ? max(0, min(SL, nslot - slot0)) : 0;
    float wmax = 0.0f;
    for (int s = 0; s < ns_here; ++s) wmax = fmaxf(wmax, fabsf(wsrc[s]));
    int ex = 0;
    if (wmax > 0.0f) frexpf(wmax, &ex);
    const float w_scale = ldexpf(1.0f, -ex);
    w_unscale = ldexpf(1.0f, ex);
    const uint32_t lanebase_w = (uint32_t)(quad * 32) << 16;
    for (int c64 = 0; c64 < SL / 64; ++c64) {
      uint32_t lo32[32];
#pragma unroll
      for (int c8 = 0; c8 < 8; ++c8) {
        uint32_t hv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int s = c64 * 64 + c8 * 8 + 2 * e;
          const float a = s < ns_here ? wsrc[s] * w_scale : 0.0f;
          const float b = s + 1 < ns_here ? wsrc[s + 1] * w_scale : 0.0f;
          hv[e] = cl_pack_half2(a, b);
          const __half2 hh = *reinterpret_cast<const __half2*>(&hv[e]);
          lo32[c8 * 4 + e] = cl_pack_half2(a - __low2float(hh), b - __high2float(hh));
        }
        const int off = c64 * (CL_NH * 128) + h * 128 + ((c8 ^ (h & 7)) << 4);
        *reinterpret_cast<uint4*>(Ws + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      tmem_st_32x32b_x32(tmem_wlo + lanebase_w + c64 * 32, lo32);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const int phi_bytes = CL_T * SL * 2;
  const int p_bytes = CL_NH * CL_T * 2;
  if (warp == 0) {
    // -------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc1 = idesc_f16_f32(CL_NH, CL_T, /*b_mn_major=*/false);
      const uint32_t idesc2 = idesc_f16_f32(CL_NH, SL, /*b_mn_major=*/true);
      const uint64_t d_w = smem_desc_sw128(smem_u32(Ws), 16, 1024);
      const uint64_t d_phik = smem_desc_sw128(smem_u32(PHI), 16, 1024);
      const uint64_t d_phin = smem_desc_sw128(smem_u32(PHI), CL_T * 128, 1024);
      const uint64_t d_p = smem_desc_sw64(smem_u32(PS), 16, 512);
      const int nks = SL / 16;
      bool ok = true;
      auto mma1 = [&](int i) {
        const int b = i & 1;
        if (!mbar_wait(&phi_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 32u)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint64_t dphi = d_phik + (uint64_t)((b * phi_bytes) >> 4);
        const uint32_t ts = tmem_s + 32 * b;
#pragma unroll 4
        for (int ks = 0; ks < nks; ++ks) {
          const uint32_t ow = (uint32_t)(((ks >> 2) * (CL_NH * 128) + (ks & 3) * 32) >> 4);
          const uint32_t op = (uint32_t)(((ks >> 2) * (CL_T * 128) + (ks & 3) * 32) >> 4);
          mma_f16(ts, d_w + ow, dphi + op, idesc1, ks > 0 ? 1u : 0u);
          mma_f16_ta(ts, tmem_wlo + 8 * ks, dphi + op, idesc1, 1u);
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
        if (!mbar_wait(&p_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 33u)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < CL_T / 16; ++ks)
          mma_f16(tmem_u, d_p + (uint64_t)((b * p_bytes + ks * 32) >> 4),
                  d_phin + (uint64_t)((b * phi_bytes + ks * 2048) >> 4), idesc2,
                  (i > 0 || ks > 0) ? 1u : 0u);
        if constexpr (C > 1)
          mma_commit_mc(&phi_free[b], cta_mask);
        else
          mma_commit(&phi_free[b]);
      }
      mma_commit(u_done);
      const unsigned long long w0 = globaltimer_ns();
      while (!mbar_try_wait(u_done, 0) && globaltimer_ns() - w0 < kWaitLimitNs) {
      }
      if constexpr (C > 1) {
        // MMA 2's commits arrive on phi_free in every CTA of the cluster. Nothing else waits
        // for the last two tiles' phases, so this CTA waits for them here: once they complete,
        // no peer's arrive is still on its way to this CTA's shared memory when it leaves.
        for (int i = ntiles >= 2 ? ntiles - 2 : 0; i < ntiles; ++i)
          mbar_wait(&phi_free[i & 1], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 43u);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------------- exact-dim producer
    if (lane == 0 && has_exact) {
      // chunks in the head warps' order: K(0); then per tile i: V(i - 1), K(i + 1); V(last)
      int cc = 0;
      bool ok = true;
      auto issue = [&](int ti, int ph) {
        const int t0 = lo + ti * CL_T;
        const __nv_bfloat16* E = ph ? p.EV : p.EK;
        for (int sb = 0; sb < nsb && ok; ++sb, ++cc) {
          const int s = cc % stages;
          if (cc >= stages &&
              !mbar_wait(&r_empty[s], (uint32_t)((cc / stages) - 1) & 1u, abort_flag,
                         WD_DECODE | 34u)) {
            ok = false;
            break;
          }
          const int tok0 = t0 + sb * TB;
          const int rows = max(0, min(TB, hi - tok0));
          uint32_t bytes = 0;
          for (int e = 0; e < n_exact; ++e)
            if (meta[e].valid) bytes += (uint32_t)(rows * meta[e].de_ld * 2);
          mbar_arrive_expect_tx(&r_full[s], bytes);
          for (int e = 0; e < n_exact; ++e) {
            const ClExact& m = meta[e];
            if (m.valid && m.de_ld > 0 && rows > 0)
              bulk_load_cta(ring + s * slot_bytes + m.off, E + m.gbase + (long long)tok0 * m.de_ld,
                            (uint32_t)(rows * m.de_ld * 2), &r_full[s]);
          }
        }
      };
      if (ntiles > 0) issue(0, 0);
      for (int i = 0; i < ntiles && ok; ++i) {
        if (i >= 1) issue(i - 1, 1);
        if (i + 1 < ntiles) issue(i + 1, 0);
      }
      if (ntiles > 0 && ok) issue(ntiles - 1, 1);
    }
  } else if (warp < 4) {
    // -------------------------------------------------------------------- basis generators
    // thread gt: local frequencies gt and gt + 64 (global f = slot0 / 2 + local); per tile
    // the unit phasor of f (t0 + tau) / P by rotation from the exactly reduced phase.
    const int gt = threadIdx.x - 64;
    const int nf = SL / 2;
    const int f0 = slot0 / 2;
    float ra[2], rb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int f = f0 + gt + CL_GEN * u;
      ra[u] = 1.0f;
      rb[u] = 0.0f;
      if (gt + CL_GEN * u < nf) phase_sincos(f % P, P, p.two_over_P, &rb[u], &ra[u]);
    }
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      if (i >= 2 && !mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag,
                                       WD_DECODE | 35u))
        break;
      const long long tm0 = (long long)lo + i * CL_T;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int fl = gt + CL_GEN * u;
        if (fl < nf) {
          const int f = f0 + fl;
          float s, c;
          phase_sincos(((long long)f * tm0) % P, P, p.two_over_P, &s, &c);
          uint8_t* base = PHI + b * phi_bytes + (fl >> 5) * (CL_T * 128) + 4 * (fl & 3);
          const int chunk = (fl & 31) >> 2;
#pragma unroll 8
          for (int tau = 0; tau < CL_T; ++tau) {
            *reinterpret_cast<uint32_t*>(base + tau * 128 + ((chunk ^ (tau & 7)) << 4)) =
                cl_pack_half2(c, s);
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
    const uint32_t lanebase = (uint32_t)(quad * 32) << 16;
    const bool own_q = (quad / NOWN) == (int)rank;  // this CTA owns quadrant `quad`
    const int li_q = quad - q_first;                 // its index among the owned ones
    const int owner = quad / NOWN;                   // owning CTA of quadrant `quad`
    const int wq = warp - 4;                         // share of the exact-dim work
    // received-P slot of a quadrant this CTA does not own
    const int npi = own_q ? 0 : (quad < q_first ? quad : quad - NOWN);
    // exact-dim value items of this warp: (exact KV head e, 8-dim chunk c, query head jq)
    // (the warp's items in (e, c, jq) order, jq fastest; lane takes items lane + 32 u)
    int it_e[CL_MAX_IPL], it_c[CL_MAX_IPL], it_jq[CL_MAX_IPL];
    int n_items = 0;
#pragma unroll
    for (int u = 0; u < CL_MAX_IPL; ++u) {
      const int target = lane + 32 * u;
      it_e[u] = -1;
      it_c[u] = 0;
      it_jq[u] = 0;
      int k = 0;
      for (int e = wq; e < n_exact; e += 4) {
        const ClExact& me = meta[e];
        if (!me.valid) continue;
        const int cnt = (me.de_ld / 8) * G;
        if (target < k + cnt) {
          it_e[u] = e;
          it_c[u] = (target - k) / G;
          it_jq[u] = (target - k) % G;
          break;
        }
        k += cnt;
      }
      n_items += it_e[u] >= 0 ? 1 : 0;
    }
    // exact-dim scores: lane = (query head sh of the warp's KV heads, token group sg); the
    // warp's 32 / C query heads (its KV heads e = wq, wq + 4, ... times G) take SGN = C
    // token groups. q_e of the lane's head in registers (unscaled, 8-dim chunks as pairs).
    const int SGN = C;
    const int HW = 32 / SGN;
    const int shi = lane % HW, sg = lane / HW;
    int sh_off = 0, sh_pitch = 0, sh_c8 = 0, sh_row = 0;
    bool sh_ok = false;  // the lane has a valid query head (its KV head may have no exact dims)
    float2 qv[8][4];
    {
      const int el = shi / G, jq = shi % G;
      const int e = wq + 4 * el;
      if (e < n_exact && meta[e].valid) {
        const ClExact& me = meta[e];
        sh_ok = true;
        sh_off = me.off;
        sh_pitch = me.de_ld * 2;
        sh_c8 = me.de_ld / 8;
        sh_row = me.li * 32 + me.row0 + jq;
        const long long ghs = (long long)hs * CL_NH + 32 * (q_first + me.li) + me.row0 + jq;
        const int bb = (int)(ghs / p.Hq), gg = (int)(ghs - (long long)bb * p.Hq) / G;
#pragma unroll
        for (int d8 = 0; d8 < 8; ++d8)
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float2 v = make_float2(0.0f, 0.0f);
            const int d = 8 * d8 + 2 * e2;
            if (d < me.de) v.x = __bfloat162float(p.q[ghs * FA_HEAD_DIM + p.perm[gg][p.dc[gg] + d]]);
            if (d + 1 < me.de) v.y = __bfloat162float(p.q[ghs * FA_HEAD_DIM + p.perm[gg][p.dc[gg] + d + 1]]);
            qv[d8][e2] = v;
          }
      } else {
#pragma unroll
        for (int d8 = 0; d8 < 8; ++d8)
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) qv[d8][e2] = make_float2(0.0f, 0.0f);
      }
    }
    float acc[CL_MAX_IPL][8];
#pragma unroll
    for (int u = 0; u < CL_MAX_IPL; ++u)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[u][e] = 0.0f;
    float m = -INFINITY, l = 0.0f;  // softmax state of head h (owned quadrant)
    bool ok = true;
    int cc = 0;  // ring slot counter (same sequence as the producer's)

    auto ring_wait = [&](int s) -> bool {
      return mbar_wait(&r_full[s], (uint32_t)(cc / stages) & 1u, abort_flag, WD_DECODE | 36u);
    };
    auto ring_release = [&](int s) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&r_empty[s]);
    };

    // A(i): exact-dim scores of tile i into xs[i & 1] (scaled by sigma log2 e); lane (query
    // head sh, token group sg) takes tokens sg, sg + SGN, ... of each ring slot
    auto scores = [&](int i) {
      float* xsb = xs + (i & 1) * NOWN * 32 * CL_XS_LD;
      {
        for (int sb = 0; sb < nsb; ++sb, ++cc) {
          const int s = cc % stages;
          ok = ring_wait(s) && ok;
          if (sh_ok) {
            const uint8_t* blk = ring + s * slot_bytes + sh_off;
            float* xrw = xsb + sh_row * CL_XS_LD + sb * TB;
            const int ntb = TB;  // tokens past the split's end are masked by the owner
            for (int t0 = sg; t0 < ntb; t0 += 4 * SGN) {
              // four tokens x two 8-dim chunks per step: the eight loads are issued before
              // any of their products (token index clamped into the block, chunk past the
              // row masked to zero after the load; both reads stay inside the slot: a row
              // is followed by the next row or by the block's padding)
              const uint8_t* rowp[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) rowp[u] = blk + min(t0 + u * SGN, ntb - 1) * sh_pitch;
              float2 acc4[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) acc4[u] = make_float2(0.0f, 0.0f);
#pragma unroll
              for (int d8 = 0; d8 < 8; d8 += 2) {
                if (d8 < sh_c8) {
                  const bool second = d8 + 1 < sh_c8;
                  uint4 xq[4][2];
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    xq[u][0] = *reinterpret_cast<const uint4*>(rowp[u] + d8 * 16);
                    xq[u][1] = *reinterpret_cast<const uint4*>(rowp[u] + d8 * 16 + 16);
                  }
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    if (!second) xq[u][1] = make_uint4(0, 0, 0, 0);
                    float2 x2[4], y2[4];
                    bf16x8_to_f32x2(xq[u][0], x2);
                    bf16x8_to_f32x2(xq[u][1], y2);
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc4[u] = __ffma2_rn(qv[d8][e], x2[e], acc4[u]);
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc4[u] = __ffma2_rn(qv[d8 + 1][e], y2[e], acc4[u]);
                  }
                }
              }
#pragma unroll
              for (int u = 0; u < 4; ++u)
                if (t0 + u * SGN < ntb) xrw[t0 + u * SGN] = (acc4[u].x + acc4[u].y) * p.qscale;
            }
          }
          ring_release(s);
        }
      }
    };
    // G(i): exact-dim values of tile i, acc = alpha acc + p E_V over this warp's items (p in
    // xs[i & 1], rescale factors in al[i & 1])
    auto values = [&](int i) {
      const int b = i & 1;
      const int nt = min(CL_T, hi - (lo + i * CL_T));
      const float* xsb = xs + b * NOWN * 32 * CL_XS_LD;
#pragma unroll
      for (int u = 0; u < CL_MAX_IPL; ++u) {
        if (u < n_items) {
          const ClExact& me = meta[it_e[u]];
          const float a = al[b * CL_NH + 32 * (q_first + me.li) + me.row0 + it_jq[u]];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[u][e] *= a;
        }
      }
      for (int sb = 0; sb < nsb; ++sb, ++cc) {
        const int s = cc % stages;
        ok = ring_wait(s) && ok;
        const uint8_t* slotp = ring + s * slot_bytes;
        const int ntb = min(TB, nt - sb * TB);
#pragma unroll
        for (int u = 0; u < CL_MAX_IPL; ++u) {
          if (u < n_items) {
            const ClExact& me = meta[it_e[u]];
            const float* prw = xsb + (me.li * 32 + me.row0 + it_jq[u]) * CL_XS_LD + sb * TB;
            const uint8_t* col = slotp + me.off + it_c[u] * 16;
            const int pitch = me.de_ld * 2;
            float2 a2[4], b2[4];  // even / odd tokens: two shorter accumulation chains
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              a2[e] = make_float2(acc[u][2 * e], acc[u][2 * e + 1]);
              b2[e] = make_float2(0.0f, 0.0f);
            }
            int t = 0;
            for (; t + 4 <= ntb; t += 4) {  // four tokens' loads issued together
              uint4 xv[4];
              float pt[4];
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                xv[v] = *reinterpret_cast<const uint4*>(col + (t + v) * pitch);
                pt[v] = prw[t + v];
              }
#pragma unroll
              for (int v = 0; v < 4; ++v) {
                float2 x2[4];
                bf16x8_to_f32x2(xv[v], x2);
                const float2 pp = make_float2(pt[v], pt[v]);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  if (v & 1)
                    b2[e] = __ffma2_rn(pp, x2[e], b2[e]);
                  else
                    a2[e] = __ffma2_rn(pp, x2[e], a2[e]);
                }
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) a2[e] = make_float2(a2[e].x + b2[e].x, a2[e].y + b2[e].y);
            for (; t < ntb; ++t) {
              float2 x2[4];
              bf16x8_to_f32x2(*reinterpret_cast<const uint4*>(col + t * pitch), x2);
              const float2 pp = make_float2(prw[t], prw[t]);
#pragma unroll
              for (int e = 0; e < 4; ++e) a2[e] = __ffma2_rn(pp, x2[e], a2[e]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[u][2 * e] = a2[e].x;
              acc[u][2 * e + 1] = a2[e].y;
            }
          }
        }
        ring_release(s);
      }
    };
    // Software-pipelined tile loop: the partial scores of tile i travel to their owners
    // while the values of tile i - 1 are accumulated, and the P rows of tile i travel back
    // while the exact-dim scores of tile i + 1 are computed.
    float sc[CL_T];
    if (ntiles > 0 && has_exact) scores(0);
    for (int i = 0; i < ntiles; ++i) {
      const int b = i & 1;
      const int nt = min(CL_T, hi - (lo + i * CL_T));
      float* xsb = xs + b * NOWN * 32 * CL_XS_LD;
      // ---- partial S of quadrant `quad` over this CTA's slots
      ok = mbar_wait(&s_full[b], (uint32_t)(i >> 1) & 1u, abort_flag, WD_DECODE | 37u) && ok;
      __syncwarp();
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld_32x32b_x32(tmem_s + lanebase + 32 * b, sr);
      tmem_ld_wait();
#pragma unroll
      for (int t = 0; t < CL_T; ++t) sc[t] = hvalid ? __uint_as_float(sr[t]) * w_unscale : 0.0f;
      if constexpr (C > 1) {
        if (!own_q) {
          // to the owner, as one bulk copy of the quadrant's block into slot [b][its quadrant
          // index][this CTA's sender slot]. The staging block is free again: its previous copy
          // landed before the owner answered the previous tile.
          uint8_t* stg = xsend + npi * CL_XB;
#pragma unroll
          for (int j = 0; j < CL_T / 4; ++j)
            *reinterpret_cast<float4*>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_float4(sc[4 * j], sc[4 * j + 1], sc[4 * j + 2], sc[4 * j + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int oli = quad - owner * NOWN;
            const int sslot = (int)rank < owner ? (int)rank : (int)rank - 1;
            const uint32_t dst = mapa_shared(
                smem_u32(xr + ((b * NOWN + oli) * (C - 1) + sslot) * CL_XB), (uint32_t)owner);
            const uint32_t rb = mapa_shared(smem_u32(&xr_full[b * 4 + oli]), (uint32_t)owner);
            bulk_copy_s2s(dst, stg, CL_XB, rb);
          }
        }
      }
      if (i > 0 && has_exact) values(i - 1);
      asm volatile("bar.sync 2, 128;" ::: "memory");  // scores of tile i in xs[b]; xs[b ^ 1] free
      float alpha = 1.0f;
      if (own_q) {
        // ---- owner: full scores, online softmax, P rows to every CTA
        if constexpr (C > 1) {
          if (lane == 0)
            mbar_arrive_expect_tx(&xr_full[b * 4 + li_q], (uint32_t)((C - 1) * CL_XB));
          ok = mbar_wait(&xr_full[b * 4 + li_q], (uint32_t)(i >> 1) & 1u, abort_flag,
                                 WD_DECODE | 38u) && ok;
          for (int s2 = 0; s2 < C - 1; ++s2) {
            const uint8_t* src = xr + ((b * NOWN + li_q) * (C - 1) + s2) * CL_XB + lane * 128;
#pragma unroll
            for (int j = 0; j < CL_T / 4; ++j) {
              const float4 v = *reinterpret_cast<const float4*>(src + ((j ^ (lane & 7)) << 4));
              sc[4 * j] += hvalid ? v.x : 0.0f;
              sc[4 * j + 1] += hvalid ? v.y : 0.0f;
              sc[4 * j + 2] += hvalid ? v.z : 0.0f;
              sc[4 * j + 3] += hvalid ? v.w : 0.0f;
            }
          }
        }
        float* xrow = xsb + (li_q * 32 + lane) * CL_XS_LD;
        if (has_exact) {
#pragma unroll
          for (int t = 0; t < CL_T; ++t) sc[t] += hvalid ? xrow[t] : 0.0f;
        }
#pragma unroll
        for (int t = 0; t < CL_T; ++t)
          if (t >= nt) sc[t] = -INFINITY;
        // max and sum over the tile as pairwise trees (short dependency chains)
        float red[CL_T / 2];
#pragma unroll
        for (int t = 0; t < CL_T / 2; ++t) red[t] = fmaxf(sc[2 * t], sc[2 * t + 1]);
#pragma unroll
        for (int w2 = CL_T / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int t = 0; t < w2; ++t) red[t] = fmaxf(red[t], red[t + w2]);
        const float tmax = red[0];
        const float m_new = (tmax > m + CL_LAZY) ? tmax : m;
        alpha = (m == -INFINITY) ? 0.0f : exp2f(m - m_new);
#pragma unroll
        for (int t = 0; t < CL_T; ++t) sc[t] = exp2f(sc[t] - m_new);
#pragma unroll
        for (int t = 0; t < CL_T / 2; ++t) red[t] = sc[2 * t] + sc[2 * t + 1];
#pragma unroll
        for (int w2 = CL_T / 4; w2 >= 1; w2 >>= 1)
#pragma unroll
          for (int t = 0; t < w2; ++t) red[t] += red[t + w2];
        const float psum = red[0];
        l = l * alpha + psum;
        m = m_new;
        // P buffers of tile i - 2 are free in every CTA once their MMA 2 completed
        if (i >= 2)
          ok = mbar_wait(&phi_free[b], (uint32_t)((i >> 1) - 1) & 1u, abort_flag,
                                 WD_DECODE | 39u) && ok;
        uint32_t pv[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          pv[e] = cl_pack_half2(sc[2 * e] * CL_P_SCALE, sc[2 * e + 1] * CL_P_SCALE);
        uint8_t* prow = PS + b * p_bytes + h * 64;
#pragma unroll
        for (int c = 0; c < 4; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ ((h >> 1) & 3)) << 4)) =
              make_uint4(pv[4 * c], pv[4 * c + 1], pv[4 * c + 2], pv[4 * c + 3]);
        al[b * CL_NH + h] = alpha;
        if constexpr (C > 1) {
          // the quadrant's 32 P rows (2 KB, already in the peers' swizzled layout) and its 32
          // rescale factors go to the same places in every peer, by two bulk copies each
          fence_proxy_async_smem();
          __syncwarp();
          if (lane < C && lane != (int)rank) {  // lane p sends to peer p
            const int peer = lane;
            const int pq = quad < peer * NOWN ? quad : quad - NOWN;  // peer's slot for it
            const uint32_t rb = mapa_shared(smem_u32(&pr_full[b * 4 + pq]), (uint32_t)peer);
            const uint8_t* prows = PS + b * p_bytes + quad * 32 * 64;
            const float* alq = al + b * CL_NH + quad * 32;
            bulk_copy_s2s(mapa_shared(smem_u32(prows), (uint32_t)peer), prows, 32 * 64, rb);
            bulk_copy_s2s(mapa_shared(smem_u32(alq), (uint32_t)peer), alq, 32 * 4, rb);
          }
        }
        // p (fp32) of this head for the exact-dim values
#pragma unroll
        for (int t = 0; t < CL_T; ++t) xrow[t] = sc[t];
      }
      if (i + 1 < ntiles && has_exact) scores(i + 1);
      if (!own_q) {
        // ---- the owner's P rows of this quadrant land in PS, its factors in al
        if (lane == 0) mbar_arrive_expect_tx(&pr_full[b * 4 + npi], (uint32_t)(32 * 64 + 32 * 4));
        ok = mbar_wait(&pr_full[b * 4 + npi], (uint32_t)(i >> 1) & 1u, abort_flag,
                               WD_DECODE | 40u) && ok;
        alpha = al[b * CL_NH + h];
      }
      // a head whose reference max rose rescales its U^T row (after the previous tile's
      // MMA 2 of this CTA)
      const bool need = i > 0 && alpha < 1.0f;
      if (__any_sync(0xffffffffu, need)) {
        ok = mbar_wait(&phi_free[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1u, abort_flag,
                               WD_DECODE | 41u) && ok;
        __syncwarp();
        tc_fence_after();
        const float a = need ? alpha : 1.0f;
#pragma unroll 1
        for (int c = 0; c < SL / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * a);
          tmem_st_32x32b_x32(tmem_u + lanebase + c * 32, r);
        }
        tmem_st_wait();
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[b]);
      asm volatile("bar.sync 2, 128;" ::: "memory");  // p and alpha of tile i visible
    }
    if (ntiles > 0 && has_exact) values(ntiles - 1);
    // ---- split record: running max, sum (owned heads), exact-dim values, U slice
    const bool done = ntiles == 0 || mbar_wait(u_done, 0, abort_flag, WD_DECODE | 42u);
    const bool all_ok = __all_sync(0xffffffffu, ok && done);
    __syncwarp();
    tc_fence_after();
    if (own_q && hvalid && all_ok) {
      float* rec = p.rec + ((long long)sp * bhq + gh) * p.rec_stride;
      rec[0] = m;
      rec[1] = l;
    }
    if (all_ok) {
#pragma unroll
      for (int u = 0; u < CL_MAX_IPL; ++u) {
        if (u < n_items) {
          const ClExact& me = meta[it_e[u]];
          const long long ghi = (long long)hs * CL_NH + 32 * (q_first + me.li) + me.row0 + it_jq[u];
          float* rec = p.rec + ((long long)sp * bhq + ghi) * p.rec_stride + 4 + 8 * it_c[u];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            if (8 * it_c[u] + e < me.de) rec[e] = acc[u][e];
        }
      }
    }
#pragma unroll 1
    for (int c = 0; c < SL / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32b_x32(tmem_u + lanebase + c * 32, r);
      tmem_ld_wait();
      if (hvalid && all_ok) {
        float* rec = p.rec + ((long long)sp * bhq + gh) * p.rec_stride + 4 + FA_HEAD_DIM;
#pragma unroll
        for (int j = 0; j < 32; j += 4) {
          const int slot = slot0 + c * 32 + j;
          if (slot < nslot)
            *reinterpret_cast<float4*>(rec + slot) =
                make_float4(__uint_as_float(r[j]) * CL_P_UNSCALE,
                            __uint_as_float(r[j + 1]) * CL_P_UNSCALE,
                            __uint_as_float(r[j + 2]) * CL_P_UNSCALE,
                            __uint_as_float(r[j + 3]) * CL_P_UNSCALE);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (C > 1) cluster_sync_all();  // no CTA leaves while peers may still write to it
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, p.cl_tmem_cols);
  }
}

// ------------------------------------------------------------------------- host side
size_t decode_cl_smem_bytes(int C, int SL, int slot_bytes, int stages) {
  return (size_t)cl_layout(C, SL, slot_bytes, stages).total;
}

template <int C>
static const void* cl_kernel_ptr() {
  return reinterpret_cast<const void*>(decode_cl_kernel<C>);
}

const void* decode_cl_kernel_ptr(int C) {
  switch (C) {
    case 1: return cl_kernel_ptr<1>();
    case 2: return cl_kernel_ptr<2>();
    case 4: return cl_kernel_ptr<4>();
    default: return nullptr;
  }
}

template <int C>
static cudaError_t launch_cl_t(const DecodeParams& p, int n_clusters, int smem, cudaStream_t stream) {
  cudaError_t e = raise_smem_limit(reinterpret_cast<const void*>(decode_cl_kernel<C>), smem);
  if (e != cudaSuccess) return e;
  if constexpr (C == 1) {
    decode_cl_kernel<1><<<n_clusters, CL_THREADS, smem, stream>>>(p);
    return cudaGetLastError();
  } else {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(n_clusters * C), 1, 1);
    cfg.blockDim = dim3(CL_THREADS, 1, 1);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, decode_cl_kernel<C>, p);
  }
}

cudaError_t launch_decode_cl(const DecodeParams& p, cudaStream_t stream) {
  const int smem = (int)decode_cl_smem_bytes(p.cl_C, p.cl_SL, p.cl_slot_bytes, p.cl_stages);
  const int n_hs = (p.B * p.Hq + CL_NH - 1) / CL_NH;
  const int n_clusters = n_hs * p.n_splits;
  switch (p.cl_C) {
    case 1: return launch_cl_t<1>(p, n_clusters, smem, stream);
    case 2: return launch_cl_t<2>(p, n_clusters, smem, stream);
    case 4: return launch_cl_t<4>(p, n_clusters, smem, stream);
    default: return cudaErrorInvalidValue;
  }
}

// Clusters of decode_cl_kernel<C> that can be resident at once (cached per device).
cudaError_t decode_cl_max_clusters(int C, int smem, int* n) {
  const void* fn = decode_cl_kernel_ptr(C);
  if (!fn) return cudaErrorInvalidValue;
  cudaError_t e = raise_smem_limit(fn, smem);
  if (e != cudaSuccess) return e;
  if (C == 1) {
    int occ = 0, sms = 0;
    if ((e = cached_occupancy(fn, CL_THREADS, (size_t)smem, &occ)) != cudaSuccess) return e;
    if ((e = device_sm_count(&sms)) != cudaSuccess) return e;
    *n = occ * sms;
    return cudaSuccess;
  }
  return cached_max_clusters(fn, CL_THREADS, (size_t)smem, C, n);
}

FA_WATCHDOG_READER(read_watchdog_decode_cl)

}  // namespace fa
