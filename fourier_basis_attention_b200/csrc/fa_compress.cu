// fa_compress.cu -- prefill compression of one layer on the tcgen05 tensor cores.
//
// [skill] Step 3 splits each KV head's tokens into sink / middle / recent; Step 2 projects
// the middle span onto the leading Fourier functions; [abstract] restricts the
// projection to the long-context-insensitive (masked) head dims. Per (batch b, KV head g,
// X in {K, V}):
//     C_X = Phi^T . X[S : S+M, compressed dims]          (k x dc, fp32)
//     E_X = X[S : S+M, retained dims]                     (bit-exact copy)
//     F_X = X[sink and recent tokens, all dims]           (bit-exact copy)
//
// GEMM mapping: one CTA per (batch b, KV head g, pair of 128-coefficient tiles) computes
// the coefficients of K and V together:
//   D_kt[128 coefs x 256] += A_kt[128 coefs x 64 tokens] . B[64 tokens x (128 K dims | 128 V dims)]
//   A = unit-amplitude basis table tile, K-major (tokens contiguous), TMA, 128-byte swizzle.
//   B = the cache rows of K and V, MN-major (dims contiguous: the cache's own layout), four
//       64-dim TMA boxes per stage. One N = 256 MMA covers K and V, so a cache row is read
//       from memory once for k <= 256 and the table tile feeds both.
//   D lives in tensor memory: 2 tiles x 256 fp32 columns = all 512 columns of the SM.
// All 128 dims are multiplied; the epilogue keeps the masked ones (a column gather on the
// B side is not expressible as a TMA box).
// Warp roles: warp 0 issues TMA, warp 1 issues tcgen05.mma (one thread), warps 2-9 pack
// the retained dims of every stage (first tile pair only) and run the epilogue.
// Tokens past the middle span read a zero A (TMA out-of-bounds fill), so the ragged last
// stage needs no masking. A holds unit-amplitude cos / sin (DC = 1); each accumulator row
// is scaled by its orthonormal factor (1/sqrt(M) or sqrt(2/M)) in fp32 in the epilogue.
#include <cuda.h>

#include "fa_host.h"
#include "fa_internal.cuh"

namespace fa {

constexpr int CK_BM = 128;                   // coefficient rows per tile (MMA M)
constexpr int CK_BK = 64;                    // tokens per stage
constexpr int CK_BN = 2 * FA_HEAD_DIM;       // K dims | V dims (MMA N)
constexpr int CK_A_TILE = CK_BM * CK_BK * 2; // 16 KB per coefficient tile
constexpr int CK_B_BOX = 64 * CK_BK * 2;     // 8 KB per 64-dim box
constexpr int CK_B_BYTES = 4 * CK_B_BOX;     // 32 KB
constexpr int CK_THREADS = 352;  // warp 0 TMA (cache rows), warp 1 MMA, warps 2-9 pack +
                                  // epilogue, warp 10 TMA (table tiles)
constexpr int CK_A_WARP = 10;
constexpr int CK_PACK_WARPS = 8;
constexpr int CK_STAGE_LD = CK_BN + 4;       // fp32 staging row stride (bank-conflict free)

// Two rings of stages: the table tiles (A, read from L2) and the cache rows (B, the DRAM
// stream, one stage deeper so that more of it is in flight), each with its own producer.
template <int KT>
struct CkCfg {
  static constexpr int A_BYTES = KT * CK_A_TILE;
  static constexpr int A_STAGES = KT == 2 ? 3 : 4;
  static constexpr int B_STAGES = KT == 2 ? 4 : 5;
  static constexpr int RING_BYTES = A_STAGES * A_BYTES + B_STAGES * CK_B_BYTES;
  static constexpr int TMEM_COLS = KT * CK_BN;
  static constexpr int BASE_SMEM = RING_BYTES + 1024 /*align*/ + 1024 /*misc*/;
  static_assert(CK_BM * CK_STAGE_LD * 4 <= RING_BYTES, "staging fits");
  static_assert(BASE_SMEM <= 227 * 1024, "fits in one SM's shared memory");
};


struct CompressParams {
  int M, P, k, S, L, Hkv, n_ktiles, n_pairs;
  int nsplit;  // CTAs (one cluster) that split each unit's token stages; 1 = no split
  const void* K;
  const void* V;
  float norm_single, norm_pair;
  long long c_batch, e_batch;
  long long c_off[FA_MAX_KV_HEADS], e_off[FA_MAX_KV_HEADS];
  int dc[FA_MAX_KV_HEADS], dc_ld[FA_MAX_KV_HEADS];
  int de_ld[FA_MAX_KV_HEADS], e_pitch[FA_MAX_KV_HEADS];
  unsigned char perm[FA_MAX_KV_HEADS][FA_HEAD_DIM];
  float* C[2];
  __nv_bfloat16* E[2];
};

// Bounded wait used on abort paths only (no abort-flag check): lets in-flight async
// copies land before the CTA's shared memory is released.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const unsigned long long t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > 200000000ull) break;
  }
}

template <int KT>
__global__ void __launch_bounds__(CK_THREADS, 1)
    compress_kernel(const __grid_constant__ CUtensorMap tm_phi,
                    const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v,
                    const __grid_constant__ CompressParams p) {
  using Cfg = CkCfg<KT>;
  constexpr int SA = Cfg::A_STAGES, SB = Cfg::B_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;                      // both rings (the epilogue's staging reuses them)
  uint8_t* aring = smem;                       // [SA][A_BYTES] table tiles
  uint8_t* bring = smem + SA * Cfg::A_BYTES;   // [SB][CK_B_BYTES] cache rows
  uint8_t* misc = smem + Cfg::RING_BYTES;
  uint64_t* fullA = reinterpret_cast<uint64_t*>(misc);
  uint64_t* emptyA = fullA + SA;
  uint64_t* fullB = emptyA + SA;
  uint64_t* emptyB = fullB + SB;
  uint64_t* accum = emptyB + SB;
  uint64_t* drain = accum + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* acc_flag = abort_flag + 1;  // the split epilogue's "accumulators valid"
  unsigned char* perm_s = reinterpret_cast<unsigned char*>(misc + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // unit = (head, coefficient-tile pair); with nsplit > 1 the nsplit CTAs of a cluster share
  // one unit and take contiguous thirds / quarters / ... of its token stages (rank = the
  // CTA's rank in its one-dimensional cluster)
  const int unit = blockIdx.x / p.nsplit;
  const int rank = blockIdx.x - unit * p.nsplit;
  const int pair = unit % p.n_pairs;
  const int head = unit / p.n_pairs;  // flattened b * Hkv + g
  const int b = head / p.Hkv;
  const int g = head - b * p.Hkv;
  const int dc = p.dc[g];
  const int kt0 = pair * KT;                       // first coefficient tile of this CTA
  const int kt_n = min(KT, p.n_ktiles - kt0);       // tiles present (>= 1)
  const bool do_pack = (pair == 0);
  const int nk_all = (p.M + CK_BK - 1) / CK_BK;
  const int st0 = (int)((long long)rank * nk_all / p.nsplit);  // first stage of this CTA
  const int nk = (int)((long long)(rank + 1) * nk_all / p.nsplit) - st0;  // >= 1 (host rule)
  // A head with no compressed dims needs only the packing pass of the first pair.
  if (dc == 0 && pair != 0) return;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(&fullA[s], 1);
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1 + (do_pack ? CK_PACK_WARPS : 0));
    }
    mbar_init(accum, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    prefetch_tmap(&tm_phi);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
  }
  if (threadIdx.x < FA_HEAD_DIM) perm_s[threadIdx.x] = p.perm[g][threadIdx.x];
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_d = *tmem_slot;

  if (warp == 0 || warp == CK_A_WARP) {
    // ---------------------------------------------------------------- TMA producers
    // warp 0: the cache rows (ring B); warp CK_A_WARP: the table tiles (ring A). No L2
    // prefetch of the rows ahead of their loads: with 128 or more CTAs in flight, prefetched
    // lines left L2 before their loads came (B = 4: 2.95 GB read for 2.15 GB of rows and
    // table, and slower), while the TMA loads alone read each row once.
    if (lane == 0) {
      const bool is_b = warp == 0;
      const int NS = is_b ? SB : SA;
      uint64_t* fl = is_b ? fullB : fullA;
      uint64_t* em = is_b ? emptyB : emptyA;
      const uint32_t tx = is_b ? (uint32_t)CK_B_BYTES : (uint32_t)(kt_n * CK_A_TILE);
      int issued = 0;
      for (int it = 0; it < nk; ++it) {
        const int s = it % NS;
        const uint32_t use = (uint32_t)(it / NS);
        if (it >= NS && !mbar_wait(&em[s], (use & 1u) ^ 1u, abort_flag, WD_COMPRESS | 1u))
          break;
        mbar_arrive_expect_tx(&fl[s], tx);
        if (is_b) {
          uint8_t* b_s = bring + s * CK_B_BYTES;
          const int t = p.S + (st0 + it) * CK_BK;
          tma_load_3d(b_s, &tm_k, &fl[s], 0, t, head);
          tma_load_3d(b_s + CK_B_BOX, &tm_k, &fl[s], 64, t, head);
          tma_load_3d(b_s + 2 * CK_B_BOX, &tm_v, &fl[s], 0, t, head);
          tma_load_3d(b_s + 3 * CK_B_BOX, &tm_v, &fl[s], 64, t, head);
        } else {
          uint8_t* a_s = aring + s * Cfg::A_BYTES;
          for (int kt = 0; kt < kt_n; ++kt)
            tma_load_2d(a_s + kt * CK_A_TILE, &tm_phi, &fl[s], (st0 + it) * CK_BK,
                        (kt0 + kt) * CK_BM);
        }
        ++issued;
      }
      if (*abort_flag) {
        // let the copies already issued land before shared memory goes away
        for (int it = (issued > NS ? issued - NS : 0); it < issued; ++it)
          drain_wait(&fl[it % NS], (uint32_t)(it / NS) & 1u);
      } else {
        // tail: every stage's last release (MMA commit, and pack arrivals on ring B) landed
        for (int it = (nk > NS ? nk - NS : 0); it < nk; ++it)
          mbar_wait(&em[it % NS], (uint32_t)(it / NS) & 1u, abort_flag, WD_COMPRESS | 5u);
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(CK_BM, CK_BN, /*b_mn_major=*/true);
      bool ok = true;
      for (int it = 0; it < nk; ++it) {
        const int sa = it % SA, sb = it % SB;
        if (!mbar_wait(&fullA[sa], (uint32_t)(it / SA) & 1u, abort_flag, WD_COMPRESS | 2u) ||
            !mbar_wait(&fullB[sb], (uint32_t)(it / SB) & 1u, abort_flag, WD_COMPRESS | 7u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(aring + sa * Cfg::A_BYTES);
        const uint32_t b_addr = smem_u32(bring + sb * CK_B_BYTES);
#pragma unroll
        for (int kk = 0; kk < CK_BK / 16; ++kk) {
          // B: 16 tokens = two 8-row groups of 128-byte rows; the four 64-dim boxes are
          // CK_B_BOX apart (leading byte offset).
          const uint64_t bd = smem_desc_sw128(b_addr + kk * 2048, CK_B_BOX, 1024);
#pragma unroll
          for (int kt = 0; kt < KT; ++kt) {
            if (kt < kt_n) {
              // A: 16 tokens = 32 bytes further along the swizzled 128-byte row.
              const uint64_t ad = smem_desc_sw128(a_addr + kt * CK_A_TILE + kk * 32, 16, 1024);
              mma_f16(tmem_d + kt * CK_BN, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
            }
          }
        }
        mma_commit(&emptyA[sa]);
        mma_commit(&emptyB[sb]);
      }
      if (ok) {
        mma_commit(accum);
        // tensor memory is released only after every MMA of this CTA has completed
        mbar_wait(accum, 0, abort_flag, WD_COMPRESS | 6u);
      } else {
        mma_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    // ---------------------------------------------------------------- pack + epilogue
    const int et = threadIdx.x - 64;  // 0..255
    const int pw = warp - 2;          // 0..7
    if (do_pack) {
      // Lane i of every pack warp owns retained dims i, i + 32, ... of the head; warp pw
      // owns tokens pw, pw + 8, ... of each stage. Source offsets inside the swizzled B
      // boxes are fixed per dim; only the row and its swizzle phase change per token.
      // Shared memory is close to saturated by the MMA operand reads and the TMA fills,
      // so each warp issues all of a stage's loads back to back (one exposed latency per
      // stage), then writes the rows as coalesced 64-byte global stores.
      const int de = FA_HEAD_DIM - dc;
      const int de_ld = p.de_ld[g];
      const int e_pitch = p.e_pitch[g];    // elements between consecutive rows
      const int ngrp = (de_ld + 31) >> 5;  // 32-dim groups per row
      __nv_bfloat16* const E0 = p.E[0] + (long long)b * p.e_batch + p.e_off[g];
      __nv_bfloat16* const E1 = p.E[1] + (long long)b * p.e_batch + p.e_off[g];
      constexpr int TPW = CK_BK / CK_PACK_WARPS;  // tokens per warp per stage
      for (int it = 0; it < nk; ++it) {
        const int s = it % SB;
        if (!mbar_wait(&fullB[s], (uint32_t)(it / SB) & 1u, abort_flag, WD_COMPRESS | 3u))
          break;
        const uint8_t* b_s = bring + s * CK_B_BYTES;
        const int ntok = min(CK_BK, p.M - (st0 + it) * CK_BK);
        for (int c = 0; c < ngrp; ++c) {
          const int i = lane + 32 * c;
          int boff = -1, cbit = 0;
          if (i < de) {
            const int d = perm_s[dc + i];
            boff = (d >> 6) * CK_B_BOX + ((d & 7) << 1);
            cbit = (d & 63) >> 3;
          }
          unsigned short v[2][TPW];
#pragma unroll
          for (int x = 0; x < 2; ++x)
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
              const int tau = pw + j * CK_PACK_WARPS;
              v[x][j] = 0;
              if (boff >= 0 && tau < ntok)
                v[x][j] = *reinterpret_cast<const unsigned short*>(
                    b_s + x * 2 * CK_B_BOX + tau * 128 + boff + ((cbit ^ (tau & 7)) << 4));
            }
          if (c == ngrp - 1) {
            // every shared-memory value of the stage is loaded (the release orders this
            // warp's loads before the arrival): the stage may be refilled while the rows
            // are stored
            __syncwarp();
            if (lane == 0) mbar_arrive(&emptyB[s]);
          }
          if (i < de_ld) {
#pragma unroll
            for (int x = 0; x < 2; ++x)
#pragma unroll
              for (int j = 0; j < TPW; ++j) {
                const int tau = pw + j * CK_PACK_WARPS;
                if (tau < ntok)
                  reinterpret_cast<unsigned short*>((x ? E1 : E0) +
                                                    (long long)((st0 + it) * CK_BK + tau) * e_pitch)[i] =
                      v[x][j];
              }
          }
        }
        if (ngrp == 0) {  // nothing retained: only the release
          __syncwarp();
          if (lane == 0) mbar_arrive(&emptyB[s]);
        }
      }
    }
    // all pack warps are done reading the stages before any staging write reuses them
    asm volatile("bar.sync 1, 256;" ::: "memory");
    const int acc_ready =
        (dc > 0 && !*abort_flag) ? (mbar_wait(accum, 0, abort_flag, WD_COMPRESS | 4u) ? 1 : 0) : 0;
    const int acc_all = bar1_and_256(acc_ready);
    if (p.nsplit > 1) {
      if (et == 0) *acc_flag = acc_all;  // read by every thread after the __syncthreads below
    } else if (dc > 0 && acc_all) {
      tc_fence_after();
      float* stage_f = reinterpret_cast<float*>(stages);
      const int rb = warp & 3;       // TMEM lanes this warp may access: 32*rb .. 32*rb+31
      const int half = pw >> 2;      // warps 2-5: K columns, warps 6-9: V columns
      const int row = rb * 32 + lane;
      const int dc_ld = p.dc_ld[g];
      const int nchunk = dc_ld >> 2;
      const int per_x = CK_BM * nchunk;
      float* const C0 = p.C[0] + (long long)b * p.c_batch + p.c_off[g];
      float* const C1 = p.C[1] + (long long)b * p.c_batch + p.c_off[g];
      for (int kt = 0; kt < kt_n; ++kt) {
        if (kt > 0) asm volatile("bar.sync 1, 256;" ::: "memory");  // staging reads done
#pragma unroll 1
        for (int cb = 0; cb < FA_HEAD_DIM / 32; ++cb) {
          uint32_t r[32];
          const int col = half * FA_HEAD_DIM + cb * 32;
          tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(rb * 32) << 16) + kt * CK_BN + col, r);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(stage_f + row * CK_STAGE_LD + col);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                 __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
        asm volatile("bar.sync 1, 256;" ::: "memory");
        const int jt = (kt0 + kt) * CK_BM;
        const int rows = min(CK_BM, p.k - jt);
        for (int c = et; c < 2 * per_x; c += 256) {
          const int x = c >= per_x ? 1 : 0;
          const int rem = c - x * per_x;
          const int r = rem / nchunk;
          const int q = rem - r * nchunk;
          if (r >= rows) continue;
          const int j = jt + r;
          const int f = (j + 1) >> 1;
          const float nrm = (f == 0 || 2 * f == p.P) ? p.norm_single : p.norm_pair;
          float v[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = q * 4 + e;
            v[e] = (i < dc) ? nrm * stage_f[r * CK_STAGE_LD + x * FA_HEAD_DIM + perm_s[i]] : 0.0f;
          }
          *reinterpret_cast<float4*>((x ? C1 : C0) + (long long)j * dc_ld + q * 4) =
              make_float4(v[0], v[1], v[2], v[3]);
        }
      }
    }
  }

  if (p.nsplit > 1 && dc > 0) {
    // Token-split reduction. Per coefficient tile: every CTA stages its partial sums
    // (TMEM -> fp32 staging rows, as above); after a cluster barrier, rank r sums rows
    // [r 128 / nsplit, (r + 1) 128 / nsplit) of the tile over the cluster's CTAs in rank
    // order 0, 1, ..., nsplit - 1 (distributed shared memory reads), scales and writes them;
    // a second barrier keeps every staging buffer alive until its readers are done. All
    // threads of every CTA take both barriers of every tile, aborted or not.
    __syncthreads();
    const int acc_ok = *acc_flag;
    float* stage_f = reinterpret_cast<float*>(stages);
    const int rows_per = CK_BM / p.nsplit;
    const int r0 = rank * rows_per;
    const int dc_ld = p.dc_ld[g];
    const int nchunk = dc_ld >> 2;
    const int per_x = rows_per * nchunk;
    float* const C0 = p.C[0] + (long long)b * p.c_batch + p.c_off[g];
    float* const C1 = p.C[1] + (long long)b * p.c_batch + p.c_off[g];
    uint32_t peer[16];
#pragma unroll
    for (int r = 0; r < 16; ++r)
      peer[r] = r < p.nsplit ? mapa_shared(smem_u32(stage_f), (uint32_t)r) : 0u;
    for (int kt = 0; kt < kt_n; ++kt) {
      if (warp >= 2 && warp < 2 + CK_PACK_WARPS && acc_ok) {  // the pack / epilogue warps
        tc_fence_after();
        const int rb = warp & 3;
        const int half = (warp - 2) >> 2;
        const int row = rb * 32 + lane;
#pragma unroll 1
        for (int cb = 0; cb < FA_HEAD_DIM / 32; ++cb) {
          uint32_t r[32];
          const int col = half * FA_HEAD_DIM + cb * 32;
          tmem_ld_32x32b_x32(tmem_d + ((uint32_t)(rb * 32) << 16) + kt * CK_BN + col, r);
          tmem_ld_wait();
          float4* dst = reinterpret_cast<float4*>(stage_f + row * CK_STAGE_LD + col);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            dst[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                 __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
      }
      cluster_sync_all();  // every CTA's partial of tile kt is staged
      const int jt = (kt0 + kt) * CK_BM;
      const int rows = min(CK_BM, p.k - jt);
      for (int c = threadIdx.x; c < 2 * per_x; c += CK_THREADS) {
        const int x = c >= per_x ? 1 : 0;
        const int rem = c - x * per_x;
        const int r = r0 + rem / nchunk;
        const int q = rem - (rem / nchunk) * nchunk;
        if (r >= rows) continue;
        const int j = jt + r;
        const int f = (j + 1) >> 1;
        const float nrm = (f == 0 || 2 * f == p.P) ? p.norm_single : p.norm_pair;
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int i = q * 4 + e;
          float acc = 0.0f;
          if (i < dc) {
            const uint32_t off = (uint32_t)(r * CK_STAGE_LD + x * FA_HEAD_DIM + perm_s[i]) * 4u;
            float part[16];
#pragma unroll
            for (int s2 = 0; s2 < 16; ++s2)
              if (s2 < p.nsplit) part[s2] = ld_shared_cluster_f32(peer[s2] + off);
            acc = part[0];
#pragma unroll
            for (int s2 = 1; s2 < 16; ++s2)
              if (s2 < p.nsplit) acc += part[s2];
          }
          v[e] = (i < dc) ? nrm * acc : 0.0f;
        }
        *reinterpret_cast<float4*>((x ? C1 : C0) + (long long)j * dc_ld + q * 4) =
            make_float4(v[0], v[1], v[2], v[3]);
      }
      cluster_sync_all();  // the peers' reads of this CTA's staging rows are done
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_d, Cfg::TMEM_COLS);
  }
}

// Sink and recent rows, all dims: F[head][i] = X[head][i] for i < S; the recent rows form
// a ring starting at row S + rhead: F[head][S + (rhead + a) % R] = X[head][L - R + a].
__global__ void __launch_bounds__(256) copy_sink_recent_kernel(
    const uint4* __restrict__ K, const uint4* __restrict__ V, uint4* __restrict__ FK,
    uint4* __restrict__ FV, int L, int S, int R, int rhead, long long n_heads) {
  const int nrow = S + R;
  const long long total = n_heads * nrow * 16;  // 16 x 16 bytes per 128-dim row
  for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total;
       id += (long long)gridDim.x * blockDim.x) {
    const long long row = id >> 4;
    const int c = (int)(id & 15);
    const long long head = row / nrow;
    const int i = (int)(row - head * nrow);
    const int a = i - S - rhead < 0 ? i - S - rhead + R : i - S - rhead;  // age in the ring
    const long long t = (i < S) ? i : (long long)(L - R) + a;
    const long long src = ((head * L + t) << 4) + c;
    FK[id] = K[src];
    FV[id] = V[src];
  }
}

// One thread waits on an mbarrier that expects an arrival nobody makes; the bounded wait
// expires after `limit_ns`, records WD_SELFTEST and the kernel returns.
__global__ void watchdog_selftest_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
    mbar_wait(&bar, 0, &abort_flag, WD_SELFTEST | 1u, limit_ns);
  }
}

// ------------------------------------------------------------------------- host side
cudaError_t launch_watchdog_selftest(unsigned int wait_ns, cudaStream_t stream) {
  watchdog_selftest_kernel<<<1, 32, 0, stream>>>((unsigned long long)wait_ns);
  return cudaGetLastError();
}

FA_WATCHDOG_READER(read_watchdog_compress)

// The first nonzero word of the units whose kernels wait on mbarriers (compress, the
// tensor-core decode, the cluster decode); every word is cleared.
cudaError_t read_and_clear_watchdog(unsigned int* word) {
  cudaError_t (*readers[])(unsigned int*) = {read_watchdog_compress, read_watchdog_decode_tc,
                                             read_watchdog_decode_cl};
  *word = 0;
  for (auto rd : readers) {
    unsigned int w = 0;
    cudaError_t e = rd(&w);
    if (e != cudaSuccess) return e;
    if (*word == 0) *word = w;
  }
  return cudaSuccess;
}

typedef CUresult (*PFN_encodeTiled)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion,
                                    CUtensorMapFloatOOBfill);

static PFN_encodeTiled get_encode_fn() {
  static PFN_encodeTiled fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_encodeTiled>(ptr);
  }
  return fn;
}

// Token split of the compress units (one unit = one (batch, KV head) and coefficient-tile
// pair, one CTA). When the units leave most SMs idle (small batches), each unit's token
// stages are split over a cluster of nsplit CTAs whose partial coefficients are summed in
// rank order through distributed shared memory. nsplit is the largest of 16, 8, 4, 2 for
// which units x nsplit CTAs fit on the SMs at once, all units' clusters can be resident
// together, and every CTA keeps at least 4 stages (256 tokens); else 1. The choice depends
// only on the plan and the device, so repeated calls give identical bits.
static cudaError_t compress_split(const void* fn, int smem, long long units, int stages,
                                  int* nsplit) {
  *nsplit = 1;
  int sms = 0;
  cudaError_t e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  if (units * 2 > sms) return cudaSuccess;
  for (int c = 16; c >= 2; c >>= 1) {
    if (units * c > sms || stages < 4 * c) continue;
    if (c > 8) {
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e != cudaSuccess) {
        (void)cudaGetLastError();
        continue;
      }
    }
    int ncl = 0;
    if (cached_max_clusters(fn, CK_THREADS, (size_t)smem, c, &ncl) != cudaSuccess) {
      (void)cudaGetLastError();  // this cluster size is not available here
      continue;
    }
    if (ncl >= units) {
      *nsplit = c;
      return cudaSuccess;
    }
  }
  return cudaSuccess;
}

// Returns a CUDA error, or cudaErrorInvalidValue with *why set for a host-side reason.
cudaError_t launch_compress(const fa_plan* plan, const void* K, const void* V,
                            const void* phiT, const fa_cache* cache, cudaStream_t stream,
                            const char** why) {
  const fa_shape& sh = plan->shape;
  const long long n_heads = (long long)sh.B * sh.Hkv;
  const int nrow = plan->S + plan->R;
  if (nrow > 0) {
    const long long total = n_heads * nrow * 16;
    long long blocks = (total + 255) / 256;
    if (blocks > 148 * 16) blocks = 148 * 16;
    copy_sink_recent_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        static_cast<const uint4*>(K), static_cast<const uint4*>(V),
        static_cast<uint4*>(cache->F_K), static_cast<uint4*>(cache->F_V), sh.L, plan->S,
        plan->R, plan->recent_head, n_heads);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (plan->M == 0) return cudaSuccess;

  PFN_encodeTiled encode = get_encode_fn();
  if (!encode) {
    *why = "cuTensorMapEncodeTiled is unavailable from the driver";
    return cudaErrorInvalidValue;
  }
  CUtensorMap tm_phi, tm_k, tm_v;
  {
    cuuint64_t dims[2] = {(cuuint64_t)plan->M, (cuuint64_t)sh.k};
    cuuint64_t strides[1] = {(cuuint64_t)plan->phi_ld * 2};
    cuuint32_t box[2] = {CK_BK, CK_BM};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&tm_phi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(phiT), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the basis table";
      return cudaErrorInvalidValue;
    }
  }
  for (int w = 0; w < 2; ++w) {
    cuuint64_t dims[3] = {FA_HEAD_DIM, (cuuint64_t)sh.L, (cuuint64_t)n_heads};
    cuuint64_t strides[2] = {FA_HEAD_DIM * 2, (cuuint64_t)sh.L * FA_HEAD_DIM * 2};
    cuuint32_t box[3] = {64, CK_BK, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(w ? &tm_v : &tm_k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
               const_cast<void*>(w ? V : K), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
      *why = "cuTensorMapEncodeTiled rejected the K/V cache";
      return cudaErrorInvalidValue;
    }
  }

  CompressParams cp;
  memset(&cp, 0, sizeof(cp));
  cp.M = plan->M;
  cp.P = plan->P;
  cp.k = sh.k;
  cp.S = plan->S;
  cp.L = sh.L;
  cp.K = K;
  cp.V = V;
  cp.Hkv = sh.Hkv;
  cp.n_ktiles = (sh.k + CK_BM - 1) / CK_BM;
  cp.c_batch = plan->c_batch;
  cp.e_batch = plan->e_batch;
  for (int g = 0; g < sh.Hkv; ++g) {
    cp.c_off[g] = plan->c_off[g];
    cp.e_off[g] = plan->e_off[g];
    cp.dc[g] = plan->dc[g];
    cp.dc_ld[g] = plan->dc_ld[g];
    cp.de_ld[g] = plan->de_ld[g];
    cp.e_pitch[g] = plan->e_pitch[g];
    memcpy(cp.perm[g], plan->perm[g], FA_HEAD_DIM);
  }
  cp.C[0] = static_cast<float*>(cache->C_K);
  cp.C[1] = static_cast<float*>(cache->C_V);
  cp.norm_single = (float)(1.0 / sqrt((double)plan->P));
  cp.norm_pair = (float)sqrt(2.0 / (double)plan->P);
  cp.E[0] = static_cast<__nv_bfloat16*>(cache->E_K);
  cp.E[1] = static_cast<__nv_bfloat16*>(cache->E_V);

  // One tile per CTA when k <= 128, else pairs of tiles (512 TMEM columns).
  const int KT = cp.n_ktiles >= 2 ? 2 : 1;
  cp.n_pairs = (cp.n_ktiles + KT - 1) / KT;
  const long long units = (long long)cp.n_pairs * n_heads;
  const int smem = KT == 2 ? CkCfg<2>::BASE_SMEM : CkCfg<1>::BASE_SMEM;
  const void* fn = KT == 2 ? reinterpret_cast<const void*>(compress_kernel<2>)
                           : reinterpret_cast<const void*>(compress_kernel<1>);
  cudaError_t e = raise_smem_limit(fn, smem);
  if (e != cudaSuccess) return e;
  int nsplit = 1;
  if ((e = compress_split(fn, smem, units, (plan->M + CK_BK - 1) / CK_BK, &nsplit)) != cudaSuccess)
    return e;
  cp.nsplit = nsplit;
  const long long grid = units * nsplit;
  if (nsplit == 1) {
    if (KT == 2)
      compress_kernel<2><<<(unsigned)grid, CK_THREADS, smem, stream>>>(tm_phi, tm_k, tm_v, cp);
    else
      compress_kernel<1><<<(unsigned)grid, CK_THREADS, smem, stream>>>(tm_phi, tm_k, tm_v, cp);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid, 1, 1);
  cfg.blockDim = dim3(CK_THREADS, 1, 1);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (KT == 2) return cudaLaunchKernelEx(&cfg, compress_kernel<2>, tm_phi, tm_k, tm_v, cp);
  return cudaLaunchKernelEx(&cfg, compress_kernel<1>, tm_phi, tm_k, tm_v, cp);
}

}  // namespace fa
