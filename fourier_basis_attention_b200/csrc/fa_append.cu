// fa_append.cu -- decode-time cache maintenance: one new token per sequence.
//
// The recent window of [skill] Step 3 is the last R tokens of the current sequence, so
// each new token pushes the oldest recent token into the middle span, whose compressed
// dims are held as fixed-length spectral coefficients ([abstract] method details). With
// the basis period P fixed, extending the projection C = Phi^T X by the middle token t is
// the rank-1 update C_j += phi_j(t) x_c (j < k); its retained dims become E row t.
//
// CTAs over (batch row, KV head, K or V) x row chunks of C: each reads the token x that
// joins the middle (the oldest ring row of F, or the new token itself when R = 0) and
// folds it into its rows of the k x dc_ld block of C; chunk 0 also writes E row t. The C
// update is a read-modify-write: HBM-bound at 8 bytes per coefficient. The new token
// takes the freed ring row after every chunk has read x: inside the kernel when there is
// one chunk per head, else in a second launch (few heads: the chunks spread the
// read-modify-write over all SMs).
#include <math.h>
#include <string.h>

#include "fa_decode_common.cuh"

namespace fa {

constexpr int AP_THREADS = 256;
constexpr int AP_BATCH = 8;  // float4 pieces of C in flight per thread

struct AppendParams {
  int Hkv, S, R, t, P, k, rhead;
  int n_chunks, chunk_rows;  // row chunks of C per (head, K / V)
  float norm_single, norm_pair, two_over_P;
  long long c_batch, e_batch;
  long long c_off[FA_MAX_KV_HEADS], e_off[FA_MAX_KV_HEADS];
  int dc[FA_MAX_KV_HEADS], dc_ld[FA_MAX_KV_HEADS], de_ld[FA_MAX_KV_HEADS];
  int e_pitch[FA_MAX_KV_HEADS];
  unsigned char perm[FA_MAX_KV_HEADS][FA_HEAD_DIM];
  const __nv_bfloat16* x_new[2];
  __nv_bfloat16* F[2];
  __nv_bfloat16* E[2];
  float* C[2];
};

__global__ void __launch_bounds__(AP_THREADS) append_kernel(const __grid_constant__ AppendParams p) {
  __shared__ float xc[FA_HEAD_DIM];               // compressed dims of x, in C column order
  __shared__ __nv_bfloat16 xb[FA_HEAD_DIM];       // x, all dims
  __shared__ float ub[FA_MAX_K_DECODE + 1];       // phi_j(t) of this chunk's rows j0 <= j < j1
  const int tid = threadIdx.x;
  const int head = blockIdx.x, which = blockIdx.y, z = blockIdx.z;
  const int j0 = z * p.chunk_rows, j1 = min(p.k, j0 + p.chunk_rows);
  const int b = head / p.Hkv, g = head - (head / p.Hkv) * p.Hkv;
  const int dc = p.dc[g], dc_ld = p.dc_ld[g], de_ld = p.de_ld[g];
  const __nv_bfloat16* xnew = p.x_new[which] + (long long)head * FA_HEAD_DIM;
  __nv_bfloat16* ring_row =
      p.F[which] + ((long long)head * (p.S + p.R) + p.S + p.rhead) * FA_HEAD_DIM;
  const __nv_bfloat16* src = p.R > 0 ? ring_row : xnew;
  const int nq = dc_ld >> 2;
  float4* C4 = reinterpret_cast<float4*>(p.C[which] + (long long)b * p.c_batch + p.c_off[g] +
                                         (long long)j0 * dc_ld);
  const int n4 = (j1 - j0) * nq;  // k <= FA_MAX_K_DECODE, nq <= 32
  constexpr int STEP = AP_THREADS * AP_BATCH;
  // the first pieces of C are in flight while x and the basis values are fetched
  float4 v[AP_BATCH];
#pragma unroll
  for (int u = 0; u < AP_BATCH; ++u)
    if (tid + u * AP_THREADS < n4) v[u] = C4[tid + u * AP_THREADS];

  if (tid < FA_HEAD_DIM) xb[tid] = src[tid];
  // basis values of token t: phase f t reduced modulo P in integers, then sincospi
  for (int j = j0 + tid; j < j1; j += AP_THREADS) {
    const int f = (j + 1) >> 1;
    float s = 0.0f, c = 1.0f;
    if (f > 0) phase_sincos(((long long)f * p.t) % p.P, p.P, p.two_over_P, &s, &c);
    const float nrm = (f == 0 || 2 * f == p.P) ? p.norm_single : p.norm_pair;
    ub[j - j0] = nrm * ((j > 0 && (j & 1) == 0) ? s : c);
  }
  __syncthreads();
  if (tid < FA_HEAD_DIM) xc[tid] = tid < dc ? __bfloat162float(xb[p.perm[g][tid]]) : 0.0f;
  // the new token takes the ring row that x has left (x is in shared memory now)
  if (p.n_chunks == 1 && p.R > 0 && tid < FA_HEAD_DIM / 8)
    reinterpret_cast<uint4*>(ring_row)[tid] = reinterpret_cast<const uint4*>(xnew)[tid];
  // E row t: retained dims in ascending order, padding columns zero
  if (z == 0 && tid < de_ld) {
    __nv_bfloat16* e = p.E[which] + (long long)b * p.e_batch + p.e_off[g] +
                       (long long)p.t * p.e_pitch[g];
    e[tid] = tid < FA_HEAD_DIM - dc ? xb[p.perm[g][dc + tid]] : __float2bfloat16_rn(0.0f);
  }
  __syncthreads();
  // C_j += phi_j(t) x_c over the chunk's rows of the k x dc_ld block, float4 columns; the
  // next AP_BATCH pieces are loaded before the current ones are updated and stored
  for (int i0 = tid; i0 < n4; i0 += STEP) {
    float4 nv[AP_BATCH];
#pragma unroll
    for (int u = 0; u < AP_BATCH; ++u) {
      const int i = i0 + STEP + u * AP_THREADS;
      if (i < n4) nv[u] = C4[i];
    }
#pragma unroll
    for (int u = 0; u < AP_BATCH; ++u) {
      const int i = i0 + u * AP_THREADS;
      if (i < n4) {
        const int j = i / nq, q = i - j * nq;
        const float w = ub[j];
        v[u].x = fmaf(w, xc[4 * q], v[u].x);
        v[u].y = fmaf(w, xc[4 * q + 1], v[u].y);
        v[u].z = fmaf(w, xc[4 * q + 2], v[u].z);
        v[u].w = fmaf(w, xc[4 * q + 3], v[u].w);
        C4[i] = v[u];
      }
    }
#pragma unroll
    for (int u = 0; u < AP_BATCH; ++u) v[u] = nv[u];
  }
}

// New tokens into the freed ring rows (used when the fold ran in several chunks per head).
__global__ void __launch_bounds__(256) append_ring_kernel(const __grid_constant__ AppendParams p,
                                                          int n_rows) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;  // 16-byte piece of a row
  if (id >= n_rows * 16) return;
  const int row = id >> 4, c = id & 15, which = row & 1, head = row >> 1;
  const uint4* src = reinterpret_cast<const uint4*>(p.x_new[which] + (long long)head * FA_HEAD_DIM);
  uint4* dst = reinterpret_cast<uint4*>(
      p.F[which] + ((long long)head * (p.S + p.R) + p.S + p.rhead) * FA_HEAD_DIM);
  dst[c] = src[c];
}

cudaError_t launch_append(const fa_plan* plan, const void* k_new, const void* v_new,
                          const fa_cache* cache, cudaStream_t stream) {
  const fa_shape& sh = plan->shape;
  AppendParams ap;
  memset(&ap, 0, sizeof(ap));
  ap.Hkv = sh.Hkv;
  ap.S = plan->S;
  ap.R = plan->R;
  ap.t = plan->M;
  ap.P = plan->P;
  ap.k = plan->kk;
  ap.rhead = plan->recent_head;
  ap.norm_single = (float)(1.0 / sqrt((double)plan->P));
  ap.norm_pair = (float)sqrt(2.0 / (double)plan->P);
  ap.two_over_P = (float)(2.0 / (double)plan->P);
  ap.c_batch = plan->c_batch;
  ap.e_batch = plan->e_batch;
  for (int g = 0; g < sh.Hkv; ++g) {
    ap.c_off[g] = plan->c_off[g];
    ap.e_off[g] = plan->e_off[g];
    ap.dc[g] = plan->dc[g];
    ap.dc_ld[g] = plan->dc_ld[g];
    ap.de_ld[g] = plan->de_ld[g];
    ap.e_pitch[g] = plan->e_pitch[g];
    memcpy(ap.perm[g], plan->perm[g], FA_HEAD_DIM);
  }
  ap.x_new[0] = static_cast<const __nv_bfloat16*>(k_new);
  ap.x_new[1] = static_cast<const __nv_bfloat16*>(v_new);
  ap.F[0] = static_cast<__nv_bfloat16*>(cache->F_K);
  ap.F[1] = static_cast<__nv_bfloat16*>(cache->F_V);
  ap.E[0] = static_cast<__nv_bfloat16*>(cache->E_K);
  ap.E[1] = static_cast<__nv_bfloat16*>(cache->E_V);
  ap.C[0] = static_cast<float*>(cache->C_K);
  ap.C[1] = static_cast<float*>(cache->C_V);
  // enough CTAs for two per SM, in chunks of at least 64 rows of C
  int sms = 148;
  cudaError_t e = device_sm_count(&sms);
  if (e != cudaSuccess) return e;
  const long long units = 2LL * sh.B * sh.Hkv;
  int nz = (int)((2LL * sms + units - 1) / units);
  const int max_nz = (ap.k + 63) / 64;
  nz = nz < 1 ? 1 : (nz > max_nz ? max_nz : nz);
  ap.chunk_rows = (ap.k + nz - 1) / nz;
  ap.n_chunks = (ap.k + ap.chunk_rows - 1) / ap.chunk_rows;
  const dim3 grid((unsigned)(sh.B * sh.Hkv), 2, (unsigned)ap.n_chunks);
  append_kernel<<<grid, AP_THREADS, 0, stream>>>(ap);
  e = cudaGetLastError();
  if (e != cudaSuccess || ap.n_chunks == 1 || ap.R == 0) return e;
  const int n_rows = (int)units;
  append_ring_kernel<<<(n_rows * 16 + 255) / 256, 256, 0, stream>>>(ap, n_rows);
  return cudaGetLastError();
}

}  // namespace fa
