// fa_basis.cu -- the orthonormal real Fourier basis over the middle span, as a table.
//
// Basis ([abstract] "orthogonal Fourier bases"; [skill] Step 2, leading real-FFT terms):
//   phi_0(t) = 1/sqrt(M);  phi_{2f-1}(t) = s_f cos(2 pi f t / M);  phi_{2f}(t) = s_f sin(2 pi f t / M)
// with s_f = sqrt(2/M), except s_f = 1/sqrt(M) for the Nyquist cosine f = M/2 (M even).
// The table is stored transposed, phiT[j][t], so that it is the K-major A operand of the
// tensor-core projection in fa_compress (which reads the unscaled variant: s_f = 1).
#include "fa_host.h"
#include "fa_internal.cuh"

namespace fa {

// One thread writes a run of `run` chunks of 8 consecutive columns of frequency f: of its
// cosine row (j = 2f - 1, or j = 0 for f = 0) and of its sine row (j = 2f, when j < k), both
// from one sincospif per column (16-byte stores for bf16). The phase r = (f * t) mod M
// advances by f per column, in exact integer arithmetic (one 64-bit reduction per run), and
// is mapped to x = 2r/M in (-1, 1] before sincospif, so the angle carries no large-argument
// rounding.

template <typename T>
__device__ __forceinline__ void store_chunk(T* dst, const float (&v)[8]) {
  if constexpr (sizeof(T) == 2) {
    __nv_bfloat162 pr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[e] = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<uint4*>(pr);
  } else {
    reinterpret_cast<float4*>(dst)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(dst)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) build_basis_kernel(int M, int k, long long ld,
                                                          float norm_single, float norm_pair,
                                                          int run, T* __restrict__ out) {
  // norm_single = norm_pair = 1 gives the unscaled (unit-amplitude) table.
  const long long nchunk = ld / 8;
  const long long nrun = (nchunk + run - 1) / run;
  const int nf = (k >> 1) + 1;  // frequencies of rows 0 .. k - 1
  const long long total = (long long)nf * nrun;
  for (long long id = (long long)blockIdx.x * blockDim.x + threadIdx.x; id < total;
       id += (long long)gridDim.x * blockDim.x) {
    const int f = (int)(id / nrun);
    const long long c0 = (id - (long long)f * nrun) * run;  // first chunk of the run
    const int jc = f == 0 ? 0 : 2 * f - 1;                  // cosine row (< k)
    const bool has_sin = f > 0 && 2 * f < k;                // sine row 2f
    const float nrm = (f == 0 || 2 * f == M) ? norm_single : norm_pair;
    const int fm = f % M;
    int r = (int)(((long long)fm * (c0 * 8)) % M);
    for (int cr = 0; cr < run && c0 + cr < nchunk; ++cr) {
      const long long t0 = (c0 + cr) * 8;
      float vc[8], vs[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        if (t0 + e < M) {
          const int rr = (2 * r > M) ? r - M : r;  // phase in (-M/2, M/2]
          float sn, cs;
          sincospif((float)(2 * rr) / (float)M, &sn, &cs);
          vc[e] = nrm * cs;
          vs[e] = nrm * sn;
        } else {
          vc[e] = 0.0f;
          vs[e] = 0.0f;
        }
        r += fm;
        if (r >= M) r -= M;
      }
      store_chunk(out + (long long)jc * ld + t0, vc);
      if (has_sin) store_chunk(out + (long long)(2 * f) * ld + t0, vs);
    }
  }
}

cudaError_t launch_build_basis(int M, int k, long long ld, int dtype, int normalized, void* out,
                               cudaStream_t stream, int num_sms) {
  const float norm_single = normalized ? (float)(1.0 / sqrt((double)M)) : 1.0f;
  const float norm_pair = normalized ? (float)sqrt(2.0 / (double)M) : 1.0f;
  // runs of 4 chunks when the table is large enough to fill the GPU with them (the 64-bit
  // phase reduction amortised: 13-15% faster on tables of 1M chunks and more), else 1;
  // a thread serves both rows of a frequency
  const long long nf = (k >> 1) + 1;
  const long long chunks = nf * (ld / 8);
  const int run = chunks >= 2LL * num_sms * 512 ? 4 : 1;
  const long long total = nf * ((ld / 8 + run - 1) / run);
  long long blocks = (total + 255) / 256;
  const long long cap = (long long)num_sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (dtype == FA_BF16)
    build_basis_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, stream>>>(
        M, k, ld, norm_single, norm_pair, run, static_cast<__nv_bfloat16*>(out));
  else
    build_basis_kernel<float><<<(unsigned)blocks, 256, 0, stream>>>(
        M, k, ld, norm_single, norm_pair, run, static_cast<float*>(out));
  return cudaGetLastError();
}

}  // namespace fa
