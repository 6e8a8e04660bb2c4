// fa_host.h -- host-side interfaces between the C ABI (fa_abi.cu) and the kernel units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "../../include/fourier_attention.h"

namespace fa {

// Launch configuration of one fa_decode call (derived by decode_configure).
struct DecodeConfig {
  int n_splits, split_len, n_fsplits, n_rec, F, F_pad, SPT, NTU, TG, DEC, TGE, NKV;
  int tc, tc_F2, tc_tmem_cols, de_ld_max;  // tensor-core split kernel chosen, its slots / TMEM
  int hm, hm_F2;  // warp-MMA split kernel chosen (blocked E, large k), its slots
  // cluster tensor-core split kernel chosen (blocked E), its cluster size, slots per CTA,
  // ring token block, ring stages and slot bytes, TMEM columns, shared-memory bytes
  int cl, cl_C, cl_SL, cl_TB, cl_stages, cl_slot_bytes, cl_tmem_cols, cl_smem;
  int cb_gt;      // query heads per combine CTA (a divisor of G)
  size_t qw_bytes, rec_bytes, smem_main, smem_combine;
  int rec_stride, qw_stride;
};

cudaError_t launch_build_basis(int M, int k, long long ld, int dtype, int normalized, void* out,
                               cudaStream_t stream, int num_sms);
cudaError_t launch_compress(const fa_plan* plan, const void* K, const void* V,
                            const void* phiT, const fa_cache* cache, cudaStream_t stream,
                            const char** why);
cudaError_t decode_configure(const fa_plan* plan, int requested, DecodeConfig* c,
                             const char** why = nullptr);
// Decode checks + configuration as the entry points run them: FA_OK, or a status with
// fa_last_error() set (argument checks, unsupported shapes, configuration limits).
int decode_setup(const fa_plan* plan, int requested, DecodeConfig* c);
cudaError_t launch_decode(const fa_plan* plan, const DecodeConfig& c, const void* q,
                          const fa_cache* cache, void* out, int out_dtype, void* workspace,
                          cudaStream_t stream);
cudaError_t launch_append(const fa_plan* plan, const void* k_new, const void* v_new,
                          const fa_cache* cache, cudaStream_t stream);
int sensitivity_plan(const fa_shape* shape, fa_plan* plan);  // fa_status code
size_t sensitivity_out_offset(const DecodeConfig& c);
cudaError_t launch_sensitivity(const fa_plan* plan, const DecodeConfig& c, const void* q,
                               const void* K, const void* noise, float* scores, void* workspace,
                               cudaStream_t stream);
cudaError_t read_and_clear_watchdog(unsigned int* word);
cudaError_t read_watchdog_decode_tc(unsigned int* word);  // per-unit readers
cudaError_t read_watchdog_decode_cl(unsigned int* word);
cudaError_t launch_watchdog_selftest(unsigned int wait_ns, cudaStream_t stream);

// Per-device launch facts, queried once and cached (fa_runtime.cu).
cudaError_t device_sm_count(int* sms);
// Raises `func`'s dynamic shared-memory limit to at least `bytes` on the current device.
cudaError_t raise_smem_limit(const void* func, int bytes);
// Resident blocks per SM of `func` at `threads` threads and `smem` dynamic shared bytes.
cudaError_t cached_occupancy(const void* func, int threads, size_t smem, int* blocks);
// Clusters of `cluster` CTAs of `func` that can be resident at once on the current device.
cudaError_t cached_max_clusters(const void* func, int threads, size_t smem, int cluster, int* n);
// Cluster tensor-core decode kernel (fa_decode_cl.cu): shared-memory bytes of a layout,
// and resident clusters of it.
size_t decode_cl_smem_bytes(int C, int SL, int slot_bytes, int stages);
cudaError_t decode_cl_max_clusters(int C, int smem, int* n);

// Records `msg` as the calling thread's fa_last_error() text and returns `code`.
int set_last_error(int code, const char* msg);

}  // namespace fa
