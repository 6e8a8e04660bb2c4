// fa_abi.cu -- the extern "C" entry points: argument validation, plan derivation,
// launches, error reporting. See include/fourier_attention.h for the contract.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <string>

#include "fa_host.h"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(FA_ERR_CUDA, "%s: %s (%s)", where, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int round8(int x) { return (x + 7) & ~7; }

int check_ptr(const void* p, const char* name, bool required) {
  if (!p) return required ? fail(FA_ERR_INVALID, "%s is NULL", name) : FA_OK;
  if (!aligned16(p)) return fail(FA_ERR_INVALID, "%s is not 16-byte aligned", name);
  return FA_OK;
}

// Fills the layout fields of a plan (everything below the dim split) from shape, S, R, M,
// P, kk, G, dc and de (E holds P rows per KV head). E is token-major exactly when the tensor-core decode is used: it can
// run when k <= 255, G is 1, 2 or 4 and every KV head keeps at most 32 dims, and it is
// chosen when the k-length work per token and KV head (k G) is at least 255 and there are
// at least 128 query heads (one full tensor-core head set), or, for smaller k G (k = 63 with
// G = 4), when there are at least 1024 query heads (8 head sets). Below that the CUDA-core
// decode measured faster (LLaMA-3 layer, L = 8K, k = 63: 103 against 115 us at B = 8; the
// tensor-core decode wins from B = 32: 265 against 344 us, and 452 against 650 us at B = 64).
void derive_layout(fa_plan* plan) {
  const fa_shape& s = plan->shape;
  int max_de = 0;
  for (int g = 0; g < s.Hkv; ++g) max_de = plan->de[g] > max_de ? plan->de[g] : max_de;
  const int G = plan->G;
  const bool tm = plan->M > 0 && s.k <= 255 && (G == 1 || G == 2 || G == 4) && max_de <= 32 &&
                  ((s.k * G >= 255 && (long long)s.B * s.Hq >= 128) ||
                   (long long)s.B * s.Hq >= 1024);
  const int w = max_de == 0 ? 0 : (max_de <= 8 ? 8 : (max_de <= 16 ? 16 : 32));
  plan->e_token_major = tm ? 1 : 0;
  long long ce = 0, ee = 0;
  for (int g = 0; g < s.Hkv; ++g) {
    plan->dc_ld[g] = round8(plan->dc[g]);
    plan->c_off[g] = ce;
    ce += (long long)plan->kk * plan->dc_ld[g];
    if (tm) {
      plan->de_ld[g] = w;
      plan->e_off[g] = (long long)g * w;
      plan->e_pitch[g] = s.Hkv * w;
    } else {
      plan->de_ld[g] = round8(plan->de[g]);
      plan->e_off[g] = ee;
      plan->e_pitch[g] = plan->de_ld[g];
      ee += (long long)plan->P * plan->de_ld[g];
    }
  }
  if (tm) ee = (long long)plan->P * s.Hkv * w;
  plan->c_batch = ce;
  plan->e_batch = ee;
  plan->f_elems = (long long)s.B * s.Hkv * (plan->S + plan->R) * FA_HEAD_DIM;
  plan->e_elems = (long long)s.B * ee;
  plan->c_elems = (long long)s.B * ce;
}

// Re-checks the fields kernels rely on, so a plan edited by hand cannot drive a launch
// out of bounds.
int check_plan(const fa_plan* plan) {
  if (!plan) return fail(FA_ERR_INVALID, "plan is NULL");
  const fa_shape& s = plan->shape;
  if (s.D != FA_HEAD_DIM) return fail(FA_ERR_UNSUPPORTED, "head dim %d != 128", s.D);
  if (s.Hkv < 1 || s.Hkv > FA_MAX_KV_HEADS || s.Hq < 1 || s.Hq % s.Hkv != 0 || s.B < 1 ||
      s.L < 1)
    return fail(FA_ERR_INVALID, "plan shape is inconsistent");
  if (plan->S < 0 || plan->R < 0 || plan->M < 0 || plan->S + plan->M + plan->R != s.L)
    return fail(FA_ERR_INVALID, "plan token partition is inconsistent");
  if (plan->G != s.Hq / s.Hkv) return fail(FA_ERR_INVALID, "plan G is inconsistent");
  if (plan->kk != (plan->M > 0 ? s.k : 0)) return fail(FA_ERR_INVALID, "plan kk is inconsistent");
  if (plan->P < plan->M || (plan->M == 0 && plan->P != 0))
    return fail(FA_ERR_INVALID, "plan period P=%d is inconsistent with M=%d", plan->P, plan->M);
  if (plan->phi_ld != round8(plan->P > 8 ? plan->P : 8))
    return fail(FA_ERR_INVALID, "plan phi_ld is inconsistent");
  if (plan->recent_head < 0 || plan->recent_head >= (plan->R > 0 ? plan->R : 1))
    return fail(FA_ERR_INVALID, "plan recent_head is inconsistent");
  for (int g = 0; g < s.Hkv; ++g) {
    if (plan->dc[g] < 0 || plan->dc[g] > FA_HEAD_DIM || plan->de[g] != FA_HEAD_DIM - plan->dc[g])
      return fail(FA_ERR_INVALID, "plan dims of KV head %d are inconsistent", g);
    bool seen[FA_HEAD_DIM] = {false};
    for (int i = 0; i < FA_HEAD_DIM; ++i) {
      const int d = plan->perm[g][i];
      if (d >= FA_HEAD_DIM || seen[d])
        return fail(FA_ERR_INVALID, "plan perm of KV head %d is not a permutation", g);
      seen[d] = true;
    }
  }
  fa_plan ref = *plan;
  derive_layout(&ref);
  bool same = ref.e_token_major == plan->e_token_major && ref.c_batch == plan->c_batch &&
              ref.e_batch == plan->e_batch && ref.f_elems == plan->f_elems &&
              ref.e_elems == plan->e_elems && ref.c_elems == plan->c_elems;
  for (int g = 0; g < s.Hkv && same; ++g)
    same = ref.dc_ld[g] == plan->dc_ld[g] && ref.de_ld[g] == plan->de_ld[g] &&
           ref.e_pitch[g] == plan->e_pitch[g] && ref.c_off[g] == plan->c_off[g] &&
           ref.e_off[g] == plan->e_off[g];
  if (!same) return fail(FA_ERR_INVALID, "plan layout fields are inconsistent");
  return FA_OK;
}

}  // namespace

int fa::set_last_error(int code, const char* msg) { return fail(code, "%s", msg); }

extern "C" {

const char* fa_last_error(void) { return g_last_error.c_str(); }

int fa_plan_init(const fa_shape* shape, const uint8_t* dim_mask, fa_plan* plan) {
  if (!shape || !dim_mask || !plan) return fail(FA_ERR_INVALID, "NULL argument");
  const fa_shape s = *shape;
  if (s.D != FA_HEAD_DIM) return fail(FA_ERR_UNSUPPORTED, "head dim %d != 128", s.D);
  if (s.B < 1 || s.Hq < 1 || s.Hkv < 1 || s.L < 1 || s.S < 0 || s.R < 0 || s.k < 1)
    return fail(FA_ERR_INVALID, "shape fields out of range (B=%d Hq=%d Hkv=%d L=%d S=%d R=%d k=%d)",
                s.B, s.Hq, s.Hkv, s.L, s.S, s.R, s.k);
  if (s.Hkv > FA_MAX_KV_HEADS)
    return fail(FA_ERR_UNSUPPORTED, "Hkv=%d exceeds %d", s.Hkv, FA_MAX_KV_HEADS);
  if (s.Hq % s.Hkv != 0) return fail(FA_ERR_INVALID, "Hq=%d is not a multiple of Hkv=%d", s.Hq, s.Hkv);
  memset(plan, 0, sizeof(*plan));
  plan->shape = s;
  plan->S = s.S < s.L ? s.S : s.L;
  plan->R = s.R < s.L - plan->S ? s.R : s.L - plan->S;
  plan->M = s.L - plan->S - plan->R;
  plan->kk = plan->M > 0 ? s.k : 0;
  plan->G = s.Hq / s.Hkv;
  plan->P = plan->M;
  plan->recent_head = 0;
  plan->phi_ld = round8(plan->P > 8 ? plan->P : 8);
  bool any_dc = false;
  for (int g = 0; g < s.Hkv; ++g) {
    int n = 0;
    for (int d = 0; d < FA_HEAD_DIM; ++d)
      if (dim_mask[g * FA_HEAD_DIM + d]) plan->perm[g][n++] = (uint8_t)d;
    plan->dc[g] = n;
    for (int d = 0; d < FA_HEAD_DIM; ++d)
      if (!dim_mask[g * FA_HEAD_DIM + d]) plan->perm[g][n++] = (uint8_t)d;
    plan->de[g] = FA_HEAD_DIM - plan->dc[g];
    any_dc = any_dc || plan->dc[g] > 0;
  }
  if (plan->M > 0 && any_dc && s.k > plan->M)
    return fail(FA_ERR_UNSUPPORTED, "k=%d exceeds the middle span M=%d", s.k, plan->M);
  derive_layout(plan);
  return FA_OK;
}

int fa_plan_reserve(fa_plan* plan, int32_t L_max) {
  if (int r = check_plan(plan)) return r;
  if (plan->M < 1) return fail(FA_ERR_UNSUPPORTED, "fa_plan_reserve needs a middle span (M >= 1)");
  if (plan->P != plan->M || plan->recent_head != 0)
    return fail(FA_ERR_UNSUPPORTED, "plan already has room reserved or tokens appended");
  const long long P = (long long)L_max - plan->S - plan->R;
  if (L_max < plan->shape.L || P >= (1 << 21))
    return fail(FA_ERR_INVALID, "L_max=%d must satisfy L=%d <= L_max and L_max - S - R < 2^21",
                L_max, plan->shape.L);
  plan->P = (int32_t)P;
  plan->phi_ld = round8(plan->P > 8 ? plan->P : 8);
  derive_layout(plan);
  return FA_OK;
}

int fa_build_basis(int32_t M, int32_t k, int32_t dtype, int32_t normalized, void* phiT,
                   int64_t ld, void* stream) {
  if (M < 1 || k < 1 || k > M) return fail(FA_ERR_INVALID, "need 1 <= k <= M (k=%d, M=%d)", k, M);
  if (dtype != FA_BF16 && dtype != FA_F32) return fail(FA_ERR_INVALID, "unknown dtype %d", dtype);
  if (ld < M || ld % 8 != 0) return fail(FA_ERR_INVALID, "ld=%lld must be >= M and a multiple of 8", (long long)ld);
  if (int r = check_ptr(phiT, "phiT", true)) return r;
  int sms = 148;
  cudaError_t e = fa::device_sm_count(&sms);
  if (e != cudaSuccess) return cuda_fail(e, "fa_build_basis: device query");
  e = fa::launch_build_basis(M, k, ld, dtype, normalized ? 1 : 0, phiT,
                             static_cast<cudaStream_t>(stream), sms);
  if (e != cudaSuccess) return cuda_fail(e, "fa_build_basis: launch");
  return FA_OK;
}

int fa_compress(const fa_plan* plan, const void* K, const void* V, const void* phiT,
                const fa_cache* cache, void* stream) {
  if (int r = check_plan(plan)) return r;
  if (!cache) return fail(FA_ERR_INVALID, "cache is NULL");
  if (int r = check_ptr(K, "K", true)) return r;
  if (int r = check_ptr(V, "V", true)) return r;
  const bool mid = plan->M > 0;
  if (int r = check_ptr(phiT, "phiT", mid)) return r;
  if (int r = check_ptr(cache->F_K, "cache->F_K", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->F_V, "cache->F_V", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->E_K, "cache->E_K", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->E_V, "cache->E_V", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->C_K, "cache->C_K", plan->c_elems > 0)) return r;
  if (int r = check_ptr(cache->C_V, "cache->C_V", plan->c_elems > 0)) return r;
  const char* why = nullptr;
  cudaError_t e = fa::launch_compress(plan, K, V, phiT, cache, static_cast<cudaStream_t>(stream), &why);
  if (e != cudaSuccess) {
    if (why) return fail(FA_ERR_CUDA, "fa_compress: %s", why);
    return cuda_fail(e, "fa_compress: launch");
  }
  return FA_OK;
}

static int decode_checks(const fa_plan* plan) {
  if (int r = check_plan(plan)) return r;
  const int G = plan->G;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(FA_ERR_UNSUPPORTED, "fa_decode supports Hq/Hkv in {1, 2, 4, 8}, got %d", G);
  if (plan->M > 0 && plan->shape.k > FA_MAX_K_DECODE)
    return fail(FA_ERR_UNSUPPORTED, "fa_decode supports k <= %d, got %d", FA_MAX_K_DECODE, plan->shape.k);
  if (plan->P >= (1 << 21)) return fail(FA_ERR_UNSUPPORTED, "fa_decode supports P < 2^21");
  return FA_OK;
}

}  // extern "C"

int fa::decode_setup(const fa_plan* plan, int requested, fa::DecodeConfig* c) {
  if (int r = decode_checks(plan)) return r;
  const char* why = nullptr;
  cudaError_t e = fa::decode_configure(plan, requested, c, &why);
  if (e == cudaSuccess) return FA_OK;
  if (why) return fail(FA_ERR_UNSUPPORTED, "fa_decode: %s", why);
  return cuda_fail(e, "fa_decode: configure");
}

extern "C" {

size_t fa_decode_workspace_size(const fa_plan* plan, int32_t num_splits) {
  fa::DecodeConfig c;
  if (fa::decode_setup(plan, num_splits, &c) != FA_OK) return 0;
  return c.qw_bytes + c.rec_bytes;
}

int fa_decode_describe(const fa_plan* plan, int32_t num_splits, fa_decode_info* info) {
  if (!info) return fail(FA_ERR_INVALID, "info is NULL");
  fa::DecodeConfig c;
  if (int r = fa::decode_setup(plan, num_splits, &c)) return r;
  const bool mid = plan->M > 0;
  info->split_kernel = !mid ? FA_SPLIT_NONE
                       : c.tc ? FA_SPLIT_TC_TOKEN_MAJOR
                       : c.cl ? FA_SPLIT_TC_CLUSTER
                       : c.hm ? FA_SPLIT_WARP_MMA
                              : FA_SPLIT_CUDA_CORES;
  info->num_splits = c.n_splits;
  info->cluster = c.cl ? c.cl_C : 1;
  // prologue (with the sink / recent rows on the tensor-core and warp-MMA paths), the split
  // kernel (with the sink / recent rows on the CUDA-core path), the combine
  const bool split_launch = mid || plan->S + plan->R > 0;
  info->launches = (mid ? 1 : 0) + (split_launch ? 1 : 0) + 1;
  return FA_OK;
}

int fa_decode(const fa_plan* plan, const void* q, const fa_cache* cache, void* out,
              int32_t out_dtype, void* workspace, size_t workspace_bytes, int32_t num_splits,
              void* stream) {
  if (int r = decode_checks(plan)) return r;
  if (out_dtype != FA_BF16 && out_dtype != FA_F32)
    return fail(FA_ERR_INVALID, "unknown out_dtype %d", out_dtype);
  if (!cache) return fail(FA_ERR_INVALID, "cache is NULL");
  if (int r = check_ptr(q, "q", true)) return r;
  if (int r = check_ptr(out, "out", true)) return r;
  if (int r = check_ptr(cache->F_K, "cache->F_K", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->F_V, "cache->F_V", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->E_K, "cache->E_K", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->E_V, "cache->E_V", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->C_K, "cache->C_K", plan->c_elems > 0)) return r;
  if (int r = check_ptr(cache->C_V, "cache->C_V", plan->c_elems > 0)) return r;
  if (int r = check_ptr(workspace, "workspace", true)) return r;
  fa::DecodeConfig c;
  if (int r = fa::decode_setup(plan, num_splits, &c)) return r;
  if (workspace_bytes < c.qw_bytes + c.rec_bytes)
    return fail(FA_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                workspace_bytes, c.qw_bytes + c.rec_bytes);
  cudaError_t e = fa::launch_decode(plan, c, q, cache, out, out_dtype, workspace,
                                    static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_decode: launch");
  return FA_OK;
}

int fa_append(fa_plan* plan, const void* k_new, const void* v_new, const fa_cache* cache,
              void* stream) {
  if (int r = check_plan(plan)) return r;
  if (plan->M < 1) return fail(FA_ERR_UNSUPPORTED, "fa_append needs a middle span (M >= 1)");
  if (plan->M >= plan->P)
    return fail(FA_ERR_UNSUPPORTED, "no room left: M = P = %d (see fa_plan_reserve)", plan->P);
  if (plan->kk > FA_MAX_K_DECODE)
    return fail(FA_ERR_UNSUPPORTED, "fa_append supports k <= %d, got %d", FA_MAX_K_DECODE, plan->kk);
  if (!cache) return fail(FA_ERR_INVALID, "cache is NULL");
  if (int r = check_ptr(k_new, "k_new", true)) return r;
  if (int r = check_ptr(v_new, "v_new", true)) return r;
  if (int r = check_ptr(cache->F_K, "cache->F_K", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->F_V, "cache->F_V", plan->f_elems > 0)) return r;
  if (int r = check_ptr(cache->E_K, "cache->E_K", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->E_V, "cache->E_V", plan->e_elems > 0)) return r;
  if (int r = check_ptr(cache->C_K, "cache->C_K", plan->c_elems > 0)) return r;
  if (int r = check_ptr(cache->C_V, "cache->C_V", plan->c_elems > 0)) return r;
  cudaError_t e = fa::launch_append(plan, k_new, v_new, cache, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_append: launch");
  plan->M += 1;
  plan->shape.L += 1;
  if (plan->R > 0) plan->recent_head = (plan->recent_head + 1) % plan->R;
  return FA_OK;
}

static int sensitivity_setup(const fa_shape* shape, fa_plan* plan, fa::DecodeConfig* c,
                             size_t* bytes) {
  if (!shape) return fail(FA_ERR_INVALID, "shape is NULL");
  if (int r = fa::sensitivity_plan(shape, plan)) return r;  // fa_plan_init set the message
  if (int r = fa::decode_setup(plan, 0, c)) return r;
  *bytes = fa::sensitivity_out_offset(*c) +
           (size_t)plan->shape.B * plan->shape.Hq * FA_HEAD_DIM * sizeof(float);
  return FA_OK;
}

size_t fa_dim_sensitivity_workspace_size(const fa_shape* shape) {
  fa_plan plan;
  fa::DecodeConfig c;
  size_t bytes = 0;
  return sensitivity_setup(shape, &plan, &c, &bytes) == FA_OK ? bytes : 0;
}

int fa_dim_sensitivity(const fa_shape* shape, const void* q, const void* K, const void* noise,
                       float* scores, void* workspace, size_t workspace_bytes, void* stream) {
  fa_plan plan;
  fa::DecodeConfig c;
  size_t need = 0;
  if (int r = sensitivity_setup(shape, &plan, &c, &need)) return r;
  if (int r = check_ptr(q, "q", true)) return r;
  if (int r = check_ptr(K, "K", true)) return r;
  if (int r = check_ptr(noise, "noise", true)) return r;
  if (int r = check_ptr(scores, "scores", true)) return r;
  if (int r = check_ptr(workspace, "workspace", true)) return r;
  if (workspace_bytes < need)
    return fail(FA_ERR_INVALID, "workspace of %zu bytes is smaller than the %zu required",
                workspace_bytes, need);
  cudaError_t e = fa::launch_sensitivity(&plan, c, q, K, noise, scores, workspace,
                                         static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_dim_sensitivity: launch");
  return FA_OK;
}

int fa_select_dims(const float* scores, int32_t Hkv, int32_t n_compressed, uint8_t* mask_out) {
  if (!scores || !mask_out) return fail(FA_ERR_INVALID, "NULL argument");
  if (Hkv < 1 || Hkv > FA_MAX_KV_HEADS || n_compressed < 0 || n_compressed > FA_HEAD_DIM)
    return fail(FA_ERR_INVALID, "Hkv=%d or n_compressed=%d out of range", Hkv, n_compressed);
  for (int g = 0; g < Hkv; ++g) {
    const float* sc = scores + g * FA_HEAD_DIM;
    for (int d = 0; d < FA_HEAD_DIM; ++d) {
      // rank of d in (score, index) order; NaN scores rank last
      int rank = 0;
      const bool dn = sc[d] != sc[d];
      for (int e = 0; e < FA_HEAD_DIM; ++e) {
        const bool en = sc[e] != sc[e];
        const bool before = (en != dn) ? dn : (dn ? e < d : (sc[e] < sc[d] || (sc[e] == sc[d] && e < d)));
        rank += before ? 1 : 0;
      }
      mask_out[g * FA_HEAD_DIM + d] = rank < n_compressed ? 1 : 0;
    }
  }
  return FA_OK;
}

int fa_watchdog_selftest(uint32_t wait_ns, void* stream) {
  if (wait_ns < 1000u || wait_ns > 1000000000u)
    return fail(FA_ERR_INVALID, "wait_ns=%u outside [1 us, 1 s]", wait_ns);
  cudaError_t e = fa::launch_watchdog_selftest(wait_ns, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_watchdog_selftest: launch");
  return FA_OK;
}

int fa_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "fa_device_status: stream");
  unsigned int w = 0;
  e = fa::read_and_clear_watchdog(&w);
  if (e != cudaSuccess) return cuda_fail(e, "fa_device_status: watchdog");
  if (w != 0)
    return fail(FA_ERR_DEVICE, "kernel %u hit the wait limit at site %u", w >> 8, w & 0xFFu);
  return FA_OK;
}

}  // extern "C"
