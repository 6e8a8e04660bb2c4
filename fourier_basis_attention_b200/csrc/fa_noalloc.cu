// fa_noalloc.cu -- fa_decode_noalloc: one decode step with library-owned scratch.
//
// For callers that cannot allocate device memory (plug-ins inside a framework that owns
// every allocation, serving loops that pooled all of HBM at start-up, paths that must not
// pay cudaMalloc's implicit synchronisation). The split-L partial records and the
// per-query coefficient vectors live in one fixed device array below instead of a
// caller-provided workspace; everything else is fa_decode itself.
#include <stdio.h>

#include <mutex>

#include "fa_host.h"

namespace {

constexpr int kMaxDevices = 64;

// The scratch. In host code `g_scratch` names a host-side stand-in, not device memory:
// its device address comes from cudaGetSymbolAddress (see scratch_address below).
static __device__ __align__(256) unsigned char g_scratch[FA_NOALLOC_SCRATCH_BYTES];

typedef int (*PFN_ctxGetCurrent)(void** ctx);  // CUresult cuCtxGetCurrent(CUcontext*)

std::mutex g_mu;
struct ScratchEntry {
  void* ctx;   // the CUDA context the address belongs to
  void* addr;  // device address of g_scratch in that context
};
ScratchEntry g_addr[kMaxDevices] = {};

// Current CUDA context (the driver's handle), or nullptr if it cannot be read.
void* current_context() {
  static PFN_ctxGetCurrent fn = nullptr;
  static bool looked = false;
  if (!looked) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_ctxGetCurrent>(p);
    looked = true;
  }
  void* ctx = nullptr;
  if (!fn || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of g_scratch on the current device. It is looked up once per device and
// context: after cudaDeviceReset the library's module is loaded into a new context with a
// new address, so a changed context handle triggers a fresh lookup.
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fa::set_last_error(FA_ERR_CUDA, "fa_decode_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return fa::set_last_error(FA_ERR_UNSUPPORTED, "fa_decode_noalloc: device index out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  void* ctx = current_context();
  ScratchEntry& ent = g_addr[dev];
  if (!ent.addr || !ctx || ent.ctx != ctx) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || !p) {
      char msg[256];
      snprintf(msg, sizeof(msg), "fa_decode_noalloc: cudaGetSymbolAddress failed: %s",
               cudaGetErrorString(e));
      return fa::set_last_error(FA_ERR_CUDA, msg);
    }
    // the context handle is read after the lookup, which may have created the context
    ent.ctx = current_context();
    ent.addr = p;
  }
  *out = ent.addr;
  return FA_OK;
}

}  // namespace

extern "C" int fa_decode_noalloc(const fa_plan* plan, const void* q, const fa_cache* cache,
                                 void* out, int32_t out_dtype, int32_t num_splits,
                                 void* stream) {
  fa::DecodeConfig c;
  if (int r = fa::decode_setup(plan, num_splits, &c)) return r;  // precise reason recorded
  size_t need = c.qw_bytes + c.rec_bytes;
  int splits = num_splits;
  if (need > FA_NOALLOC_SCRATCH_BYTES && num_splits <= 0) {
    // lower the automatic split count until the partial records fit
    for (splits = c.n_splits - 1; splits >= 1; --splits) {
      need = fa_decode_workspace_size(plan, splits);
      if (need != 0 && need <= FA_NOALLOC_SCRATCH_BYTES) break;
    }
    if (splits < 1) splits = 1;
  }
  if (need > FA_NOALLOC_SCRATCH_BYTES) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "fa_decode_noalloc: needs %zu bytes of scratch, the built-in scratch holds %u; "
             "use fa_decode with a workspace",
             need, (unsigned)FA_NOALLOC_SCRATCH_BYTES);
    return fa::set_last_error(FA_ERR_UNSUPPORTED, msg);
  }
  void* scratch = nullptr;
  if (int r = scratch_address(&scratch)) return r;
  return fa_decode(plan, q, cache, out, out_dtype, scratch, FA_NOALLOC_SCRATCH_BYTES, splits,
                   stream);
}
