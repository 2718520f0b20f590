// Allocation-free decode entry point.
//
// Some callers cannot hand the library a workspace: their device memory is
// owned by another allocator (for instance a serving framework that reserves
// the whole GPU for its own pool at start-up and forbids cudaMalloc outside
// it), or they run the decode step in a loop where a cudaMalloc/cudaFree pair
// would synchronise the device every token.  For them this file keeps the
// decode step's scratch in a fixed device array that lives in the library
// itself, so a call needs only the caller's inputs and outputs.
//
// Limits and rules (also stated in include/hils.h):
//  - the array holds kScratchBytes (32 MiB) on every GPU that loads the
//    library, until the process exits; shapes whose decode scratch is larger
//    are rejected with HILS_ERR_WORKSPACE before anything is launched;
//  - all calls share the array and it keeps the last call's contents; every
//    call writes each scratch entry it later reads, so nothing needs clearing,
//    but calls that overlap on the GPU (other streams, other host threads)
//    race on it and must be serialised by the caller;
//  - the first call on a device looks the array's device address up with
//    cudaGetSymbolAddress (which can load the library's module on that
//    device); make that first call before any stream capture.  The address
//    is tied to the device's context: when the context changes (a
//    cudaDeviceReset, or a primary context released and created again), the
//    module is loaded anew and the next call looks the address up again.
// No cudaMalloc, cudaFree or allocating library routine is called here.
#include <cuda.h>

#include <mutex>

#include "../../include/hils.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];          // device address of g_decode_scratch, per device
unsigned long long g_scratch_ctx[kMaxDevices];  // id of the context it was resolved in

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current context (0 if it cannot be read;
// then the cached address is trusted as it is).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static bool looked_up = false;
  if (!looked_up) {
    void *f1 = nullptr, *f2 = nullptr;
    cudaDriverEntryPointQueryResult r1, r2;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f1, cudaEnableDefault, &r1) == cudaSuccess &&
        r1 == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f1);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f2, cudaEnableDefault, &r2) == cudaSuccess &&
        r2 == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f2);
    looked_up = true;
  }
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx &&
      get_id(ctx, &id) == CUDA_SUCCESS)
    return id;
  return 0;
}

// Device address of the scratch array on the current device (set-up on the
// first call per device, and again whenever the device's context changed).
// Returns nullptr and fills *e on failure.
void *scratch_on_current_device(cudaError_t *e) {
  int dev = -1;
  *e = cudaGetDevice(&dev);
  if (*e != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *e = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  // cudaGetSymbolAddress makes the device's primary context current, so the
  // context is read after it on the first call
  if (g_scratch_addr[dev]) {
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && ctx != g_scratch_ctx[dev]) g_scratch_addr[dev] = nullptr;
  }
  if (!g_scratch_addr[dev]) {
    void *ptr = nullptr;
    *e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (*e != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
    g_scratch_ctx[dev] = current_context_id();
  }
  *e = cudaSuccess;
  return g_scratch_addr[dev];
}

}  // namespace

extern "C" __attribute__((visibility("default"))) hils_status hils_decode_fwd_noalloc(
    const hils_params *p, const void *q, const void *k_cache, const void *v_cache,
    const void *lmk_k, int32_t *sel_idx, float *chunk_w, float *lse_lmk, void *out, float *lse,
    void *stream) {
  // invalid shapes: let the ordinary entry point report them (no CUDA call)
  const size_t need = hils_workspace_size(p, HILS_OP_DECODE);
  if (need == 0)
    return hils_decode_fwd(p, q, k_cache, v_cache, lmk_k, sel_idx, chunk_w, lse_lmk, out, lse,
                           nullptr, 0, stream);
  // shapes needing more scratch than the fixed array are refused up front
  if (need > kScratchBytes) {
    hils::hils_internal_set_error(
        "hils_decode_fwd_noalloc: these shapes need more decode scratch than the library's "
        "fixed 32 MiB array; call hils_decode_fwd with a workspace instead");
    return HILS_ERR_WORKSPACE;
  }
  cudaError_t e;
  void *scratch = scratch_on_current_device(&e);
  if (!scratch) {
    hils::hils_internal_set_error("hils_decode_fwd_noalloc: cudaGetSymbolAddress of the scratch array failed");
    return HILS_ERR_CUDA;
  }
  // the ordinary decode path, with the library's own array as its workspace
  return hils_decode_fwd(p, q, k_cache, v_cache, lmk_k, sel_idx, chunk_w, lse_lmk, out, lse,
                         scratch, kScratchBytes, stream);
}
