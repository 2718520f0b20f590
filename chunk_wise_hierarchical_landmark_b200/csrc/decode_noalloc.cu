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
//    device); make that first call before any stream capture.
// No cudaMalloc, cudaFree or allocating library routine is called here.
#include <mutex>

#include "../../include/hils.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];  // device address of g_decode_scratch, per device

// Device address of the scratch array on the current device (set-up on the
// first call per device).  Returns nullptr and fills *e on failure.
void *scratch_on_current_device(cudaError_t *e) {
  int dev = -1;
  *e = cudaGetDevice(&dev);
  if (*e != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *e = cudaErrorInvalidDevice;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *ptr = nullptr;
    *e = cudaGetSymbolAddress(&ptr, g_decode_scratch);
    if (*e != cudaSuccess) return nullptr;
    g_scratch_addr[dev] = ptr;
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
