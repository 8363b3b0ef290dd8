// lwm_attn_fwd_noalloc: the forward pass with its scratch memory in a
// fixed, library-owned device array instead of a caller-supplied workspace.
//
// The pages have no counterpart to this; it exists for callers that cannot
// allocate device memory at the point where they run the forward pass (see
// the declaration in lwm_attn.h).  It takes the ordinary forward path
// unchanged: it only supplies the workspace pointer and size.
#include <cuda_runtime.h>

#include <mutex>

#include "lwm_attn.h"

namespace {

// 40 MiB: the forward's scratch (status word, per-tile segment bounds and the
// rotated q and k) for up to about 10M bf16 elements per tensor, e.g. 2,048
// tokens x 32 heads x 128.  Every GPU that loads this library holds it until
// the process exits.
constexpr size_t kNoAllocScratchBytes = (size_t)40 << 20;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name is only a host-side stand-in, so
// the address must come from cudaGetSymbolAddress with the device current.
lwm_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return LWM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LWM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LWM_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return LWM_OK;
}

}  // namespace

extern "C" {

lwm_status lwm_attn_fwd_noalloc(const lwm_attn_desc* desc, const void* q, const void* k,
                                const void* v, void* o, float* lse, void* stream) {
  const size_t need = lwm_attn_workspace_size(desc, 0);
  if (need == 0) {
    // invalid or unsupported description: let the ordinary entry say which
    return lwm_attn_fwd(desc, q, k, v, o, lse, nullptr, 0, stream);
  }
  if (need > kNoAllocScratchBytes) return LWM_ERR_WORKSPACE;
  void* scratch = nullptr;
  const lwm_status s = scratch_for_current_device(&scratch);
  if (s != LWM_OK) return s;
  return lwm_attn_fwd(desc, q, k, v, o, lse, scratch, kNoAllocScratchBytes, stream);
}

lwm_status lwm_attn_fwd_noalloc_read_status(void* stream) {
  void* scratch = nullptr;
  const lwm_status s = scratch_for_current_device(&scratch);
  if (s != LWM_OK) return s;
  return lwm_attn_read_status(scratch, stream);
}

}  // extern "C"
