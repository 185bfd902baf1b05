// kda_noalloc.cu — a prefill entry point that allocates nothing.
//
// Some callers cannot call cudaMalloc: code that runs while a CUDA graph is
// being captured into a memory pool it does not own, plugins inside a host
// application that owns every device allocation, or real-time paths where an
// allocation (and the device synchronisation it may trigger) is not allowed.
// kda_prefill asks such callers for a workspace they may not be able to get.
// kda_prefill_noalloc instead uses a scratch area that is part of this library:
// a file-scope __device__ array of KDA_NOALLOC_SCRATCH_BYTES, created when the
// library's device code is loaded on a GPU and kept until the process exits.
//
// It runs exactly the same kernels as kda_prefill (it calls kda_prefill with the
// built-in area as the workspace), so results are identical.  Nothing in the
// area has to be cleared between calls: every table and tile a call reads is
// written earlier in the same call (the area starts zeroed at load time).
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/kda_prefill.h"

namespace {

constexpr size_t kScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of the built-in area on the current device.  The array's name
// in host code is only a stand-in for the symbol, so the address is looked up
// once per device (with that device current) and remembered.
kda_status_t scratch_on_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
    return KDA_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_kda_noalloc_scratch) != cudaSuccess || p == nullptr)
      return KDA_ERR_LAUNCH_FAILED;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return KDA_OK;
}

}  // namespace

extern "C" kda_status_t kda_prefill_noalloc(const void* q, const void* k, const void* v,
                                            const float* g, const void* beta, float scale,
                                            const float* h0, const int32_t* cu_seqlens,
                                            const kda_shape_t* shape, void* out, float* ht,
                                            float* ckpt_state, const int32_t* ckpt_offsets,
                                            const kda_options_t* options, void* stream) {
  if (shape == nullptr) return KDA_ERR_NULL_ARG;
  const size_t need = kda_prefill_workspace_size(shape, ckpt_state != nullptr, options);
  if (need == 0)  // invalid shape or options: kda_prefill names the error, launching nothing
    return kda_prefill(q, k, v, g, beta, scale, h0, cu_seqlens, shape, out, ht, ckpt_state,
                       ckpt_offsets, nullptr, 0, options, stream);
  if (need > kScratchBytes) return KDA_ERR_WORKSPACE_TOO_SMALL;  // shape too large for the area
  void* scratch = nullptr;
  const kda_status_t st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  return kda_prefill(q, k, v, g, beta, scale, h0, cu_seqlens, shape, out, ht, ckpt_state,
                     ckpt_offsets, scratch, kScratchBytes, options, stream);
}
