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
// written earlier in the same call (the area starts zeroed at load time).  The
// status word in the area is never read through this entry point, so the modes
// that report only through it (validate, the forced-timeout test hook) are refused.
#include <cuda_runtime.h>

#include "../../include/kda_prefill.h"

namespace {

constexpr size_t kScratchBytes = KDA_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_kda_noalloc_scratch[kScratchBytes];

kda_status_t current_device_supported() {
  int dev = -1, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return KDA_ERR_UNSUPPORTED_DEVICE;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return KDA_ERR_UNSUPPORTED_DEVICE;
  return (major == 10 && minor == 0) ? KDA_OK : KDA_ERR_UNSUPPORTED_DEVICE;
}

// Device address of the built-in area on the current device.  The array's name in
// host code is only a stand-in for the symbol, so the address is looked up with the
// device current, on every call: the lookup is cheap, and a cached address would go
// stale if the context were torn down and the module loaded again elsewhere.
kda_status_t scratch_on_current_device(void** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_kda_noalloc_scratch);
  if (e != cudaSuccess || p == nullptr) {
    (void)cudaGetLastError();   // a failed lazy load leaves no sticky error behind
    return KDA_ERR_SCRATCH_UNAVAILABLE;
  }
  *out = p;
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
  // the status word of the built-in area is not readable here: refuse the modes that
  // would report only through it (kda_prefill with a workspace of the caller's serves them)
  if (options && (options->flags & (KDA_FLAG_VALIDATE | KDA_FLAG_TEST_FORCE_TIMEOUT)))
    return KDA_ERR_BAD_OPTION;
  const int has_ckpt = ckpt_state != nullptr;
  // options and shape first, with the codes kda_prefill would give
  char note[8];
  kda_status_t st = kda_prefill_describe(shape, has_ckpt, options, note, sizeof(note));
  if (st != KDA_OK) return st;
  st = current_device_supported();
  if (st != KDA_OK) return st;
  const size_t need = kda_prefill_workspace_size(shape, has_ckpt, options);
  if (need == 0) return KDA_ERR_BAD_SHAPE;
  if (need > kScratchBytes) return KDA_ERR_WORKSPACE_TOO_SMALL;  // shape too large for the area
  void* scratch = nullptr;
  st = scratch_on_current_device(&scratch);
  if (st != KDA_OK) return st;
  return kda_prefill(q, k, v, g, beta, scale, h0, cu_seqlens, shape, out, ht, ckpt_state,
                     ckpt_offsets, scratch, kScratchBytes, options, stream);
}
