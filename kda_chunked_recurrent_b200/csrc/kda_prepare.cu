// kda_prepare.cu — the prepare kernel of the split variant (two 256-thread CTAs
// per SM walking every (chunk slot, head) record; body in kda_prepare.cuh).
#include "kda_prepare.cuh"

namespace kda {
namespace prep {
extern const uint32_t kSmemAllocBytes = kSmemAlloc;
}

__global__ void __launch_bounds__(prep::kThreads, 2)
kda_prepare_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  prepare_body<false>(p, maps, smem_raw, 0, blockIdx.x, gridDim.x, p.slots * p.H);
}

// the same with the input front end compiled in (prefill from raw projections)
__global__ void __launch_bounds__(prep::kThreads, 2)
kda_prepare_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  prepare_body<false, true>(p, maps, smem_raw, 0, blockIdx.x, gridDim.x, p.slots * p.H);
}

}  // namespace kda
