// kda_recurrence.cu — the recurrence kernel of the split variant (one CTA per
// (sequence, head) over records written by the prepare kernel; body in
// kda_recurrence.cuh).
#include "kda_recurrence.cuh"

namespace kda {
namespace rec {
extern const uint32_t kSmemAllocBytes = kSmemAlloc;
extern const int kThreadsPerCta = kThreads;
}

__global__ void __launch_bounds__(rec::kThreads, 1)
kda_recurrence_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  extern __shared__ uint8_t smem_raw[];
  recurrence_body<false>(p, maps, smem_raw, blockIdx.x);
}

}  // namespace kda
