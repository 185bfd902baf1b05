// kda_fused.cu — the fused variant: one launch in which CTAs 0 .. R-1 each carry
// the recurrence of one (sequence, head) (R = N H) and every other CTA runs the
// chunk-local prepare over the records in chunk-major order, raising a ready
// flag per record that the recurrence CTAs acquire before loading it.  All CTAs
// are co-resident (cooperative launch, one CTA per SM), the prepare side never
// waits on the recurrence side, and every wait is bounded, so the launch always
// ends.  This is the one-launch, one-CTA-per-(sequence, head) design next to the
// prepare/recurrence pair ("fused" vs "decomp" in FlashInfer PR #4633
// "Description"), with the prepare work spread over the SMs the recurrence
// leaves idle; it pays off when R is small next to the SM count.
#include "kda_prepare.cuh"
#include "kda_recurrence.cuh"

namespace kda {
namespace fused {
extern const int kThreadsPerCta = rec::kThreads;
extern const uint32_t kSmemAllocBytes = rec::kSmemAlloc > prep::kSmemAlloc ? rec::kSmemAlloc : prep::kSmemAlloc;
}

__global__ void __launch_bounds__(rec::kThreads, 1)
kda_fused_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                 int64_t prep_items) {
  extern __shared__ uint8_t smem_raw[];
  if (static_cast<int32_t>(blockIdx.x) < rec_ctas) {
    recurrence_body<true>(p, maps, smem_raw, blockIdx.x);
  } else {
    if (threadIdx.x >= prep::kThreads) return;   // the prepare body uses 256 threads
    prepare_body<true>(p, maps, smem_raw, blockIdx.x - rec_ctas, gridDim.x - rec_ctas, prep_items);
  }
}

}  // namespace kda
