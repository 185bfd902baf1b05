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
// two prepare groups of 256 threads per prepare CTA (the recurrence CTAs leave
// their last two warps idle)
constexpr int kThreads = 2 * prep::kThreads;
constexpr uint32_t kPrepBytes = 2 * prep::kGroupBytes + 1024;
extern const int kThreadsPerCta = kThreads;
extern const uint32_t kSmemAllocBytes = rec::kSmemAlloc > kPrepBytes ? rec::kSmemAlloc : kPrepBytes;
static_assert(rec::kThreads <= kThreads, "recurrence warps fit the CTA");
static_assert(kPrepBytes <= 227 * 1024 && rec::kSmemAlloc <= 227 * 1024, "shared memory budget");
}

// prep_groups: prepare groups per prepare CTA (1 or 2).  Few chains need little
// prepare throughput, and one group then leaves more memory bandwidth to them.
template <bool kFE>
__device__ __forceinline__ void fused_body(const KdaParams& p, const SplitMaps& maps,
                                           int32_t rec_ctas, int64_t prep_items,
                                           int32_t prep_groups) {
  extern __shared__ uint8_t smem_raw[];
  if (static_cast<int32_t>(blockIdx.x) < rec_ctas) {
    recurrence_body<true>(p, maps, smem_raw, blockIdx.x);
  } else {
    const int grp = threadIdx.x / prep::kThreads;
    if (grp >= prep_groups) return;
    const int64_t groups = prep_groups * static_cast<int64_t>(gridDim.x - rec_ctas);
    prepare_body<true, kFE>(p, maps, smem_raw, grp,
                            prep_groups * static_cast<int64_t>(blockIdx.x - rec_ctas) + grp,
                            groups, prep_items);
  }
}

__global__ void __launch_bounds__(fused::kThreads, 1)
kda_fused_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                 int64_t prep_items, int32_t prep_groups) {
  fused_body<false>(p, maps, rec_ctas, prep_items, prep_groups);
}

// the same with the input front end compiled into the prepare side
__global__ void __launch_bounds__(fused::kThreads, 1)
kda_fused_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                    int64_t prep_items, int32_t prep_groups) {
  fused_body<true>(p, maps, rec_ctas, prep_items, prep_groups);
}

}  // namespace kda
