// kda_stream.cu — the stream variant: one cooperative launch of two 256-thread CTAs
// per SM.  CTAs 0 .. R-1 each carry the recurrence of one (sequence, head) (R = N H,
// body in kda_chain.cuh); every other CTA runs the chunk-local prepare over the
// records in chunk-major order and raises a ready flag per record.  Both kinds fit two
// to an SM (256 tensor-memory columns and at most about 110 KB of shared memory each),
// so the prepare work runs on every SM, beside the recurrences, and its records are
// read back from L2 shortly after they were written.  The prepare side never waits
// on the recurrence side and every wait is bounded, so the launch always ends.
//
// This is the one-launch design next to the prepare/recurrence pair ("fused" vs
// "decomp" in FlashInfer PR #4633 "Description"), with the prepare work spread over
// all SMs instead of the CTA of each (sequence, head).
#include "kda_chain.cuh"
#include "kda_prepare.cuh"

namespace kda {
namespace stream {
constexpr int kThreads = 256;
extern const int kThreadsPerCta = kThreads;
extern const uint32_t kSmemAllocBytes =
    chain::kSmemAlloc > prep::kSmemAlloc ? chain::kSmemAlloc : prep::kSmemAlloc;
static_assert(prep::kThreads == kThreads && chain::kThreads == kThreads, "one CTA size");
}  // namespace stream

template <bool kFE>
__device__ __forceinline__ void stream_body(const KdaParams& p, const SplitMaps& maps,
                                            int32_t rec_ctas, int64_t prep_items) {
  extern __shared__ uint8_t smem_raw[];
  if (static_cast<int32_t>(blockIdx.x) < rec_ctas) {
    chain_body(p, maps, smem_raw, blockIdx.x);
  } else {
    prepare_body<true, kFE, true>(p, maps, smem_raw, 0,
                                  static_cast<int64_t>(blockIdx.x) - rec_ctas,
                                  static_cast<int64_t>(gridDim.x) - rec_ctas, prep_items);
  }
}

__global__ void __launch_bounds__(stream::kThreads, 2)
kda_stream_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                  int64_t prep_items) {
  stream_body<false>(p, maps, rec_ctas, prep_items);
}

// the same with the input front end compiled into the prepare side
__global__ void __launch_bounds__(stream::kThreads, 2)
kda_stream_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                     int64_t prep_items) {
  stream_body<true>(p, maps, rec_ctas, prep_items);
}

}  // namespace kda
