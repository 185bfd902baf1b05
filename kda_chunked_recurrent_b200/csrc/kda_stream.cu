// kda_stream.cu — the stream variant: one cooperative launch of one 512-thread CTA per
// SM that holds the whole SM's tensor memory (512 columns) and about 223 KB of shared
// memory, split in two halves.  On CTA b < R (R = N H chains) the first half (threads
// 0..255, 256 columns, 104 KB) carries the recurrence of one (sequence, head) (body in
// kda_chain.cuh) and the second half runs a prepare group; on the other CTAs both halves
// run prepare groups.  The prepare groups take items (chunk, chain) from one counter in
// chunk-major order and raise a ready flag per record, so the prepare work runs on every
// SM, beside the recurrences, and its records are read back from L2 shortly after they
// were written.  The prepare groups never wait on the recurrences and every wait is
// bounded, so the launch always ends.
//
// (One CTA per SM: the runtime admits kernels that allocate tensor memory one CTA per SM
// in a cooperative launch, so the two roles share a CTA instead of each having one.)
//
// This is the one-launch design next to the prepare/recurrence pair ("fused" vs
// "decomp" in FlashInfer PR #4633 "Description"), with the prepare work spread over
// all SMs instead of the CTA of each (sequence, head).
#include "kda_chain.cuh"
#include "kda_prepare.cuh"

namespace kda {
namespace stream {
constexpr int kThreads = 2 * prep::kThreads;
constexpr uint32_t kHalfBytes = prep::kGroupBytes;   // one half of the CTA's shared memory
extern const int kThreadsPerCta = kThreads;
extern const uint32_t kSmemAllocBytes = 2 * kHalfBytes + 1024;
static_assert(chain::kThreads == prep::kThreads, "the recurrence takes one half of the CTA");
static_assert(chain::kBytes <= kHalfBytes, "the recurrence fits one half of the shared memory");
static_assert(2 * kHalfBytes + 1024 <= 227 * 1024, "shared memory budget");
constexpr uint32_t kPrepBar = 3;   // named barriers 3, 4 of the prepare groups (the chain uses 1, 2)
}  // namespace stream

template <bool kFE>
__device__ __forceinline__ void stream_body(const KdaParams& p, const SplitMaps& maps,
                                            int32_t rec_ctas, int64_t prep_items) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  const int warp = threadIdx.x >> 5;
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  const int half = threadIdx.x >> 8;
  if (half == 0 && static_cast<int32_t>(blockIdx.x) < rec_ctas) {
    chain_body(p, maps, smem_raw, blockIdx.x, tbase);
  } else {
    // (the item order is claimed from the counter; first / stride are unused)
    prepare_body<true, kFE, true>(p, maps, smem_raw, half, 0, 1, prep_items,
                                  PrepGroupRes{tbase + 256u * half, stream::kPrepBar + half});
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

__global__ void __launch_bounds__(stream::kThreads, 1)
kda_stream_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                  int64_t prep_items) {
  stream_body<false>(p, maps, rec_ctas, prep_items);
}

// the same with the input front end compiled into the prepare side
__global__ void __launch_bounds__(stream::kThreads, 1)
kda_stream_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps, int32_t rec_ctas,
                     int64_t prep_items) {
  stream_body<true>(p, maps, rec_ctas, prep_items);
}

}  // namespace kda
