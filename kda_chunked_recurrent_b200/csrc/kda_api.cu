// kda_api.cu — host side of the C ABI declared in include/kda_prefill.h.
//
// Validation (pointers, sizes, alignment, aliasing, workspace) happens before
// any launch or write: lmdeploy PR #5050 ("Motivation") checks the paired
// checkpoint arguments before anything is mutated, and FlashInfer PR #4262
// ("Physical schedules and true in-place state update") rejects a partial
// h0/ht overlap.  Device metadata
// (cu_seqlens, ckpt_offsets) is never read on the host.  Launch order on the
// caller's stream: [schedule] -> prepare -> recurrence (split variant), or
// [schedule] -> ready-flag clear -> one cooperative launch (fused variant).
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/kda_prefill.h"
#include "kda_common.cuh"
#include "kda_token.cuh"

namespace kda {
__global__ void kda_schedule_kernel(const KdaParams p);
__global__ void kda_prepare_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps);
__global__ void kda_prepare_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps);
__global__ void kda_fused_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps,
                                    int32_t rec_ctas, int64_t prep_items, int32_t prep_groups);
__global__ void kda_recurrence_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps);
__global__ void kda_fused_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps,
                                 int32_t rec_ctas, int64_t prep_items, int32_t prep_groups);
__global__ void kda_stream_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps,
                                  int32_t rec_ctas, int64_t prep_items);
__global__ void kda_stream_fe_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps,
                                     int32_t rec_ctas, int64_t prep_items);
namespace prep { extern const uint32_t kSmemAllocBytes; }
namespace stream { extern const uint32_t kSmemAllocBytes; extern const int kThreadsPerCta; }
namespace rec { extern const uint32_t kSmemAllocBytes; extern const int kThreadsPerCta; }
namespace fused { extern const uint32_t kSmemAllocBytes; extern const int kThreadsPerCta; }
__global__ void kda_token_narrow_kernel(const TokenParams p);
__global__ void kda_token_wide_kernel(const TokenParams p);
__global__ void kda_token_narrow_fe_kernel(const TokenParams p);
__global__ void kda_token_wide_fe_kernel(const TokenParams p);
namespace tok {
extern const uint32_t kSmemNarrow;
extern const uint32_t kSmemWide;
extern const int kThreadsPerCta;
}
}  // namespace kda

using namespace kda;

namespace {

constexpr int kVersion = 100;  // 0.1.0
constexpr long long kDefaultWaitBudget = 2000000000LL;  // clock cycles (~1 s)

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

struct Range {
  uintptr_t lo, hi;  // [lo, hi)
  bool valid() const { return lo != 0 && hi > lo; }
};
Range rng(const void* p, size_t bytes) {
  return Range{reinterpret_cast<uintptr_t>(p), reinterpret_cast<uintptr_t>(p) + bytes};
}
bool overlap(const Range& a, const Range& b) {
  return a.valid() && b.valid() && a.lo < b.hi && b.lo < a.hi;
}
bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Resolved {
  int variant;
  bool fixed;
  WorkspaceLayout lay;
};

kda_status_t check_options(const kda_options_t* o) {
  if (!o) return KDA_OK;
  if (o->variant < KDA_VARIANT_AUTO || o->variant > KDA_VARIANT_STREAM) return KDA_ERR_BAD_OPTION;
  if (o->flags & ~(static_cast<uint32_t>(KDA_FLAG_VALIDATE | KDA_FLAG_TEST_FORCE_TIMEOUT |
                                         KDA_FLAG_CU_SEQLENS_I64)))
    return KDA_ERR_BAD_OPTION;
  return KDA_OK;
}

// The input front end's switches and parameters (pointers only; values of the
// device arrays are never read on the host).
kda_status_t check_frontend(const kda_frontend_t* fe) {
  if (!fe) return KDA_OK;
  if (fe->flags & ~static_cast<uint32_t>(KDA_FE_QK_L2NORM | KDA_FE_GATE | KDA_FE_BETA_LOGIT))
    return KDA_ERR_BAD_OPTION;
  if (fe->flags & KDA_FE_GATE) {
    if (!fe->A_log || !fe->dt_bias) return KDA_ERR_NULL_ARG;
    const float lb = fe->lower_bound;
    if (!(lb >= -5.0f && lb < 0.0f)) return KDA_ERR_BAD_OPTION;   // also rejects NaN
    if ((reinterpret_cast<uintptr_t>(fe->A_log) % 4) || (reinterpret_cast<uintptr_t>(fe->dt_bias) % 16))
      return KDA_ERR_MISALIGNED;
  }
  if ((fe->flags & KDA_FE_QK_L2NORM) && !(fe->l2_eps >= 0.0f && fe->l2_eps <= 1.0f))
    return KDA_ERR_BAD_OPTION;
  return KDA_OK;
}

uint32_t fe_bits(const kda_frontend_t* fe) {
  const uint32_t f = fe ? fe->flags : 0u;
  return (f & KDA_FE_QK_L2NORM ? 1u : 0u) | (f & KDA_FE_GATE ? 2u : 0u) |
         (f & KDA_FE_BETA_LOGIT ? 4u : 0u);
}

kda_status_t check_shape(const kda_shape_t* s, bool fixed, bool ckpt) {
  if (!s) return KDA_ERR_NULL_ARG;
  if (s->num_seqs < 1 || s->num_heads < 1 || s->total_tokens < 0 || s->max_seqlen < 0)
    return KDA_ERR_BAD_SHAPE;
  if (fixed && (s->total_tokens % s->num_seqs) != 0) return KDA_ERR_BAD_SHAPE;
  // 32-bit TMA coordinates of the per-record tiles: slots * H * 128 < 2^31
  const int64_t slots = chunk_slots(s->num_seqs, s->total_tokens, fixed, ckpt);
  if (slots * static_cast<int64_t>(s->num_heads) * 128 >= (int64_t(1) << 31)) return KDA_ERR_BAD_SHAPE;
  if (static_cast<int64_t>(s->num_seqs) * s->num_heads * 128 >= (int64_t(1) << 31))
    return KDA_ERR_BAD_SHAPE;
  return KDA_OK;
}

int sm_count();

// The fused launch keeps at least this many SMs for its prepare CTAs, which run
// one prepare group each up to kFusedOneGroupMaxChains chains and two above.
constexpr int kFusedMinPrepCtas = 16;
// Token kernel shape: 4 narrow CTAs (32 value columns each) per (sequence, head)
// below this many units, one wide CTA (all 128 columns) per unit from it on.
// Measured (kda_decode, T = 1, H = 12, ms narrow / wide): 48 units 0.0097 / 0.0104,
// 96 units 0.0103 / 0.0105, 144 units 0.0128 / 0.0116, 768 units 0.0311 / 0.0272,
// 3072 units 0.0956 / 0.0744.
constexpr int64_t kTokenWideMinUnits = 128;

bool token_wide(int64_t units, uint32_t force) {
  if (force & KDA_DECODE_NARROW) return false;
  if (force & KDA_DECODE_WIDE) return true;
  return units >= kTokenWideMinUnits;
}

// Launch the per-token kernel for `units` (sequence, head) pairs.
// (The kernels with the input front end compiled in are used only when tp.fe_flags
// asks for it, so the plain path keeps its register budget.)
kda_status_t launch_token(const TokenParams& tp, int64_t units, bool wide, cudaStream_t s) {
  static std::once_flag once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(once, [] {
    const void* narrow[] = {reinterpret_cast<const void*>(kda_token_narrow_kernel),
                            reinterpret_cast<const void*>(kda_token_narrow_fe_kernel)};
    const void* wide_k[] = {reinterpret_cast<const void*>(kda_token_wide_kernel),
                            reinterpret_cast<const void*>(kda_token_wide_fe_kernel)};
    for (int i = 0; i < 2; ++i) {
      cudaError_t e1 = cudaFuncSetAttribute(narrow[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            tok::kSmemNarrow);
      cudaError_t e2 = cudaFuncSetAttribute(wide_k[i], cudaFuncAttributeMaxDynamicSharedMemorySize,
                                            tok::kSmemWide);
      if (attr_err == cudaSuccess) attr_err = e1 != cudaSuccess ? e1 : e2;
    }
  });
  if (attr_err != cudaSuccess) return KDA_ERR_LAUNCH_FAILED;
  const bool fe = tp.fe_flags != 0;
  const unsigned grid = static_cast<unsigned>(wide ? units : units * 4);
  const uint32_t smem = wide ? tok::kSmemWide : tok::kSmemNarrow;
  if (wide && fe) kda_token_wide_fe_kernel<<<grid, tok::kThreadsPerCta, smem, s>>>(tp);
  else if (wide) kda_token_wide_kernel<<<grid, tok::kThreadsPerCta, smem, s>>>(tp);
  else if (fe) kda_token_narrow_fe_kernel<<<grid, tok::kThreadsPerCta, smem, s>>>(tp);
  else kda_token_narrow_kernel<<<grid, tok::kThreadsPerCta, smem, s>>>(tp);
  return KDA_OK;
}
constexpr int kFusedOneGroupMaxChains = 16;

// Per-shape variant table, from CUDA-event timings on one B200 (1965 MHz, ms per
// call, split / fused / hybrid): B1 T8192 H12 (12 chains of 128 chunks) 0.294 /
// 0.254 / -; B1 T512 H12 (12 chains of 8 chunks) 0.040 / 0.047 / -; B4 T8192 H12
// with checkpoints (48 chains) 0.485 / 0.380 / -; B6 T8192 H12 (72) 0.546 /
// 0.652 / 0.497; B8 T8192 H12 (96) 0.642 / 1.228 / 0.615; B8 T1024 H12 (96 chains
// of 16 chunks) 0.110 / 0.186 / 0.140.  The fused launch hides the prepare work
// behind the recurrence chains while the chains (one SM each) leave enough SMs to
// its prepare groups; the hybrid runs most of the prepare work first on every SM
// and hides only the last chunks; both need sequences long enough to overlap.
// The token variant (one token at a time, state slice in registers) wins while
// every sequence is short.  Measured ms per call, split / token, H = 12: N = 1 T = 16
// 0.025 / 0.015, T = 32 0.024 / 0.022, T = 64 0.024 / 0.037; N = 8 T = 16 0.026 /
// 0.022, T = 32 0.027 / 0.037; N = 32 T = 8 0.048 / 0.031, T = 16 0.048 / 0.049;
// N = 256 T = 8 0.258 / 0.156, T = 16 0.261 / 0.276.
struct VariantRule {
  int64_t max_chains;   // N H at most this
  int64_t min_chunks;   // and at least this many chunks in the longest sequence
  int64_t max_len;      // and no sequence longer than this
  int variant;          // -> this variant
};
constexpr VariantRule kVariantTable[] = {
    {16, 0, 32, KDA_VARIANT_TOKEN},
    {INT64_MAX, 0, 16, KDA_VARIANT_TOKEN},
    {56, 32, INT64_MAX, KDA_VARIANT_FUSED},
    {INT64_MAX, 64, INT64_MAX, KDA_VARIANT_HYBRID},
    {INT64_MAX, 0, INT64_MAX, KDA_VARIANT_SPLIT},
};

bool fused_eligible(const kda_shape_t* s) {
  const int64_t chains = static_cast<int64_t>(s->num_seqs) * s->num_heads;
  return chains + kFusedMinPrepCtas <= sm_count();
}

// The stream launch holds one CTA per SM; a chain takes half of one CTA, so at most one
// chain per SM, and every half without a chain runs a prepare group.
bool stream_eligible(const kda_shape_t* s) {
  const int64_t chains = static_cast<int64_t>(s->num_seqs) * s->num_heads;
  return chains <= static_cast<int64_t>(sm_count());
}

int64_t max_chunks_per_seq(const kda_shape_t* s, bool fixed, bool ckpt);

int choose_variant(const kda_shape_t* s, const kda_options_t* o) {
  if (o && o->variant != KDA_VARIANT_AUTO) return o->variant;
  const int64_t chains = static_cast<int64_t>(s->num_seqs) * s->num_heads;
  const int64_t chunks = max_chunks_per_seq(s, false, false);
  const int64_t len = s->max_seqlen > 0 ? s->max_seqlen : s->total_tokens;
  for (const VariantRule& rule : kVariantTable)
    if (chains <= rule.max_chains && chunks >= rule.min_chunks && len <= rule.max_len) {
      if ((rule.variant == KDA_VARIANT_FUSED || rule.variant == KDA_VARIANT_HYBRID) &&
          !fused_eligible(s))
        continue;
      if (rule.variant == KDA_VARIANT_STREAM && !stream_eligible(s)) continue;
      return rule.variant;
    }
  return KDA_VARIANT_SPLIT;
}

// Hybrid variant: how many of the last chunks of every sequence the fused launch's
// prepare groups make while its recurrence CTAs run.  The recurrence CTAs walk all jmax
// chunks (the first jmax - tail from the preceding prepare launch) at one chunk step per
// kFusedStepCycles; the 2 (SMs - R) prepare groups on the free SMs make one record per
// kFusedPrepCycles each, R records per chunk row.  The tail rows must be ready before the
// chains reach them, which they do if the groups make them within the chain's time:
//   tail R kFusedPrepCycles / (2 (SMs - R))  <=  jmax kFusedStepCycles,
// so tail = slack jmax (2 (SMs - R) / R) (kFusedStepCycles / kFusedPrepCycles).  Only the
// ratio of the two cycle counts enters, and it does not depend on the clock.  Measured on
// a B200 (CUDA events, 1965 MHz): a chunk step of the fused launch 1.87 us at B8 T8192 H12
// (3.7K cycles) while its records are ready in time.  A prepare group inside the fused
// launch makes a record in 10-11 us when the launch is prepare-bound (B6 and B4 T8192 H12
// fused: 20-22K cycles).  Swept on the hybrid at B8 and B6 T8192 H12, 22K per record is
// the best value of the rule (B8: tail 20 rows, 0.555 ms, against 0.556 at 24K, 0.558 at
// 26K and 0.559 at 29K; B6: tail 40, 0.437 against 0.441, 0.445 and 0.452), so the rule
// uses it.  The front-end
// prepare is slower by the measured ratio of the prepare launches at B8 T8192 H12
// (0.506 / 0.355 ms).  The slack keeps the producer ahead.
constexpr double kFusedStepCycles = 3700.0;
constexpr double kFusedPrepCycles = 22000.0;
constexpr double kFusedPrepCyclesFE = 22000.0 * 0.506 / 0.355;
constexpr double kHybridTailSlack = 0.9;
int64_t hybrid_tail_chunks(int64_t jmax, int64_t chains, bool frontend = false) {
  const double free_groups = 2.0 * (static_cast<double>(sm_count()) - static_cast<double>(chains));
  const double per_rec = frontend ? kFusedPrepCyclesFE : kFusedPrepCycles;
  const double tail = kHybridTailSlack * static_cast<double>(jmax) * free_groups /
                      static_cast<double>(chains) * (kFusedStepCycles / per_rec);
  return std::max<int64_t>(1, std::min<int64_t>(static_cast<int64_t>(tail), jmax - 1));
}

// A named NVTX range over the host calls that enqueue one launch, so that a timeline
// tool shows which kernel each launch API call belongs to.  Header-only NVTX: without
// a tool attached the push and pop cost a few nanoseconds.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

// Upper bound on the chunks of one sequence (the fused launch's chunk-major items).
int64_t max_chunks_per_seq(const kda_shape_t* s, bool fixed, bool ckpt) {
  int64_t L = fixed ? s->total_tokens / s->num_seqs
                    : (s->max_seqlen > 0 ? s->max_seqlen : s->total_tokens);
  return (L + kC - 1) / kC + (ckpt ? 1 : 0);
}

Resolved resolve(const kda_shape_t* s, bool fixed, bool ckpt, const kda_options_t* o) {
  Resolved r{};
  r.variant = choose_variant(s, o);
  r.fixed = fixed;
  // the token variant needs no per-record tiles; AUTO sizes for the largest variant
  // so that one workspace serves whatever the table picks
  const bool tiles = !(o && o->variant == KDA_VARIANT_TOKEN);
  r.lay = make_layout(s->num_seqs, s->total_tokens, s->num_heads, fixed, tiles, ckpt,
                      r.variant == KDA_VARIANT_STREAM);
  return r;
}

int sm_count() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

kda_status_t device_check() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KDA_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return KDA_ERR_UNSUPPORTED_DEVICE;
  if (major != 10 || minor != 0) return KDA_ERR_UNSUPPORTED_DEVICE;
  return KDA_OK;
}

bool make_map_2d(CUtensorMap* m, CUtensorMapDataType dt, void* base, uint64_t inner,
                 uint64_t rows, uint32_t box_inner, uint32_t box_rows, uint32_t elem_bytes) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return encode_fn()(m, dt, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_tokens(CUtensorMap* m, const void* base, uint64_t T, uint64_t H) {
  const cuuint64_t dims[3] = {128, H, T};
  const cuuint64_t strides[2] = {128 * 2, H * 128 * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Token rows of one head, whole: box (128 channels, 1 head, 64 tokens), no swizzle,
// so a chunk lands in shared memory as [64 tok][128 ch].
bool make_map_rows(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t T,
                   uint64_t H, uint32_t elem_bytes) {
  const cuuint64_t dims[3] = {128, H, T};
  const cuuint64_t strides[2] = {128ull * elem_bytes, H * 128ull * elem_bytes};
  const cuuint32_t box[3] = {128, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return encode_fn()(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" {

int kda_version(void) { return kVersion; }

const char* kda_status_string(int s) {
  switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_NULL_ARG: return "a required pointer is NULL";
    case KDA_ERR_BAD_SHAPE: return "invalid shape";
    case KDA_ERR_MISALIGNED: return "a pointer misses its required alignment";
    case KDA_ERR_UNPAIRED_CKPT: return "ckpt_state and ckpt_offsets must be given together";
    case KDA_ERR_PARTIAL_ALIAS: return "h0/ht/ckpt_state overlap without being identical";
    case KDA_ERR_OUT_ALIAS: return "an output overlaps an input or the workspace";
    case KDA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case KDA_ERR_UNSUPPORTED_DEVICE: return "current device is not compute capability 10.0";
    case KDA_ERR_LAUNCH_FAILED: return "kernel launch failed";
    case KDA_ERR_BAD_OPTION: return "unknown or unavailable option";
    case KDA_ERR_SCRATCH_UNAVAILABLE: return "the built-in scratch area could not be set up";
    case KDA_ERR_BAD_CU_SEQLENS: return "cu_seqlens invalid (validate mode)";
    case KDA_ERR_BAD_CKPT_OFFSET: return "checkpoint offset outside its sequence (validate mode)";
    case KDA_ERR_TIMEOUT: return "a bounded on-device wait timed out";
    case KDA_ERR_BAD_STATE_INDEX: return "a state index at or above the pool size";
    default: return "unknown status";
  }
}

size_t kda_prefill_workspace_size(const kda_shape_t* shape, int has_ckpt,
                                  const kda_options_t* options) {
  if (check_options(options) != KDA_OK) return 0;
  // the layout does not depend on whether cu_seqlens is given beyond the slot
  // bound; size for the larger (packed) bound so one workspace serves both.
  if (check_shape(shape, false, has_ckpt != 0) != KDA_OK) return 0;
  const Resolved r = resolve(shape, false, has_ckpt != 0, options);
  return r.lay.total;
}

kda_status_t kda_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace) return KDA_ERR_NULL_ARG;
  if (!aligned(workspace, 256)) return KDA_ERR_MISALIGNED;
  if (workspace_bytes < kHeaderBytes) return KDA_ERR_WORKSPACE_TOO_SMALL;
  if (cudaMemsetAsync(workspace, 0, kHeaderBytes, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return KDA_ERR_LAUNCH_FAILED;
  return KDA_OK;
}

kda_status_t kda_prefill_describe(const kda_shape_t* shape, int has_ckpt,
                                  const kda_options_t* options, char* buf, size_t n) {
  if (!buf || n == 0) return KDA_ERR_NULL_ARG;
  kda_status_t st = check_options(options);
  if (st == KDA_OK) st = check_shape(shape, false, has_ckpt != 0);
  if (st != KDA_OK) {
    snprintf(buf, n, "error: %s", kda_status_string(st));
    return st;
  }
  const Resolved r = resolve(shape, false, has_ckpt != 0, options);
  const long long chains = static_cast<long long>(shape->num_seqs) * shape->num_heads;
  if (r.variant == KDA_VARIANT_TOKEN) {
    const bool wide = token_wide(chains, 0);
    snprintf(buf, n,
             "variant=token grid=%lldx%d (%s: %d CTA(s) per (sequence, head), %d value columns "
             "each) workspace_bytes=%zu",
             chains * (wide ? 1 : 4), tok::kThreadsPerCta, wide ? "wide" : "narrow",
             wide ? 1 : 4, wide ? 128 : 32, r.lay.total);
  } else if (r.variant == KDA_VARIANT_HYBRID) {
    const int64_t jmax = max_chunks_per_seq(shape, false, has_ckpt != 0);
    const bool fe = options && options->frontend && options->frontend->flags;
    const int64_t tail = hybrid_tail_chunks(jmax, chains, fe);
    snprintf(buf, n,
             "variant=hybrid chunk=%d prepare_chunks=%lld/%lld (split prepare launch) then "
             "grid=%dx%d (recurrence CTAs %lld, prepare CTAs %lld, cooperative) workspace_bytes=%zu",
             kC, static_cast<long long>(jmax - tail), static_cast<long long>(jmax), sm_count(),
             fused::kThreadsPerCta, chains, static_cast<long long>(sm_count()) - chains,
             r.lay.total);
  } else if (r.variant == KDA_VARIANT_STREAM) {
    const long long grid = sm_count();
    snprintf(buf, n,
             "variant=stream chunk=%d grid=%lldx%d (recurrences %lld, prepare groups %lld, "
             "one CTA per SM, cooperative) workspace_bytes=%zu",
             kC, grid, stream::kThreadsPerCta, chains, 2 * grid - chains, r.lay.total);
  } else if (r.variant == KDA_VARIANT_FUSED) {
    snprintf(buf, n,
             "variant=fused chunk=%d grid=%dx%d (recurrence CTAs %lld, prepare CTAs %lld, "
             "cooperative) workspace_bytes=%zu",
             kC, sm_count(), fused::kThreadsPerCta, chains,
             static_cast<long long>(sm_count()) - chains, r.lay.total);
  } else {
    snprintf(buf, n,
             "variant=split chunk=%d prepare_items=%lldx%d (persistent, 2 CTAs/SM, 256 threads) "
             "recurrence_grid=%lldx%d "
             "workspace_bytes=%zu",
             kC, static_cast<long long>(r.lay.slots), shape->num_heads, chains,
             rec::kThreadsPerCta, r.lay.total);
  }
  return KDA_OK;
}

kda_status_t kda_prefill(const void* q, const void* k, const void* v, const float* g,
                         const void* beta, float scale, const float* h0,
                         const int32_t* cu_seqlens, const kda_shape_t* shape, void* out,
                         float* ht, float* ckpt_state, const int32_t* ckpt_offsets,
                         void* workspace, size_t workspace_bytes,
                         const kda_options_t* options, void* stream) {
  // ---------------- host-side validation (no CUDA call before it passes)
  kda_status_t st = check_options(options);
  if (st != KDA_OK) return st;
  const bool fixed = (cu_seqlens == nullptr);
  const bool cu64 = options && (options->flags & KDA_FLAG_CU_SEQLENS_I64);
  if (cu64 && fixed) return KDA_ERR_BAD_OPTION;   // the flag describes a cu_seqlens array
  const size_t cu_elem = cu64 ? 8 : 4;
  if (!shape) return KDA_ERR_NULL_ARG;
  st = check_shape(shape, fixed, ckpt_state != nullptr);
  if (st != KDA_OK) return st;
  const int64_t N = shape->num_seqs, T = shape->total_tokens, H = shape->num_heads;
  if (T > 0 && (!q || !k || !v || !g || !beta || !out)) return KDA_ERR_NULL_ARG;
  if (!workspace) return KDA_ERR_NULL_ARG;
  if ((ckpt_state == nullptr) != (ckpt_offsets == nullptr)) return KDA_ERR_UNPAIRED_CKPT;
  const kda_frontend_t* fe = options ? options->frontend : nullptr;
  st = check_frontend(fe);
  if (st != KDA_OK) return st;
  const bool fe_gate = fe && (fe->flags & KDA_FE_GATE);
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
      !aligned(out, 16) || !aligned(beta, 2) || !aligned(h0, 16) || !aligned(ht, 16) ||
      !aligned(ckpt_state, 16) || !aligned(cu_seqlens, cu_elem) || !aligned(ckpt_offsets, 4) ||
      !aligned(workspace, 256))
    return KDA_ERR_MISALIGNED;
  const size_t tok16 = static_cast<size_t>(T * H * 128 * 2);
  const size_t state = static_cast<size_t>(N * H * 128 * 128 * 4);
  const Range rq = rng(q, tok16), rk = rng(k, tok16), rv = rng(v, tok16),
              rg = rng(g, fe_gate ? tok16 : tok16 * 2), rb = rng(beta, static_cast<size_t>(T * H * 2)),
              rh0 = rng(h0, state), rht = rng(ht, state), rck = rng(ckpt_state, state),
              rcu = rng(cu_seqlens, static_cast<size_t>(N + 1) * cu_elem),
              rco = rng(ckpt_offsets, static_cast<size_t>(N * 4)),
              rws = rng(workspace, workspace_bytes), ro = rng(out, tok16),
              ra = rng(fe_gate ? fe->A_log : nullptr, static_cast<size_t>(H * 4)),
              rdt = rng(fe_gate ? fe->dt_bias : nullptr, static_cast<size_t>(H * 128 * 4));
  if (overlap(rh0, rht) && h0 != ht) return KDA_ERR_PARTIAL_ALIAS;
  if (overlap(rck, rh0) || overlap(rck, rht)) return KDA_ERR_PARTIAL_ALIAS;
  const Range inputs[] = {rq, rk, rv, rg, rb, rcu, rco, ra, rdt};
  for (const Range& in : inputs) {
    if (overlap(ro, in) || overlap(rht, in) || overlap(rck, in) || overlap(rws, in))
      return KDA_ERR_OUT_ALIAS;
  }
  if (overlap(ro, rh0) || overlap(ro, rht) || overlap(ro, rck) || overlap(ro, rws) ||
      overlap(rws, rh0) || overlap(rws, rht) || overlap(rws, rck))
    return KDA_ERR_OUT_ALIAS;
  const bool ckpt = ckpt_state != nullptr;
  const Resolved r = resolve(shape, fixed, ckpt, options);
  const size_t need = kda_prefill_workspace_size(shape, ckpt ? 1 : 0, options);
  if (workspace_bytes < need || workspace_bytes < r.lay.total) return KDA_ERR_WORKSPACE_TOO_SMALL;
  // the fused launch needs an SM per chain plus SMs for its prepare CTAs
  if ((r.variant == KDA_VARIANT_FUSED || r.variant == KDA_VARIANT_HYBRID) && !fused_eligible(shape))
    return KDA_ERR_BAD_OPTION;
  if (r.variant == KDA_VARIANT_STREAM && !stream_eligible(shape)) return KDA_ERR_BAD_OPTION;

  // ---------------- device
  st = device_check();
  if (st != KDA_OK) return st;
  if (encode_fn() == nullptr) return KDA_ERR_LAUNCH_FAILED;
  const uint32_t flags = options ? options->flags : 0u;

  KdaParams p{};
  p.q = static_cast<const uint16_t*>(q);
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.g = g;
  p.beta = static_cast<const uint16_t*>(beta);
  p.scale = scale;
  p.h0 = h0;
  p.cu_seqlens = cu_seqlens;
  p.cu_seqlens64 = nullptr;
  p.ckpt_offsets = ckpt_offsets;
  p.out = static_cast<uint16_t*>(out);
  p.ht = ht;
  p.ckpt = ckpt_state;
  p.N = static_cast<int32_t>(N);
  p.T = static_cast<int32_t>(T);
  p.H = static_cast<int32_t>(H);
  p.max_len = shape->max_seqlen;
  p.fixed_len = fixed ? static_cast<int32_t>(T / N) : 0;
  p.split_jmax = INT32_MAX;
  p.fused_j0 = 0;
  p.ws = static_cast<uint8_t*>(workspace);
  p.lay = r.lay;
  if (cu64) {
    // kernels read the INT32 copy the schedule kernel writes into the workspace
    p.cu_seqlens64 = reinterpret_cast<const int64_t*>(cu_seqlens);
    p.cu_seqlens = reinterpret_cast<const int32_t*>(p.ws + r.lay.cu32);
  }
  p.slots = r.lay.slots;
  p.flags = flags;
  p.wait_budget = (flags & KDA_FLAG_TEST_FORCE_TIMEOUT) ? -1 : kDefaultWaitBudget;
  p.fe_flags = fe_bits(fe);
  if (fe_gate) {
    p.A_log = fe->A_log;
    p.dt_bias = fe->dt_bias;
    p.lower_bound = fe->lower_bound;
  }
  if (fe && (fe->flags & KDA_FE_QK_L2NORM)) p.l2_eps = fe->l2_eps;

  // ---------------- tensor maps (encoded per call; passed by value)
  SplitMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  const uint64_t recs = static_cast<uint64_t>(r.lay.slots) * H;
  uint8_t* ws = p.ws;
  bool mok = true;
  if (T > 0) {
    mok &= make_map_tokens(&maps.v_in, v, T, H);
    mok &= make_map_rows(&maps.q_in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, q, T, H, 2);
    mok &= make_map_rows(&maps.k_in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, k, T, H, 2);
    if (fe_gate)   // the raw gate, BF16
      mok &= make_map_rows(&maps.g_in, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g, T, H, 2);
    else
      mok &= make_map_rows(&maps.g_in, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g, T, H, 4);
    mok &= make_map_rows(&maps.o_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, T, H, 2);
    if (r.variant == KDA_VARIANT_STREAM) {
      mok &= make_map_2d(&maps.qw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.qw, 128, recs * 128, 64, 128, 2);
      mok &= make_map_2d(&maps.u, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.u, 128, recs * 64, 64, 64, 2);
    } else {
      mok &= make_map_2d(&maps.wt, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.wt, 64, recs * 128, 64, 128, 2);
      mok &= make_map_2d(&maps.qg, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.qg, 128, recs * 64, 64, 64, 2);
      mok &= make_map_2d(&maps.ut, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.ut, 64, recs * 128, 64, 128, 2);
    }
    mok &= make_map_2d(&maps.kd, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.kd, 128, recs * 64, 64, 64, 2);
    mok &= make_map_2d(&maps.aqk, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, ws + r.lay.aqk, 64, recs * 64, 64, 64, 2);
  }
  if (!mok) return KDA_ERR_LAUNCH_FAILED;

  // ---------------- launches
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    cudaError_t e1 = cudaFuncSetAttribute(kda_prepare_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          prep::kSmemAllocBytes);
    cudaError_t e2 = cudaFuncSetAttribute(kda_recurrence_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          rec::kSmemAllocBytes);
    cudaError_t e3 = cudaFuncSetAttribute(kda_fused_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          fused::kSmemAllocBytes);
    cudaError_t e4 = cudaFuncSetAttribute(kda_prepare_fe_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          prep::kSmemAllocBytes);
    cudaError_t e5 = cudaFuncSetAttribute(kda_fused_fe_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          fused::kSmemAllocBytes);
    cudaError_t e6 = cudaFuncSetAttribute(kda_stream_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          stream::kSmemAllocBytes);
    cudaError_t e7 = cudaFuncSetAttribute(kda_stream_fe_kernel,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          stream::kSmemAllocBytes);
    // the stream CTA's two halves (about 223 KB) need the largest shared-memory carveout
    cudaError_t e8 = cudaFuncSetAttribute(kda_stream_kernel,
                                          cudaFuncAttributePreferredSharedMemoryCarveout,
                                          cudaSharedmemCarveoutMaxShared);
    cudaError_t e9 = cudaFuncSetAttribute(kda_stream_fe_kernel,
                                          cudaFuncAttributePreferredSharedMemoryCarveout,
                                          cudaSharedmemCarveoutMaxShared);
    const cudaError_t es[] = {e1, e2, e3, e4, e5, e6, e7, e8, e9};
    for (cudaError_t e : es)
      if (attr_err == cudaSuccess) attr_err = e;
  });
  if (attr_err != cudaSuccess) return KDA_ERR_LAUNCH_FAILED;
  (void)cudaGetLastError();
  void* const* ev = options ? options->events : nullptr;
  auto mark = [&](int i) {
    if (ev && ev[i]) cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  };
  // metadata kernel: INT64 narrowing, validation, and (chunked variants) the chunk table
  const bool sched = (r.variant == KDA_VARIANT_TOKEN)
                         ? (cu64 || (flags & KDA_FLAG_VALIDATE))
                         : (!fixed || ckpt || (flags & KDA_FLAG_VALIDATE));
  if (sched) {
    NvtxRange nr("kda_schedule");
    kda_schedule_kernel<<<1, 1024, 0, s>>>(p);
    mark(0);
  }
  if (r.variant == KDA_VARIANT_TOKEN) {
    NvtxRange nr("kda_token");
    mark(1);
    TokenParams tp{};
    tp.q = p.q;
    tp.k = p.k;
    tp.v = p.v;
    tp.g = p.g;
    tp.beta = p.beta;
    tp.scale = scale;
    tp.src = h0;
    tp.dst = ht;
    tp.cu_seqlens = p.cu_seqlens;
    tp.fixed_len = p.fixed_len;
    tp.ckpt_offsets = ckpt_offsets;
    tp.ckpt = ckpt_state;
    tp.out = p.out;
    tp.N = p.N;
    tp.T = p.T;
    tp.H = p.H;
    tp.ws = p.ws;
    tp.status = reinterpret_cast<int32_t*>(p.ws);
    tp.flags = flags;
    tp.wait_budget = p.wait_budget;
    tp.fe_flags = p.fe_flags;
    tp.A_log = p.A_log;
    tp.dt_bias = p.dt_bias;
    tp.lower_bound = p.lower_bound;
    tp.l2_eps = p.l2_eps;
    st = launch_token(tp, N * H, token_wide(N * H, 0), s);
    if (st != KDA_OK) return st;
    mark(2);
  } else if (r.variant == KDA_VARIANT_STREAM) {
    NvtxRange nr("kda_stream");
    mark(1);
    // one cooperative launch of two CTAs per SM: CTAs 0 .. N H - 1 run the recurrences,
    // the rest prepare the chunk records in chunk-major order
    void* fn = p.fe_flags ? reinterpret_cast<void*>(kda_stream_fe_kernel)
                          : reinterpret_cast<void*>(kda_stream_kernel);
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, stream::kThreadsPerCta,
                                                      stream::kSmemAllocBytes) != cudaSuccess ||
        per_sm < 1)
      return KDA_ERR_LAUNCH_FAILED;
    int32_t rec_ctas = static_cast<int32_t>(N * H);
    const int64_t grid = sm_count();
    if (rec_ctas > grid) return KDA_ERR_BAD_OPTION;
    const int64_t jmax = max_chunks_per_seq(shape, fixed, ckpt);
    int64_t prep_items = jmax * static_cast<int64_t>(rec_ctas);
    // ready flags and the item counter the prepare CTAs claim from, cleared every call
    if (r.lay.slots > 0 &&
        cudaMemsetAsync(ws + r.lay.ready, 0, r.lay.claim + 8 - r.lay.ready, s) != cudaSuccess)
      return KDA_ERR_LAUNCH_FAILED;
    p.claim_items = 1;
    void* args[] = {&p, &maps, &rec_ctas, &prep_items};
    if (cudaLaunchCooperativeKernel(fn, dim3(static_cast<unsigned>(grid)),
                                    dim3(stream::kThreadsPerCta), args, stream::kSmemAllocBytes,
                                    s) != cudaSuccess)
      return KDA_ERR_LAUNCH_FAILED;
    mark(2);
  } else if (r.variant == KDA_VARIANT_FUSED || r.variant == KDA_VARIANT_HYBRID) {
    const int64_t jmax = max_chunks_per_seq(shape, fixed, ckpt);
    int64_t j0 = 0;
    if (r.variant == KDA_VARIANT_HYBRID && T > 0) {
      NvtxRange nr("kda_prepare");
      // the prepare launch makes chunks [0, j0) of every sequence first
      j0 = jmax - hybrid_tail_chunks(jmax, N * H, p.fe_flags != 0);
      p.split_jmax = static_cast<int32_t>(j0);
      const int64_t items = r.lay.slots * H;
      const int64_t pgrid = std::min<int64_t>(items, 2 * static_cast<int64_t>(sm_count()));
      if (p.fe_flags)
        kda_prepare_fe_kernel<<<static_cast<unsigned>(pgrid), 256, prep::kSmemAllocBytes, s>>>(p, maps);
      else
        kda_prepare_kernel<<<static_cast<unsigned>(pgrid), 256, prep::kSmemAllocBytes, s>>>(p, maps);
      p.split_jmax = INT32_MAX;
    }
    p.fused_j0 = static_cast<int32_t>(j0);
    NvtxRange nr("kda_fused");
    mark(1);
    // one cooperative launch: CTAs 0 .. N H - 1 run the recurrences, the rest of
    // the SMs (one CTA each) prepare the chunk records in chunk-major order
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm,
                                                      p.fe_flags ? kda_fused_fe_kernel
                                                                 : kda_fused_kernel,
                                                      fused::kThreadsPerCta,
                                                      fused::kSmemAllocBytes) != cudaSuccess ||
        per_sm < 1)
      return KDA_ERR_LAUNCH_FAILED;
    int32_t rec_ctas = static_cast<int32_t>(N * H);
    const int grid = sm_count();   // one CTA per SM (checked above: chains + 16 <= SMs)
    int64_t prep_items = (jmax - j0) * static_cast<int64_t>(rec_ctas);
    if (r.lay.slots > 0 &&
        cudaMemsetAsync(ws + r.lay.ready, 0, static_cast<size_t>(r.lay.slots) * H * sizeof(int32_t),
                        s) != cudaSuccess)
      return KDA_ERR_LAUNCH_FAILED;
    int32_t prep_groups = rec_ctas <= kFusedOneGroupMaxChains ? 1 : 2;
    void* args[] = {&p, &maps, &rec_ctas, &prep_items, &prep_groups};
    void* fused_fn = p.fe_flags ? reinterpret_cast<void*>(kda_fused_fe_kernel)
                                : reinterpret_cast<void*>(kda_fused_kernel);
    if (cudaLaunchCooperativeKernel(fused_fn, dim3(grid),
                                    dim3(fused::kThreadsPerCta), args, fused::kSmemAllocBytes,
                                    s) != cudaSuccess)
      return KDA_ERR_LAUNCH_FAILED;
    mark(2);
  } else {
    if (T > 0) {
      NvtxRange nr("kda_prepare");
      // persistent prepare grid: two CTAs per SM walk the (chunk slot, head) items
      const int64_t items = r.lay.slots * H;
      const int64_t grid = std::min<int64_t>(items, 2 * static_cast<int64_t>(sm_count()));
      if (p.fe_flags)
        kda_prepare_fe_kernel<<<static_cast<unsigned>(grid), 256, prep::kSmemAllocBytes, s>>>(p, maps);
      else
        kda_prepare_kernel<<<static_cast<unsigned>(grid), 256, prep::kSmemAllocBytes, s>>>(p, maps);
    }
    mark(1);
    NvtxRange nr("kda_recurrence");
    kda_recurrence_kernel<<<static_cast<unsigned>(N * H), rec::kThreadsPerCta,
                            rec::kSmemAllocBytes, s>>>(p, maps);
    mark(2);
  }
  if (cudaGetLastError() != cudaSuccess) return KDA_ERR_LAUNCH_FAILED;
  return KDA_OK;
}

kda_status_t kda_decode(const void* q, const void* k, const void* v, const float* g,
                        const void* beta, float scale, float* state,
                        const int32_t* state_indices, const kda_decode_shape_t* shape,
                        void* out, float* step_states, int32_t* device_status, uint32_t flags,
                        const kda_frontend_t* frontend, void* stream) {
  if (!shape) return KDA_ERR_NULL_ARG;
  const uint32_t fe = frontend ? frontend->flags : 0u;
  {
    const kda_status_t fst = check_frontend(frontend);
    if (fst != KDA_OK && fst != KDA_ERR_MISALIGNED) return fst;   // alignment after NULL checks
  }
  if (flags & ~static_cast<uint32_t>(KDA_DECODE_KEEP_STATE | KDA_DECODE_NARROW |
                                     KDA_DECODE_WIDE))
    return KDA_ERR_BAD_OPTION;
  if ((flags & KDA_DECODE_NARROW) && (flags & KDA_DECODE_WIDE)) return KDA_ERR_BAD_OPTION;
  const int64_t N = shape->num_seqs, T = shape->tokens_per_seq, H = shape->num_heads,
                P = shape->pool_size;
  if (N < 1 || T < 1 || H < 1 || P < 1) return KDA_ERR_BAD_SHAPE;
  if (!state_indices && P < N) return KDA_ERR_BAD_SHAPE;
  // 32-bit token rows and grid
  if (N * T * H * 128 >= (int64_t(1) << 31) || N * H * 4 >= (int64_t(1) << 31))
    return KDA_ERR_BAD_SHAPE;
  if (!q || !k || !v || !g || !beta || !state || !out) return KDA_ERR_NULL_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
      !aligned(out, 16) || !aligned(beta, 2) || !aligned(state, 16) ||
      !aligned(step_states, 16) || !aligned(state_indices, 4) || !aligned(device_status, 4))
    return KDA_ERR_MISALIGNED;
  if (check_frontend(frontend) != KDA_OK) return KDA_ERR_MISALIGNED;
  const size_t tok16 = static_cast<size_t>(N * T * H * 128 * 2);
  const size_t g_bytes = (fe & KDA_FE_GATE) ? tok16 : tok16 * 2;   // raw BF16 gate or FP32 g
  const size_t st1 = static_cast<size_t>(H * 128 * 128 * 4);   // one slot, all heads
  const Range rq = rng(q, tok16), rk = rng(k, tok16), rv = rng(v, tok16),
              rg = rng(g, g_bytes), rb = rng(beta, static_cast<size_t>(N * T * H * 2)),
              ri = rng(state_indices, static_cast<size_t>(N * 4)),
              rs = rng(state, st1 * static_cast<size_t>(P)), ro = rng(out, tok16),
              rst = rng(step_states, st1 * static_cast<size_t>(N * T)),
              rds = rng(device_status, 4);
  const bool gate = (fe & KDA_FE_GATE) != 0;
  const Range ra = rng(gate ? frontend->A_log : nullptr, static_cast<size_t>(H * 4)),
              rdt = rng(gate ? frontend->dt_bias : nullptr, static_cast<size_t>(H * 128 * 4));
  const Range inputs[] = {rq, rk, rv, rg, rb, ri, ra, rdt};
  const Range outputs[] = {rs, ro, rst, rds};
  for (const Range& o : outputs)
    for (const Range& in : inputs)
      if (overlap(o, in)) return KDA_ERR_OUT_ALIAS;
  for (int i = 0; i < 4; ++i)
    for (int j = i + 1; j < 4; ++j)
      if (overlap(outputs[i], outputs[j])) return KDA_ERR_OUT_ALIAS;
  kda_status_t st = device_check();
  if (st != KDA_OK) return st;

  TokenParams tp{};
  tp.q = static_cast<const uint16_t*>(q);
  tp.k = static_cast<const uint16_t*>(k);
  tp.v = static_cast<const uint16_t*>(v);
  tp.g = g;
  tp.beta = static_cast<const uint16_t*>(beta);
  tp.scale = scale;
  tp.src = state;
  tp.dst = (flags & KDA_DECODE_KEEP_STATE) ? nullptr : state;
  tp.slot = state_indices;
  tp.pool = static_cast<int32_t>(P);
  tp.cu_seqlens = nullptr;
  tp.fixed_len = static_cast<int32_t>(T);
  tp.steps = step_states;
  tp.out = static_cast<uint16_t*>(out);
  tp.N = static_cast<int32_t>(N);
  tp.T = static_cast<int32_t>(N * T);
  tp.H = static_cast<int32_t>(H);
  tp.status = device_status;
  tp.flags = 0;
  tp.wait_budget = kDefaultWaitBudget;
  tp.fe_flags = fe_bits(frontend);
  if (gate) {
    tp.A_log = frontend->A_log;
    tp.dt_bias = frontend->dt_bias;
    tp.lower_bound = frontend->lower_bound;
  }
  if (fe & KDA_FE_QK_L2NORM) tp.l2_eps = frontend->l2_eps;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  (void)cudaGetLastError();
  NvtxRange nr("kda_decode");
  st = launch_token(tp, N * H, token_wide(N * H, flags), s);
  if (st != KDA_OK) return st;
  if (cudaGetLastError() != cudaSuccess) return KDA_ERR_LAUNCH_FAILED;
  return KDA_OK;
}

kda_status_t kda_prefill_status(void* workspace, void* stream, int32_t* device_status,
                                 int clear) {
  if (!workspace || !device_status) return KDA_ERR_NULL_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t val = 0;
  if (cudaMemcpyAsync(&val, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return KDA_ERR_LAUNCH_FAILED;
  if (clear && cudaMemsetAsync(workspace, 0, sizeof(int32_t), s) != cudaSuccess)
    return KDA_ERR_LAUNCH_FAILED;
  if (cudaStreamSynchronize(s) != cudaSuccess) return KDA_ERR_LAUNCH_FAILED;
  *device_status = val;
  return KDA_OK;
}

}  // extern "C"
