/*
 * kda_prefill.h — C ABI of the B200 (sm_100a) KDA multi-token recurrent prefill.
 *
 * Kimi Delta Attention (KDA) is a gated delta rule with one decay per key
 * channel.  Per (sequence n, head h) a K x V = 128 x 128 FP32 state S is carried
 * through the tokens of the sequence:
 *
 *     S   <- Diag(exp(g_t)) S
 *     S   <- S + beta_t k_t (v_t - S^T k_t)^T      (S^T k_t taken after the decay)
 *     o_t  = scale * S^T q_t                       (S after token t's update)
 *
 * Interface facts taken from the pages that describe this operation:
 *   - K = V = 128, BF16 q/k/v/beta, FP32 recurrent state, gate bound in
 *     [-5, 0]: lmdeploy PR #5050 "Motivation" (native path requirements);
 *     FlashInfer PR #4262 "Dispatch contract".
 *   - ragged batches packed with B = 1 plus cu_seqlens: FlashInfer PR #4262
 *     "Dispatch contract"; FlashKDA item page "What Sets It Apart".
 *   - initial state, final state updated in place when the two pointers are
 *     the same allocation, partial overlap rejected: FlashInfer PR #4262
 *     "Physical schedules and true in-place state update".
 *   - checkpoint export of the state at a caller offset into caller-owned
 *     contiguous buffers, the two checkpoint arguments paired, offset values
 *     the caller's responsibility (no device-to-host read): lmdeploy PR #5050
 *     "Motivation" and "Scope".
 *   - caller-owned workspace, CUDA-graph-capturable calls once warm:
 *     FlashInfer PR #4633 "Description"; FlashInfer PR #4262 "CUDA graph and
 *     tensor-map safety".
 *   - 16-byte base alignment for TMA operands: FlashInfer PR #4633 "Reviewer
 *     Notes".
 *
 * General rules for every entry point below
 *   - All tensor pointers are DEVICE pointers on the current CUDA device, owned
 *     by the caller; the library never allocates, frees or keeps them.
 *   - `stream` is a cudaStream_t (passed as void*; NULL = legacy default stream).
 *     All device work is enqueued on it; no call synchronizes the host except
 *     kda_prefill_status.
 *   - Host-side validation happens before any launch and before any write to a
 *     caller buffer; on an error code nothing has been enqueued.
 *   - The library never reads cu_seqlens or ckpt_offsets on the host.  Their
 *     values are the caller's responsibility; with KDA_FLAG_VALIDATE the
 *     kernels check them and record KDA_ERR_BAD_CU_SEQLENS /
 *     KDA_ERR_BAD_CKPT_OFFSET in the workspace status word (see
 *     kda_prefill_status) instead of computing.
 */
#ifndef KDA_PREFILL_H_
#define KDA_PREFILL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KDA_HEAD_DIM 128 /* K = V = 128, the only head size */

typedef enum {
  KDA_OK = 0,
  KDA_ERR_NULL_ARG = 1,            /* a required pointer is NULL                    */
  KDA_ERR_BAD_SHAPE = 2,           /* N < 1, H < 1, T < 0, max_seqlen out of range,
                                      fixed layout with T not divisible by N        */
  KDA_ERR_MISALIGNED = 3,          /* a pointer misses its required alignment        */
  KDA_ERR_UNPAIRED_CKPT = 4,       /* exactly one of ckpt_state / ckpt_offsets given */
  KDA_ERR_PARTIAL_ALIAS = 5,       /* h0 and ht overlap without being identical, or
                                      ckpt_state overlaps h0 / ht                   */
  KDA_ERR_OUT_ALIAS = 6,           /* an output overlaps an input or the workspace   */
  KDA_ERR_WORKSPACE_TOO_SMALL = 7, /* workspace_bytes < kda_prefill_workspace_size   */
  KDA_ERR_UNSUPPORTED_DEVICE = 8,  /* current device is not compute capability 10.0  */
  KDA_ERR_LAUNCH_FAILED = 9,       /* the CUDA runtime refused a launch              */
  KDA_ERR_BAD_OPTION = 10,         /* unknown variant / chunk / flag value           */
  KDA_ERR_SCRATCH_UNAVAILABLE = 11,/* kda_prefill_noalloc: the built-in scratch area
                                      could not be set up on this device (e.g. out of
                                      memory when the library's device code loads)  */
  /* codes the kernels record in the workspace status word */
  KDA_ERR_BAD_CU_SEQLENS = 16,     /* cu_seqlens[0] != 0, decreasing, or last != T,
                                      or a length above max_seqlen (validate mode)   */
  KDA_ERR_BAD_CKPT_OFFSET = 17,    /* an offset outside [0, len] (validate mode)     */
  KDA_ERR_TIMEOUT = 18,            /* a bounded on-chip wait gave up (the kernel
                                      returned without finishing its work)          */
  KDA_ERR_BAD_STATE_INDEX = 19     /* kda_decode: a state index >= pool_size          */
} kda_status_t;

/* Sizes known on the host.  No device memory is read to obtain them. */
typedef struct {
  int32_t num_seqs;     /* N >= 1: sequences (fixed layout: the batch B)              */
  int32_t total_tokens; /* T_total >= 0: rows of q/k/v/g/beta/out                     */
  int32_t num_heads;    /* H >= 1                                                      */
  int32_t max_seqlen;   /* an upper bound on every sequence length; 0 = use T_total    */
} kda_shape_t;

typedef enum {
  KDA_VARIANT_AUTO = 0,  /* per-shape choice from the measured table                   */
  KDA_VARIANT_SPLIT = 1, /* prepare kernel over all chunks, then the recurrence kernel */
  KDA_VARIANT_FUSED = 2, /* one cooperative launch: one recurrence CTA per (sequence,
                            head) on its own SM, the other SMs prepare the chunk records
                            and hand each one over through a ready flag in the workspace.
                            Needs N*H + 16 <= SM count, else KDA_ERR_BAD_OPTION.  AUTO
                            picks it for at most 56 chains of at least 32 chunks.      */
  KDA_VARIANT_HYBRID = 3, /* the prepare launch for the first chunks of every sequence, then
                            the fused launch, whose prepare CTAs make the last chunks while
                            its recurrence CTAs already run.  Same SM condition as FUSED;
                            AUTO picks it above 56 chains of at least 64 chunks.          */
  KDA_VARIANT_TOKEN = 4,  /* the recurrence one token at a time with the state in
                            registers: 4 CTAs of 32 value columns per (sequence, head)
                            below 128 units, one CTA of 128 columns per unit from 128 on;
                            no chunk records, workspace = header only.  AUTO picks it when
                            max_seqlen (else T_total) is at most 16, or at most 32 with
                            N*H <= 16.                                                   */
  KDA_VARIANT_STREAM = 5  /* one cooperative launch of one 512-thread CTA per SM: on CTA
                            b < N*H one half carries the recurrence of (sequence, head) b
                            (state with the key channel on the tensor-memory lanes) and the
                            other half a prepare group; the other CTAs run two prepare
                            groups, so prepare work runs on every SM beside the
                            recurrences; records reach the recurrence through L2 and are
                            dropped from it once read.  Needs N*H <= SM count, else
                            KDA_ERR_BAD_OPTION.  Opt-in only: AUTO does not pick it (it
                            moves the fewest DRAM bytes but was slower than the others
                            on every measured shape).                                     */
} kda_variant_t;

enum {
  KDA_FLAG_VALIDATE = 1u << 0,       /* kernels check cu_seqlens / ckpt_offsets values  */
  KDA_FLAG_CU_SEQLENS_I64 = 1u << 2, /* cu_seqlens holds INT64 entries (8-byte aligned);
                                        the metadata kernel converts them on the device  */
  KDA_FLAG_TEST_FORCE_TIMEOUT = 1u << 1 /* test hook: every bounded wait gives up at once;
                                          exercises the error path, never for production */
};

/*
 * Optional input front end (kda_options_t.frontend for kda_prefill, the
 * `frontend` argument of kda_decode): the kernels form the recurrence inputs from
 * raw projections, in FP32, so that no rounded intermediate reaches the state
 * (a BF16 copy of the normalised k or of beta would move it by about 2e-3).  The parameter set (A_log per head, dt_bias per head and key channel, a
 * finite negative lower bound, q/k L2 normalisation, beta given as a logit) is
 * FlashInfer PR #4262's "Dispatch contract"; the pages print no formula, and the
 * one below is this library's reading (it puts every log-decay in
 * (lower_bound, 0)):
 *   KDA_FE_QK_L2NORM   q, k <- x / sqrt(sum_c x_c^2 + l2_eps) per (token, head)
 *   KDA_FE_GATE        `g` holds the raw gate a as BF16, same layout as q (16-byte
 *                      aligned); g_c = lower_bound * sigmoid(exp(A_log[h]) *
 *                      (a_c + dt_bias[h][c])), sigmoid(x) = 1 / (1 + exp(-x))
 *   KDA_FE_BETA_LOGIT  `beta` holds logits; beta <- sigmoid(beta)
 * A_log [H] FP32 (4-byte aligned) and dt_bias [H, 128] FP32 (16-byte aligned) are
 * device arrays, read only with KDA_FE_GATE.  lower_bound must lie in [-5, 0)
 * (the gate bound of lmdeploy PR #5050 "Motivation"), l2_eps in [0, 1]; otherwise
 * KDA_ERR_BAD_OPTION.
 */
enum {
  KDA_FE_QK_L2NORM = 1u << 0,
  KDA_FE_GATE = 1u << 1,
  KDA_FE_BETA_LOGIT = 1u << 2
};
typedef struct {
  uint32_t flags;        /* KDA_FE_*                                            */
  float lower_bound;     /* KDA_FE_GATE                                         */
  float l2_eps;          /* KDA_FE_QK_L2NORM                                    */
  const float* A_log;    /* KDA_FE_GATE: [H]                                    */
  const float* dt_bias;  /* KDA_FE_GATE: [H, 128]                               */
} kda_frontend_t;

typedef struct {
  int32_t variant;  /* kda_variant_t                                               */
  uint32_t flags;   /* KDA_FLAG_*                                                   */
  /* Optional profiling hook: cudaEvent_t handles (created by the caller) that
     kda_prefill records on `stream` right after its launches: [0] after the
     metadata kernel (when one is launched), [1] after the prepare kernel, [2]
     after the last kernel of the call.  NULL entries are skipped.  The events
     let a caller time each kernel on the launching stream. */
  void* events[3];
  /* NULL, or the input front end (kda_frontend_t above): q, k, g (and beta) then hold
     raw projections.  Every variant takes all three switches (the chunked variants
     keep T diag(beta) as an FP16 tensor-core operand, so a beta squashed in FP32
     keeps 2^-11 relative precision on its diagonal). */
  const kda_frontend_t* frontend;
  int32_t reserved[2];
} kda_options_t;

/*
 * Bytes of workspace kda_prefill needs for this shape and option set (NULL
 * options = defaults).  `has_ckpt` != 0 when checkpoint export is requested.
 * Returns 0 for an invalid shape or option set.  The workspace must be 256-byte
 * aligned and, before its first use, initialised once with kda_workspace_init.
 *
 * Source: the pages' prefill backends take their scratch from one caller-owned
 * workspace so that a warmed call allocates nothing and can be captured in a CUDA
 * graph (FlashInfer PR #4633 "Description": decomp's two launches share one scratch
 * arena, and graph capture goes through a caller-owned workspace; FlashInfer PR
 * #4262 "CUDA graph and tensor-map safety").  The size is a pure function of the
 * host-side shape, so it can be queried before any device work.  The layout in it
 * (per-chunk records, chunk table, status word) is this library's own.
 */
size_t kda_prefill_workspace_size(const kda_shape_t* shape, int has_ckpt,
                                  const kda_options_t* options);

/*
 * Initialise a workspace (clears its status word).  Enqueued on `stream`.
 * Needed once per workspace allocation, before the first kda_prefill with it.
 * Source: this library's design (the status word below); the pages' workspaces
 * are warmed eagerly before capture (FlashInfer PR #4262 "CUDA graph and
 * tensor-map safety"), and this is the equivalent one-time step here.
 */
kda_status_t kda_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * Multi-token recurrent prefill (one launch sequence on `stream`).
 *
 *   q, k      [T_total, H, 128] BF16, contiguous, 16-byte aligned.  Rows of all
 *             sequences packed back to back (fixed layout [B, T, H, 128] is the
 *             same memory).  k is expected to be L2-normalised per row: the
 *             FP16 tensor-core operands (the state read, v, W, U) assume |S| and
 *             |v| well inside 65504.
 *   v         [T_total, H, 128] BF16, contiguous, 16-byte aligned.
 *   g         [T_total, H, 128] FP32 log-decay per key channel, contiguous,
 *             16-byte aligned; expected in [-5, 0] (outside it the chunked
 *             factorisation may overflow FP32; values are not checked).
 *   beta      [T_total, H] BF16, contiguous, 2-byte aligned (read with plain loads).
 *   scale     output scale (e.g. 1/sqrt(128)).
 *   h0        [N, H, 128, 128] FP32 initial state S[k][v] (row index = key
 *             channel), contiguous, 16-byte aligned; NULL = zero state.
 *   cu_seqlens [N+1] INT32 device array of sequence starts (4-byte aligned), or
 *             NULL for the fixed layout (N sequences of T_total / N tokens each).
 *             With KDA_FLAG_CU_SEQLENS_I64 the array holds INT64 entries (pass its
 *             address cast to const int32_t*; 8-byte aligned): a device kernel
 *             checks and narrows it into the workspace, the host never reads it.
 *   shape     host struct, see kda_shape_t.
 *   out       [T_total, H, 128] BF16 output o (round-to-nearest-even from FP32).
 *   ht        [N, H, 128, 128] FP32 final state, or NULL.  May be exactly h0
 *             (same pointer): the state is then updated in place.
 *   ckpt_state [N, H, 128, 128] FP32 checkpoint states, or NULL.
 *   ckpt_offsets [N] INT32 device array, or NULL; must be given together with
 *             ckpt_state.  Offset p_n is a prefix length of sequence n,
 *             0 <= p_n <= len_n: p = 0 exports h0, p = len the final state.
 *   workspace, workspace_bytes  caller-owned scratch (see above).
 *   options   NULL = defaults (auto variant, no flags).
 *   stream    cudaStream_t.
 *
 * Returns KDA_OK when the work was enqueued; errors see kda_status_t.  A zero-
 * length sequence leaves ht = h0 (also when h0 and ht alias).
 */
kda_status_t kda_prefill(const void* q, const void* k, const void* v, const float* g,
                         const void* beta, float scale, const float* h0,
                         const int32_t* cu_seqlens, const kda_shape_t* shape, void* out,
                         float* ht, float* ckpt_state, const int32_t* ckpt_offsets,
                         void* workspace, size_t workspace_bytes,
                         const kda_options_t* options, void* stream);

/*
 * Read (and clear when `clear` != 0) the status word the kernels of earlier
 * kda_prefill calls recorded in `workspace`.  Synchronises `stream`.  The word
 * keeps the first device-side error since the last clear (KDA_OK if none).
 * Source: this library's design, with no counterpart passage on the pages.  The
 * pages never read device metadata on the host (lmdeploy PR #5050 "Motivation":
 * offset values are the caller's responsibility, no device-to-host copy on the hot
 * path), so errors found on the device (validate mode, a bounded wait that gave
 * up) are recorded here and read only when the caller asks.
 */
kda_status_t kda_prefill_status(void* workspace, void* stream, int32_t* device_status,
                                 int clear);

/* Static description of a status code (never NULL).  Source: this library's
   design (the codes above); no counterpart passage on the pages. */
const char* kda_status_string(int status);

/*
 * Write a one-line description of what kda_prefill would launch for this
 * shape (variant, chunk size, grids, workspace bytes) into buf (NUL-
 * terminated, truncated to n bytes).  Host only.
 * Source: FlashInfer PR #4633 "Description" picks decomp or fused per call from a
 * measured table keyed on the SM count and offers describe_variant_policy to report
 * the policy a device gets; this call is that report for one shape.
 */
kda_status_t kda_prefill_describe(const kda_shape_t* shape, int has_ckpt,
                                  const kda_options_t* options, char* buf, size_t n);

/*
 * Prefill without any device allocation by the caller.  (Not an operation of
 * the method itself: the pages have no counterpart; it is an interface for
 * callers that cannot allocate.)
 *
 * For callers that cannot call cudaMalloc — code running while a CUDA graph is
 * captured into a memory pool it does not own, plugins whose host application
 * owns every device allocation, or real-time paths where an allocation and the
 * synchronisation it may cause are not allowed — and so cannot provide the
 * workspace kda_prefill needs.  This entry point uses a scratch area built into
 * the library instead: a static device array of KDA_NOALLOC_SCRATCH_BYTES that
 * every GPU which loads the library holds until the process exits.  The caller
 * still passes all inputs and outputs (same meaning, layout and rules as for
 * kda_prefill); the library calls no cudaMalloc/cudaFree or allocating routine.
 *
 *   - Shapes whose kda_prefill_workspace_size exceeds KDA_NOALLOC_SCRATCH_BYTES
 *     are refused with KDA_ERR_WORKSPACE_TOO_SMALL before anything is enqueued
 *     (48 MiB covers, e.g., 12 heads x 2048 tokens, or 8 x 1024 tokens at H = 4).
 *   - Every call looks up the area's device address (cudaGetSymbolAddress) with
 *     the current device.  With lazy module loading (the CUDA default) the first
 *     call on a device may load the library's device code and create the area
 *     there; if that fails (out of memory) the call returns
 *     KDA_ERR_SCRATCH_UNAVAILABLE and enqueues nothing.  Make that first call
 *     outside any stream capture.
 *   - All calls on a device share the one area: calls that may overlap on the
 *     GPU (different streams without ordering between them) race and must not
 *     be issued.  Calls ordered on one stream are fine; nothing in the area has
 *     to be cleared between calls.
 *   - The device status word lives in the built-in area and is not readable
 *     through this entry point, so KDA_FLAG_VALIDATE and
 *     KDA_FLAG_TEST_FORCE_TIMEOUT are refused (KDA_ERR_BAD_OPTION), and a bounded
 *     wait that gives up on the device cannot be seen here: use kda_prefill with
 *     your own workspace when validate mode or status reporting is needed.
 *   - Checks run in this order: options and shape (their kda_prefill codes), the
 *     device (KDA_ERR_UNSUPPORTED_DEVICE), the area's size
 *     (KDA_ERR_WORKSPACE_TOO_SMALL), then kda_prefill's own checks.
 */
#define KDA_NOALLOC_SCRATCH_BYTES ((size_t)48 << 20)
kda_status_t kda_prefill_noalloc(const void* q, const void* k, const void* v, const float* g,
                                 const void* beta, float scale, const float* h0,
                                 const int32_t* cu_seqlens, const kda_shape_t* shape,
                                 void* out, float* ht, float* ckpt_state,
                                 const int32_t* ckpt_offsets, const kda_options_t* options,
                                 void* stream);

/*
 * Decode and draft verification over a pool of states (one launch on `stream`).
 *
 * The same recurrence as kda_prefill, for N sequences of exactly T new tokens
 * each (T = 1: decode of one token; T = 1 + d: verification of d draft tokens),
 * each continuing from a state held in a caller-owned pool.  Serving engines keep
 * the per-(sequence, head) recurrent states of many requests in one pool and pass
 * the slot of every request (SGLang kda_flashinfer.py "FlashInferKDAKernel":
 * decode and target-verify over a state pool with per-request state indices).
 * The pages define no separate verify arithmetic; here verification is the plain
 * recurrence over the T tokens with the state after every token exported, so
 * that the caller can keep the state of the accepted prefix.
 *
 *   q, k, v   [N, T, H, 128] BF16, contiguous, 16-byte aligned.
 *   g         [N, T, H, 128] FP32 log-decay, contiguous, 16-byte aligned.
 *   beta      [N, T, H] BF16, 2-byte aligned.
 *   scale     output scale.
 *   state     [P, H, 128, 128] FP32 pool, S[k][v] per (slot, head), 16-byte
 *             aligned.  Slot i of sequence n is read before its first token and,
 *             unless KDA_DECODE_KEEP_STATE, overwritten with the state after its
 *             last token (in place).
 *   state_indices [N] INT32 device array, 4-byte aligned, or NULL (sequence n uses
 *             slot n; then P >= N).  A negative entry marks a padding row: its
 *             slot is neither read nor written and its out rows are set to zero.
 *             An entry >= P is handled like a padding row and recorded as
 *             KDA_ERR_BAD_STATE_INDEX in *device_status.  Two sequences sharing a
 *             slot race (undefined result).  Values are never read on the host.
 *   shape     host struct, see kda_decode_shape_t.
 *   out       [N, T, H, 128] BF16 output o.
 *   step_states [N, T, H, 128, 128] FP32, 16-byte aligned, or NULL: the state
 *             after each token (step_states[n][t] = state after token t).
 *   device_status  INT32 device word, 4-byte aligned, or NULL: the first device
 *             error is stored there with atomicCAS from KDA_OK (the caller clears
 *             it); without it device errors are not reported.
 *   frontend  NULL, or the input front end (kda_frontend_t above): q, k, g and beta
 *             then hold raw projections that the kernel turns into the recurrence
 *             inputs.
 *   flags     KDA_DECODE_KEEP_STATE: the pool is read only.  KDA_DECODE_NARROW /
 *             KDA_DECODE_WIDE force the kernel shape (timing aid; the default
 *             picks by the number of (sequence, head) units).
 *   stream    cudaStream_t.
 *
 * Outputs (state, out, step_states, device_status) must not overlap the inputs
 * or each other (KDA_ERR_OUT_ALIAS).  Returns KDA_OK when the launch was
 * enqueued.  No workspace and no allocation; CUDA-graph capturable.
 */

typedef struct {
  int32_t num_seqs;       /* N >= 1                                               */
  int32_t tokens_per_seq; /* T >= 1 new tokens of every sequence                  */
  int32_t num_heads;      /* H >= 1                                               */
  int32_t pool_size;      /* P >= 1 state slots in `state`                        */
} kda_decode_shape_t;

enum {
  KDA_DECODE_KEEP_STATE = 1u << 0, /* the pool is read only                              */
  KDA_DECODE_NARROW = 1u << 1,     /* force 4 CTAs of 32 value columns per (sequence,
                                      head) (default below 128 units)                   */
  KDA_DECODE_WIDE = 1u << 2        /* force 1 CTA of 128 value columns per unit (default
                                      from 128 units); not together with NARROW         */
};

kda_status_t kda_decode(const void* q, const void* k, const void* v, const float* g,
                        const void* beta, float scale, float* state,
                        const int32_t* state_indices, const kda_decode_shape_t* shape,
                        void* out, float* step_states, int32_t* device_status, uint32_t flags,
                        const kda_frontend_t* frontend, void* stream);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH.  Source: this library's
   design; no counterpart passage on the pages. */
int kda_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KDA_PREFILL_H_ */
