// kda_common.cuh — shapes, workspace layout and launch parameters shared by the
// KDA prefill kernels and their host launcher.
//
// Chunked form used by every kernel (one (sequence, head), chunk of C = 64
// tokens, local r = 0..63, G_r = running sum of g within the chunk, Gamma_r =
// exp(G_r), beta folded into the triangular factor):
//   A[r,s]   = sum_k k_r[k] k_s[k] exp(G_r[k] - G_s[k])          (s < r)
//   T        = (I + diag(beta) A)^-1,   Tb = T diag(beta)
//   W        = Tb (K * Gamma),            U = Tb V
//   Aqk[r,s] = sum_k q_r[k] k_s[k] exp(G_r[k] - G_s[k])          (s <= r)
//   Ud       = U - W S0
//   O        = scale [ (Q * Gamma) S0 + Aqk Ud ]
//   S1       = Diag(Gamma_63) S0 + (K * exp(G_63 - G))^T Ud
// The split of this factorisation into a prepare launch and a recurrence launch
// is the two-launch design FlashInfer PR #4633 calls decomp ("Description");
// the algebra itself is derived here from the per-token recurrence.  exp(G_r - G_s) is formed from 16-token sub-blocks so that no FP32
// factor leaves [e^-80, e^80] when every g lies in [-5, 0] (the gate bound of
// lmdeploy PR #5050 "Motivation").
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>

namespace kda {

constexpr int kD = 128;        // K = V = 128
constexpr int kC = 64;         // chunk length
constexpr int kSB = 16;        // sub-block length for the decay factorisation
constexpr float kLog2e = 1.4426950408889634f;

// ---- workspace layout --------------------------------------------------------
// header (status word, per-call validity) | chunk table | per-record tiles.
// A "record" is one (chunk slot, head) pair: rec = slot * H + h.
constexpr size_t kHeaderBytes = 1024;
constexpr size_t kTileWT = 128 * 64 * 2;   // W^T   [128 k][64 tok] f16
constexpr size_t kTileQG = 64 * 128 * 2;   // Q*Gamma [64 tok][128 k] f16 (token rows)
constexpr size_t kTileUT = 128 * 64 * 2;   // U^T   [128 v][64 tok] f16
constexpr size_t kTileKd = 64 * 128 * 2;   // Kd    [64 tok][128 k] f16 (token rows)
constexpr size_t kTileAqk = 64 * 64 * 2;   // Aqk   [64 r][64 s]  f16
constexpr size_t kTileGC = 128 * 4;        // Gamma at the chunk end, f32 [128]
// records of the stream variant (same bytes per record, token-row orientation)
constexpr size_t kTileQW = 128 * 128 * 2;  // [Q*Gamma; W] [128 rows][128 k] f16 (rows 0..63 Q Gamma)
constexpr size_t kTileU = 64 * 128 * 2;    // U [64 tok][128 v] f16

struct WorkspaceLayout {
  size_t cu32;         // int32 [N+1]   narrowed copy of INT64 cu_seqlens
  size_t chunk_base;   // int32 [N+1]   first slot of each sequence
  size_t seq_order;    // int32 [N]     longest-first order of sequences
  size_t slot_span;    // int2 [slots]  chunk slot -> {first token, count | chunk index << 7}
  size_t wt, qg, ut, kd, aqk, gc;     // per-record tiles
  size_t qw, u;                       // per-record tiles of the stream variant
  size_t ready;        // int32 [recs]  per-record ready flags (fused variant)
  size_t claim;        // u64           next item to claim (stream variant); cleared with the flags
  size_t total;
  int64_t slots;       // chunk slots (upper bound on the number of chunks)
};

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Number of chunk slots that always suffices.  A sequence of length L is cut into
// ceil(L / C) chunks; a checkpoint offset p (0 < p < L) adds one chunk boundary
// at p, so sum_n chunks_n <= T / C + 2 N.  The fixed layout without checkpoints
// is exactly N ceil(L / C).
__host__ __device__ inline int64_t chunk_slots(int64_t N, int64_t T, bool fixed, bool ckpt) {
  if (fixed && !ckpt) return N * ((T / N + kC - 1) / kC);
  return T / kC + (ckpt ? 2 : 1) * N;
}

inline WorkspaceLayout make_layout(int64_t N, int64_t T, int64_t H, bool fixed, bool split,
                                   bool ckpt, bool stream = false) {
  WorkspaceLayout L{};
  size_t off = kHeaderBytes;
  L.cu32 = off;
  off = align_up(off + sizeof(int32_t) * (N + 1), 256);
  L.chunk_base = off;
  off = align_up(off + sizeof(int32_t) * (N + 1), 256);
  L.seq_order = off;
  off = align_up(off + sizeof(int32_t) * N, 256);
  L.slots = (N > 0 && T > 0) ? chunk_slots(N, T, fixed, ckpt) : 0;
  L.slot_span = off;
  off = align_up(off + 2 * sizeof(int32_t) * static_cast<size_t>(L.slots), 1024);
  const size_t recs = split ? static_cast<size_t>(L.slots * H) : 0;
  if (stream) {   // [Q Gamma; W] and U replace W^T, Q Gamma and U^T (same bytes)
    L.qw = off;  off = align_up(off + recs * kTileQW, 1024);
    L.u = off;   off = align_up(off + recs * kTileU, 1024);
  } else {
    L.wt = off;  off = align_up(off + recs * kTileWT, 1024);
    L.qg = off;  off = align_up(off + recs * kTileQG, 1024);
    L.ut = off;  off = align_up(off + recs * kTileUT, 1024);
  }
  L.kd = off;  off = align_up(off + recs * kTileKd, 1024);
  L.aqk = off; off = align_up(off + recs * kTileAqk, 1024);
  L.gc = off;  off = align_up(off + recs * kTileGC, 1024);
  L.ready = off; off += recs * sizeof(int32_t);
  L.claim = align_up(off, 8); off = align_up(L.claim + 8, 1024);
  L.total = off;
  return L;
}

// Status words at the start of the workspace header.
struct WsHeader {
  int32_t status;    // first device error since the last clear (sticky)
  int32_t call_ok;   // 1 when the schedule kernel of this call found valid metadata
  int32_t pad[254];
};

// ---- kernel parameters ----------------------------------------------------------
struct KdaParams {
  // inputs
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const float* g;
  const uint16_t* beta;
  float scale;
  const float* h0;
  const int32_t* cu_seqlens;     // NULL: fixed layout (an INT32 view; see cu_seqlens64)
  const int64_t* cu_seqlens64;   // INT64 caller array, narrowed into the workspace by the
                                 // schedule kernel (cu_seqlens then points at the copy)
  const int32_t* ckpt_offsets;   // NULL: no checkpoint
  // outputs
  uint16_t* out;
  float* ht;
  float* ckpt;
  // sizes
  int32_t N, T, H, max_len;
  int32_t fixed_len;             // sequence length in the fixed layout
  int32_t split_jmax;            // prepare launch: only chunks j < split_jmax of a sequence
  int32_t fused_j0;              // fused launch: its prepare groups make chunks j >= fused_j0;
                                 // chunks below come from a preceding prepare launch
  int64_t slots;
  // workspace
  uint8_t* ws;
  WorkspaceLayout lay;
  uint32_t flags;
  uint32_t claim_items;          // prepare CTAs claim items from the counter at lay.claim
  long long wait_budget;         // clock cycles per bounded wait; < 0 forces a timeout
  // input front end (0: inputs used as given; bit 0 q/k L2 norm, bit 1 gate from the
  // raw BF16 gate in g, bit 2 beta from its logit), formed in FP32 by the prepare kernel
  uint32_t fe_flags;
  const float* A_log;            // [H]
  const float* dt_bias;          // [H][128]
  float lower_bound;
  float l2_eps;
};

// Tensor maps of the split variant (passed by value, __grid_constant__).
struct SplitMaps {
  CUtensorMap v_in;     // v [T][H][128] bf16, box (64 ch, 1 head, 64 tok), 128B swizzle
  CUtensorMap q_in;     // q [T][H][128] bf16, box (128 ch, 1 head, 64 tok), no swizzle
  CUtensorMap k_in;     // k, as q
  CUtensorMap g_in;     // g [T][H][128] f32, box (128 ch, 1 head, 64 tok), no swizzle
  CUtensorMap o_out;    // out [T][H][128] bf16, box (128 ch, 1 head, 64 tok), no swizzle
  CUtensorMap wt;       // [recs*128][64] f16, box (64, 128)
  CUtensorMap qg;       // [recs*64][128] f16, box (64, 64): one 64-channel panel
  CUtensorMap ut;       // [recs*128][64] f16, box (64, 128)
  CUtensorMap kd;       // [recs*64][128] f16, box (64, 64)
  CUtensorMap aqk;      // [recs*64][64] f16, box (64, 64)
  CUtensorMap qw;       // stream: [recs*128][128] f16, box (64, 128): one 64-channel panel
  CUtensorMap u;        // stream: [recs*64][128] f16, box (64, 64): one 64-channel panel
};

enum : int32_t {
  kStatusOk = 0,
  kStatusBadCuSeqlens = 16,
  kStatusBadCkptOffset = 17,
  kStatusTimeout = 18,
};

enum : uint32_t { kFlagValidate = 1u, kFlagForceTimeout = 2u, kFlagCu64 = 4u };

__device__ __forceinline__ void record_status(uint8_t* ws, int32_t code) {
  atomicCAS(reinterpret_cast<int32_t*>(ws), 0, code);
}

// Per-sequence geometry: start row, length, first chunk slot and the chunk split
// at the checkpoint.  Values from device metadata are clamped so that every
// derived address stays in bounds whatever the metadata holds.
struct SeqInfo {
  int32_t start, len;
  int32_t ck;     // checkpoint prefix length clamped to [0, len], or -1 without checkpoints
  int32_t nA;     // chunks covering [0, ck) when 0 < ck < len, else 0
  int32_t nch;    // chunks of the sequence
  int64_t slot0;  // first chunk slot
};

__device__ __forceinline__ SeqInfo seq_info(const KdaParams& p, int32_t n, bool need_slot = true) {
  SeqInfo s;
  if (p.cu_seqlens == nullptr) {
    s.start = n * p.fixed_len;
    s.len = p.fixed_len;
  } else {
    int32_t a = p.cu_seqlens[n], b = p.cu_seqlens[n + 1];
    a = min(max(a, 0), p.T);
    b = min(max(b, a), p.T);
    s.start = a;
    s.len = b - a;
  }
  s.ck = -1;
  s.nA = 0;
  if (p.ckpt_offsets != nullptr) {
    s.ck = min(max(p.ckpt_offsets[n], 0), s.len);
    if (s.ck > 0 && s.ck < s.len) s.nA = (s.ck + kC - 1) / kC;
  }
  const int32_t rest = s.len - (s.nA > 0 ? s.ck : 0);
  s.nch = s.nA + (rest + kC - 1) / kC;
  s.slot0 = 0;
  if (need_slot) {
    if (p.cu_seqlens == nullptr && p.ckpt_offsets == nullptr) {
      s.slot0 = static_cast<int64_t>(n) * ((p.fixed_len + kC - 1) / kC);
    } else {
      s.slot0 = reinterpret_cast<const int32_t*>(p.ws + p.lay.chunk_base)[n];
    }
  }
  return s;
}

// Token range of chunk j of a sequence: [t0, t0 + c), t0 relative to the sequence.
__device__ __forceinline__ void chunk_span(const SeqInfo& s, int32_t j, int32_t& t0, int32_t& c) {
  if (j < s.nA) {
    t0 = j * kC;
    c = min(kC, s.ck - t0);
  } else {
    const int32_t base = (s.nA > 0) ? s.ck : 0;
    t0 = base + (j - s.nA) * kC;
    c = min(kC, s.len - t0);
  }
}

}  // namespace kda
