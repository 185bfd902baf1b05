// kda_token.cuh — launch parameters of the per-token KDA kernels (kda_token.cu),
// shared with the host launcher.
#pragma once
#include <cstdint>

namespace kda {

constexpr int32_t kStatusBadStateIndex = 19;   // a decode state slot at or above the pool size
constexpr uint32_t kFeQkL2Norm = 1u, kFeGate = 2u, kFeBetaLogit = 4u;   // front-end switches

// Parameters of the per-token kernels (short sequences through kda_prefill, and
// kda_decode).  A CTA owns 32 (narrow) or all 128 (wide) value columns of one
// (sequence, head).
struct TokenParams {
  const uint16_t* q;
  const uint16_t* k;
  const uint16_t* v;
  const float* g;
  const uint16_t* beta;
  float scale;
  const float* src;              // state read first, [slots][H][128][128]; NULL = zero state
  float* dst;                    // state written last (same indexing as src); NULL = none
  const int32_t* slot;           // state slot of each sequence; NULL = the sequence index
  int32_t pool;                  // number of slots when slot != NULL
  const int32_t* cu_seqlens;     // NULL: fixed layout of fixed_len tokens per sequence
  int32_t fixed_len;
  const int32_t* ckpt_offsets;   // NULL: no checkpoint
  float* ckpt;                   // [N][H][128][128]
  float* steps;                  // [N][fixed_len][H][128][128] state after every token, or NULL
  uint16_t* out;
  int32_t N, T, H;
  // input front end (kda_decode; fe_flags = 0: inputs used as given)
  uint32_t fe_flags;             // kFeQkL2Norm | kFeGate | kFeBetaLogit
  const float* A_log;            // [H]          (kFeGate)
  const float* dt_bias;          // [H][128]     (kFeGate; g then holds the raw gate as BF16)
  float lower_bound;             // (kFeGate)
  float l2_eps;                  // (kFeQkL2Norm)
  uint8_t* ws;                   // prefill workspace (metadata check of validate mode) or NULL
  int32_t* status;               // sticky status word, or NULL
  uint32_t flags;
  long long wait_budget;         // clock cycles per bounded wait; < 0 forces a timeout
};

}  // namespace kda
