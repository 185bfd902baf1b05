// kda_token.cu — the KDA recurrence taken one token at a time, for short
// sequences, single-token decode and the verification of a few draft tokens.
//
// Per (sequence, head) and token t, with S the K x V = 128 x 128 FP32 state:
//   S' = Diag(exp g_t) S
//   u  = beta_t (v_t - S'^T k_t)
//   S  = S' + k_t u^T
//   o_t = scale S^T q_t = scale (S'^T q_t + u (k_t . q_t))
// Every value column of S evolves on its own given (k_t, q_t, g_t, beta_t), so a
// CTA owns 32 columns of one (sequence, head) and keeps that 128 x 32 slice in
// registers for the whole sequence: warp w holds key rows [16 w, 16 w + 16), lane
// l holds column l of the slice.  Per token a thread folds its 16 rows into two
// partial column sums (S'^T k and S'^T q) and one partial k.q; one barrier makes
// the eight warps' partials visible, after which every thread has u and o_t for
// its column and applies the rank-1 update to its rows.  The state is read from
// HBM once and written once; tokens are staged 16 at a time into shared memory by
// the copy engine (cp.async.bulk per token row, completion on an mbarrier), one
// block ahead of the arithmetic, and exp(g) is taken once per staged element.
//
// Decode over a slot-indexed state pool and per-token state export follow the
// FlashInfer KDA decode entry (SGLang kda_flashinfer.py "FlashInferKDAKernel":
// decode and target-verify over the same per-(sequence, head) state).
#include <cstdint>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {
namespace tok {

constexpr int kCols = 32;                  // value columns per CTA (one per lane)
constexpr int kSlices = kD / kCols;        // CTAs per (sequence, head)
constexpr int kWarps = 8;
constexpr int kRows = kD / kWarps;         // key rows per warp
constexpr int kThreads = kWarps * 32;
constexpr int kBlk = 16;                   // tokens per staged block
// one staged block: k, q [16][128] bf16; g -> exp(g) [16][128] f32; this CTA's
// v columns [16][32] bf16; beta [16] f32
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffQ = kOffK + kBlk * kD * 2;
constexpr uint32_t kOffE = kOffQ + kBlk * kD * 2;
constexpr uint32_t kOffV = kOffE + kBlk * kD * 4;
constexpr uint32_t kOffB = kOffV + kBlk * kCols * 2;
constexpr uint32_t kBufBytes = (kOffB + kBlk * 4 + 127) / 128 * 128;
constexpr uint32_t kTokBytes = kD * 2 + kD * 2 + kD * 4 + kCols * 2;   // copied per token
constexpr long long kDrainBudget = 2000000000LL;                     // clock cycles
static_assert(kRows == 16, "the unpacking below assumes 16 rows per warp");

__device__ __forceinline__ void unpack8(const uint4& w, float* f) {
  const uint32_t x[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(x[i] << 16);
    f[2 * i + 1] = __uint_as_float(x[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  return static_cast<uint16_t>(pack_bf16(x, 0.f) & 0xffffu);
}

// write a thread's 16 rows of column `col` into the state at `base` ([128][128] FP32)
__device__ __forceinline__ void store_slice(float* base, const float (&s)[kRows], int warp,
                                            int col) {
#pragma unroll
  for (int r = 0; r < kRows; ++r) base[static_cast<int64_t>(warp * kRows + r) * kD + col] = s[r];
}

__device__ __forceinline__ void record(const TokenParams& p, int32_t code) {
  if (p.status != nullptr) atomicCAS(p.status, 0, code);
}

extern const uint32_t kSmemAllocBytes = 2 * kBufBytes;
extern const int kThreadsPerCta = kThreads;
extern const int kCtasPerUnit = kSlices;

}  // namespace tok

__global__ void __launch_bounds__(tok::kThreads, 3) kda_token_kernel(const TokenParams p) {
  using namespace tok;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float2 part[2][kWarps][32];   // per warp: (S'^T k, S'^T q) partial column sums
  __shared__ float kqp[2][kWarps];         // per warp: partial k . q
  __shared__ __align__(8) uint64_t full[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = static_cast<int>(blockIdx.x % kSlices);
  const int64_t unit = blockIdx.x / kSlices;
  const int32_t n = static_cast<int32_t>(unit / p.H);
  const int32_t h = static_cast<int32_t>(unit - static_cast<int64_t>(n) * p.H);
  if ((p.flags & kFlagValidate) && p.ws != nullptr &&
      reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0)
    return;

  // ---- sequence geometry (device metadata clamped so every address stays in bounds)
  int32_t start, len;
  if (p.cu_seqlens == nullptr) {
    start = n * p.fixed_len;
    len = p.fixed_len;
  } else {
    int32_t a = p.cu_seqlens[n], b = p.cu_seqlens[n + 1];
    a = min(max(a, 0), p.T);
    b = min(max(b, a), p.T);
    start = a;
    len = b - a;
  }
  const int32_t ck = p.ckpt_offsets ? min(max(p.ckpt_offsets[n], 0), len) : -1;
  const int64_t tok_stride = static_cast<int64_t>(p.H) * kD;   // elements between token rows
  const int col = slice * kCols + lane;
  int64_t sidx = n;
  if (p.slot != nullptr) {
    const int32_t si = p.slot[n];
    if (si < 0 || si >= p.pool) {
      // padding entry (negative) or out-of-range slot: no state access, zero output
      if (si >= p.pool && tid == 0 && slice == 0 && h == 0) record(p, kStatusBadStateIndex);
      for (int t = warp; t < len; t += kWarps)
        p.out[(start + t) * tok_stride + h * kD + col] = 0;
      return;
    }
    sidx = si;
  }
  const int64_t soff = (sidx * p.H + h) * static_cast<int64_t>(kD * kD);   // state origin
  const int64_t ck_off = (static_cast<int64_t>(n) * p.H + h) * kD * kD;    // checkpoint origin

  if (tid == 0) {
    mbar_init(&full[0], 1);
    mbar_init(&full[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  const int nblk = (len + kBlk - 1) / kBlk;
  // block issue: warp 0 lanes copy one token row each; warp 1 lanes fetch beta into
  // a register that is parked in shared memory once the block has landed
  auto issue = [&](int b) {
    uint8_t* buf = smem + (b & 1) * kBufBytes;
    const int t0 = b * kBlk, nt = min(kBlk, len - t0);
    if (warp == 0) {
      if (lane == 0) mbar_arrive_expect_tx(&full[b & 1], static_cast<uint32_t>(nt) * kTokBytes);
      if (lane < nt) {
        const int64_t row = static_cast<int64_t>(start + t0 + lane) * tok_stride + h * kD;
        bulk_load(buf + kOffK + lane * kD * 2, p.k + row, kD * 2, &full[b & 1]);
        bulk_load(buf + kOffQ + lane * kD * 2, p.q + row, kD * 2, &full[b & 1]);
        bulk_load(buf + kOffE + lane * kD * 4, p.g + row, kD * 4, &full[b & 1]);
        bulk_load(buf + kOffV + lane * kCols * 2, p.v + row + slice * kCols, kCols * 2,
                  &full[b & 1]);
      }
    }
  };
  float beta_next = 0.f;
  auto fetch_beta = [&](int b) {
    const int t0 = b * kBlk;
    if (warp == 1 && lane < min(kBlk, len - t0))
      beta_next = bf16_to_f32(p.beta[static_cast<int64_t>(start + t0 + lane) * p.H + h]);
  };
  if (nblk > 0) {
    issue(0);
    fetch_beta(0);
  }

  // ---- the state slice (loads overlap the first block's copies)
  float s[kRows];
  if (p.src != nullptr) {
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      s[r] = p.src[soff + static_cast<int64_t>(warp * kRows + r) * kD + col];
  } else {
#pragma unroll
    for (int r = 0; r < kRows; ++r) s[r] = 0.f;
  }
  if (ck == 0) store_slice(p.ckpt + ck_off, s, warp, col);

  bool ok = true;
  for (int b = 0; b < nblk && ok; ++b) {
    uint8_t* buf = smem + (b & 1) * kBufBytes;
    const int t0 = b * kBlk, nt = min(kBlk, len - t0);
    ok = mbar_wait(&full[b & 1], static_cast<uint32_t>((b >> 1) & 1), p.wait_budget);
    if (__syncthreads_or(!ok)) {
      // give up: record it, then wait (bounded) for this block's copies before leaving
      if (tid == 0) {
        record(p, kStatusTimeout);
        mbar_wait(&full[b & 1], static_cast<uint32_t>((b >> 1) & 1), kDrainBudget);
      }
      __syncthreads();
      ok = false;
      break;
    }
    // g -> exp(g) in place, beta parked
    float* e = reinterpret_cast<float*>(buf + kOffE);
    for (int i = tid; i < nt * kD; i += kThreads) e[i] = ex2(e[i] * kLog2e);
    if (warp == 1 && lane < nt) reinterpret_cast<float*>(buf + kOffB)[lane] = beta_next;
    fence_proxy_async_smem();   // generic writes ordered before the next bulk copies
    __syncthreads();
    if (b + 1 < nblk) {
      issue(b + 1);
      fetch_beta(b + 1);
    }
    const float* eb = e;
    for (int i = 0; i < nt; ++i) {
      const int t = t0 + i;
      const uint4* kp = reinterpret_cast<const uint4*>(buf + kOffK + i * kD * 2 + warp * kRows * 2);
      const uint4* qp = reinterpret_cast<const uint4*>(buf + kOffQ + i * kD * 2 + warp * kRows * 2);
      const float4* ep = reinterpret_cast<const float4*>(eb + i * kD + warp * kRows);
      float kf[kRows], qf[kRows];
      unpack8(kp[0], kf);
      unpack8(kp[1], kf + 8);
      unpack8(qp[0], qf);
      unpack8(qp[1], qf + 8);
      float a = 0.f, bq = 0.f, kq = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const float4 ev = ep[c];
        const float ef[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = 4 * c + j;
          s[r] *= ef[j];
          a = fmaf(s[r], kf[r], a);
          bq = fmaf(s[r], qf[r], bq);
          kq = fmaf(kf[r], qf[r], kq);
        }
      }
      part[t & 1][warp][lane] = make_float2(a, bq);
      if (lane == 0) kqp[t & 1][warp] = kq;
      __syncthreads();
      float A = 0.f, B = 0.f, KQ = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float2 pw = part[t & 1][w][lane];
        A += pw.x;
        B += pw.y;
        KQ += kqp[t & 1][w];
      }
      const float vv = bf16_to_f32(reinterpret_cast<const uint16_t*>(buf + kOffV + i * kCols * 2)[lane]);
      const float bt = reinterpret_cast<const float*>(buf + kOffB)[i];
      const float u = bt * (vv - A);
      if (warp == (t & (kWarps - 1)))
        p.out[(start + t) * tok_stride + h * kD + col] = f32_to_bf16_rn(p.scale * fmaf(u, KQ, B));
#pragma unroll
      for (int r = 0; r < kRows; ++r) s[r] = fmaf(kf[r], u, s[r]);
      if (t + 1 == ck) store_slice(p.ckpt + ck_off, s, warp, col);
      if (p.steps != nullptr)
        store_slice(p.steps + ((static_cast<int64_t>(n) * p.fixed_len + t) * p.H + h) * kD * kD,
                    s, warp, col);
    }
  }
  if (ok && p.dst != nullptr) store_slice(p.dst + soff, s, warp, col);
}

}  // namespace kda
