// kda_token.cu — the KDA recurrence taken one token at a time, for short
// sequences, single-token decode and the verification of a few draft tokens.
//
// Per (sequence, head) and token t, with S the K x V = 128 x 128 FP32 state:
//   S' = Diag(exp g_t) S
//   u  = beta_t (v_t - S'^T k_t)
//   S  = S' + k_t u^T
//   o_t = scale S^T q_t = scale (S'^T q_t + u (k_t . q_t))
// Every value column of S evolves on its own given (k_t, q_t, g_t, beta_t), so a
// CTA owns a slice of the columns of one (sequence, head) and keeps it in
// registers for the whole sequence: warp w holds key rows [16 w, 16 w + 16), lane
// l holds kCPT adjacent columns.  Two shapes are instantiated:
//   kCPT = 1  32 columns per CTA, 4 CTAs per (sequence, head): shortest chain per
//             token, for few (sequence, head) units;
//   kCPT = 4  128 columns per CTA (float4 state rows), 1 CTA per unit: fewer
//             instructions per column and 64 KB of state in flight per CTA, for
//             many units (decode of large batches).
// Per token a thread folds its 16 rows into partial column sums of S'^T k and
// S'^T q; one barrier makes the eight warps' partials visible, after which every
// thread has u and o_t for its columns and applies the rank-1 update.  The state
// is read from HBM once and written once.  Tokens are staged 16 at a time into
// shared memory by the copy engine (cp.async.bulk per token row, completion on an
// mbarrier), one block ahead of the arithmetic; once a block lands, exp(g), the
// FP32 k and q rows and k.q are formed once per block and shared by all columns.
//
// Decode over a slot-indexed state pool and per-token state export follow the
// FlashInfer KDA decode entry (SGLang kda_flashinfer.py "FlashInferKDAKernel":
// decode and target-verify over the same per-(sequence, head) state).
//
// Optional input front end (kda_decode), formed in FP32 in the per-block step so
// that no rounded intermediate reaches the recurrence (a BF16 copy of the
// normalised k or of beta moves the final state by about 2e-3 relative):
//   k, q <- x / sqrt(sum x^2 + eps)                        (kFeQkL2Norm)
//   g    <- lower_bound * sigmoid(exp(A_log) (a + dt_bias)) from the raw BF16 gate a
//                                                          (kFeGate)
//   beta <- sigmoid(beta)                                  (kFeBetaLogit)
// The parameter set is FlashInfer PR #4262's "Dispatch contract" (A_log per head,
// dt_bias per head and key channel, a negative lower bound, the three switches);
// the formula is this library's reading of it.
#include <cstdint>

#include "kda_common.cuh"
#include "kda_token.cuh"
#include "sm100_primitives.cuh"

namespace kda {
namespace tok {

constexpr int kWarps = 8;
constexpr int kRows = kD / kWarps;         // key rows per warp
constexpr int kThreads = kWarps * 32;
constexpr int kBlk = 16;                   // tokens per staged block
constexpr long long kDrainBudget = 2000000000LL;   // clock cycles
static_assert(kRows == 16, "16 key rows per warp");

constexpr uint32_t align128(uint32_t x) { return (x + 127u) / 128u * 128u; }

template <int kCPT>
struct Cfg {
  static constexpr int kCols = 32 * kCPT;          // value columns per CTA
  static constexpr int kSlices = kD / kCols;       // CTAs per (sequence, head)
  // staged block, two buffers: k, q [16][128] bf16; g [16][128] f32 (exp(g) after
  // landing, in place); this CTA's v columns [16][kCols] bf16; the raw gate
  // [16][128] bf16 when the front end forms g
  static constexpr uint32_t kOffK = 0;
  static constexpr uint32_t kOffQ = kOffK + kBlk * kD * 2;
  static constexpr uint32_t kOffG = kOffQ + kBlk * kD * 2;
  static constexpr uint32_t kOffV = kOffG + kBlk * kD * 4;
  static constexpr uint32_t kOffA = align128(kOffV + kBlk * kCols * 2);
  static constexpr uint32_t kStage = kOffA + kBlk * kD * 2;
  // per block, one buffer: k, q as f32 [16][128], beta [16], k.q [16]
  static constexpr uint32_t kOffKF = 2 * kStage;
  static constexpr uint32_t kOffQF = kOffKF + kBlk * kD * 4;
  static constexpr uint32_t kOffBeta = kOffQF + kBlk * kD * 4;
  static constexpr uint32_t kOffKQ = kOffBeta + kBlk * 4;
  // per token, two buffers: per warp and lane the partial sums (S'^T k)[kCPT], (S'^T q)[kCPT]
  // front end: dt_bias of the head [128] f32 (copied with block 0) and exp(A_log)
  static constexpr uint32_t kOffDt = kOffKQ + kBlk * 4;
  static constexpr uint32_t kOffRate = kOffDt + kD * 4;
  static constexpr uint32_t kOffPart = align128(kOffRate + 16);
  static constexpr uint32_t kPartBuf = kWarps * 32 * 2 * kCPT * 4;
  static constexpr uint32_t kSmem = kOffPart + 2 * kPartBuf;
};

template <int kCPT>
struct Vec;
template <>
struct Vec<1> {
  __device__ static void load(const float* p, float (&x)[1]) { x[0] = *p; }
  __device__ static void store(float* p, const float (&x)[1]) { *p = x[0]; }
};
template <>
struct Vec<4> {
  __device__ static void load(const float* p, float (&x)[4]) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x;
    x[1] = v.y;
    x[2] = v.z;
    x[3] = v.w;
  }
  __device__ static void store(float* p, const float (&x)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(x[0], x[1], x[2], x[3]);
  }
};

// write a thread's rows of its columns into the state at `base` ([128][128] FP32)
template <int kCPT>
__device__ __forceinline__ void store_slice(float* base, const float (&s)[kRows][kCPT], int warp,
                                            int col0) {
#pragma unroll
  for (int r = 0; r < kRows; ++r)
    Vec<kCPT>::store(base + static_cast<int64_t>(warp * kRows + r) * kD + col0, s[r]);
}

__device__ __forceinline__ void record(const TokenParams& p, int32_t code) {
  if (p.status != nullptr) atomicCAS(p.status, 0, code);
}

template <int kCPT>
__device__ __forceinline__ void store_out(uint16_t* dst, const float (&o)[kCPT]) {
  if constexpr (kCPT == 1) {
    *dst = static_cast<uint16_t>(pack_bf16(o[0], 0.f) & 0xffffu);
  } else {
    *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]));
  }
}

template <int kCPT>
__device__ __forceinline__ void zero_out(uint16_t* dst) {
  if constexpr (kCPT == 1) {
    *dst = 0;
  } else {
    *reinterpret_cast<uint2*>(dst) = make_uint2(0u, 0u);
  }
}

__device__ __forceinline__ float sigmoid_f32(float x) { return 1.f / (1.f + ex2(-x * kLog2e)); }

__device__ __forceinline__ float4 bf16x4_to_f32(const uint2 w) {
  return make_float4(__uint_as_float(w.x << 16), __uint_as_float(w.x & 0xffff0000u),
                     __uint_as_float(w.y << 16), __uint_as_float(w.y & 0xffff0000u));
}

// kFE: the input front end is compiled in (its switches are read from p.fe_flags);
// without it the plain path carries none of its registers
template <int kCPT, bool kFE>
__device__ __forceinline__ void token_body(const TokenParams& p, uint8_t* smem) {
  using C = Cfg<kCPT>;
  __shared__ __align__(8) uint64_t full[2];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int slice = static_cast<int>(blockIdx.x % C::kSlices);
  const int64_t unit = blockIdx.x / C::kSlices;
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
  const int col0 = slice * C::kCols + lane * kCPT;              // this thread's first column
  int64_t sidx = n;
  if (p.slot != nullptr) {
    const int32_t si = p.slot[n];
    if (si < 0 || si >= p.pool) {
      // padding entry (negative) or out-of-range slot: no state access, zero output
      if (si >= p.pool && tid == 0 && slice == 0 && h == 0) record(p, kStatusBadStateIndex);
      for (int t = warp; t < len; t += kWarps)
        zero_out<kCPT>(p.out + (start + t) * tok_stride + h * kD + col0);
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

  const bool fe_gate = kFE && (p.fe_flags & kFeGate) != 0;
  const bool fe_norm = kFE && (p.fe_flags & kFeQkL2Norm) != 0;
  const bool fe_beta = kFE && (p.fe_flags & kFeBetaLogit) != 0;
  const uint32_t tok_bytes = kD * 2 * 2 + (fe_gate ? kD * 2 : kD * 4) + C::kCols * 2;
  const int nblk = (len + kBlk - 1) / kBlk;
  // block issue: warp 0 lanes copy one token row each; warp 1 lanes fetch beta into
  // a register that is parked in shared memory once the block has landed
  auto issue = [&](int b) {
    uint8_t* buf = smem + (b & 1) * C::kStage;
    const int t0 = b * kBlk, nt = min(kBlk, len - t0);
    if (warp == 0) {
      if (lane == 0) {
        // block 0 also brings the head's dt_bias row for the gate
        const bool dt = fe_gate && b == 0;
        mbar_arrive_expect_tx(&full[b & 1],
                              static_cast<uint32_t>(nt) * tok_bytes + (dt ? kD * 4 : 0));
        if (dt)
          bulk_load(smem + C::kOffDt, p.dt_bias + static_cast<int64_t>(h) * kD, kD * 4,
                    &full[0]);
      }
      if (lane < nt) {
        const int64_t row = static_cast<int64_t>(start + t0 + lane) * tok_stride + h * kD;
        bulk_load(buf + C::kOffK + lane * kD * 2, p.k + row, kD * 2, &full[b & 1]);
        bulk_load(buf + C::kOffQ + lane * kD * 2, p.q + row, kD * 2, &full[b & 1]);
        if (fe_gate)
          bulk_load(buf + C::kOffA + lane * kD * 2, reinterpret_cast<const uint16_t*>(p.g) + row,
                    kD * 2, &full[b & 1]);
        else
          bulk_load(buf + C::kOffG + lane * kD * 4, p.g + row, kD * 4, &full[b & 1]);
        bulk_load(buf + C::kOffV + lane * C::kCols * 2, p.v + row + slice * C::kCols,
                  C::kCols * 2, &full[b & 1]);
      }
    }
  };
  float beta_next = 0.f;
  auto fetch_beta = [&](int b) {
    const int t0 = b * kBlk;
    if (warp == 1 && lane < min(kBlk, len - t0)) {
      beta_next = bf16_to_f32(p.beta[static_cast<int64_t>(start + t0 + lane) * p.H + h]);
      if (fe_beta) beta_next = sigmoid_f32(beta_next);
    }
  };

  if (nblk > 0) {
    issue(0);
    fetch_beta(0);
  }

  // ---- the state slice (loads overlap the first block's copies)
  float s[kRows][kCPT];
  if (p.src != nullptr) {
#pragma unroll
    for (int r = 0; r < kRows; ++r)
      Vec<kCPT>::load(p.src + soff + static_cast<int64_t>(warp * kRows + r) * kD + col0, s[r]);
  } else {
#pragma unroll
    for (int r = 0; r < kRows; ++r)
#pragma unroll
      for (int c = 0; c < kCPT; ++c) s[r][c] = 0.f;
  }
  if (ck == 0) store_slice<kCPT>(p.ckpt + ck_off, s, warp, col0);
  // exp(A_log) of the head, parked before the first block's barrier (its load overlaps
  // the state loads and the block's copies)
  if (fe_gate && warp == 1 && lane == 31 && nblk > 0)
    *reinterpret_cast<float*>(smem + C::kOffRate) = expf(p.A_log[h]);

  float* kf = reinterpret_cast<float*>(smem + C::kOffKF);
  float* qf = reinterpret_cast<float*>(smem + C::kOffQF);
  float* betas = reinterpret_cast<float*>(smem + C::kOffBeta);
  float* kqs = reinterpret_cast<float*>(smem + C::kOffKQ);
  bool ok = true;
  for (int b = 0; b < nblk && ok; ++b) {
    uint8_t* buf = smem + (b & 1) * C::kStage;
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
    // ---- per block: exp(g) in place, k and q to f32, k.q per token, beta parked.
    // Quad i4 covers channels 4 (i4 % 32) .. +3 of token i4 / 32, so the 32 lanes of a
    // warp together hold one token row and reduce its k.q with shuffles.
    float* e = reinterpret_cast<float*>(buf + C::kOffG);
    const uint2* kb = reinterpret_cast<const uint2*>(buf + C::kOffK);
    const uint2* qb = reinterpret_cast<const uint2*>(buf + C::kOffQ);
    if constexpr (!kFE) {
#pragma unroll
      for (int j = 0; j < kBlk * kD / 4 / kThreads; ++j) {
        const int i4 = tid + j * kThreads;
        const int tk = i4 >> 5;   // warp-uniform
        if (tk < nt) {
          const float4 gv = reinterpret_cast<const float4*>(e)[i4];
          reinterpret_cast<float4*>(e)[i4] = make_float4(ex2(gv.x * kLog2e), ex2(gv.y * kLog2e),
                                                         ex2(gv.z * kLog2e), ex2(gv.w * kLog2e));
          const float4 kv = bf16x4_to_f32(kb[i4]), qv = bf16x4_to_f32(qb[i4]);
          reinterpret_cast<float4*>(kf)[i4] = kv;
          reinterpret_cast<float4*>(qf)[i4] = qv;
          float dot = fmaf(kv.x, qv.x, fmaf(kv.y, qv.y, fmaf(kv.z, qv.z, kv.w * qv.w)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          if (lane == 0) kqs[tk] = dot;
        }
      }
    } else {
      const uint2* ab = reinterpret_cast<const uint2*>(buf + C::kOffA);
      // gate parameters of this head for the lane's four key channels (the loop below
      // gives lane l channels 4 l .. 4 l + 3 of every row), from shared memory so
      // that they hold no registers across the token loop
      float rate = 0.f;
      float4 dtb = make_float4(0.f, 0.f, 0.f, 0.f);
      if (fe_gate) {
        rate = *reinterpret_cast<const float*>(smem + C::kOffRate);
        dtb = reinterpret_cast<const float4*>(smem + C::kOffDt)[lane];
      }
#pragma unroll
      for (int j = 0; j < kBlk * kD / 4 / kThreads; ++j) {
        const int i4 = tid + j * kThreads;
        const int tk = i4 >> 5;   // warp-uniform
        if (tk < nt) {
          float4 gv;
          if (fe_gate) {
            const float4 av = bf16x4_to_f32(ab[i4]);
            gv = make_float4(p.lower_bound * sigmoid_f32(rate * (av.x + dtb.x)),
                             p.lower_bound * sigmoid_f32(rate * (av.y + dtb.y)),
                             p.lower_bound * sigmoid_f32(rate * (av.z + dtb.z)),
                             p.lower_bound * sigmoid_f32(rate * (av.w + dtb.w)));
          } else {
            gv = reinterpret_cast<const float4*>(e)[i4];
          }
          reinterpret_cast<float4*>(e)[i4] = make_float4(ex2(gv.x * kLog2e), ex2(gv.y * kLog2e),
                                                         ex2(gv.z * kLog2e), ex2(gv.w * kLog2e));
          float4 kv = bf16x4_to_f32(kb[i4]), qv = bf16x4_to_f32(qb[i4]);
          float dot = fmaf(kv.x, qv.x, fmaf(kv.y, qv.y, fmaf(kv.z, qv.z, kv.w * qv.w)));
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
          if (fe_norm) {
            float kk = fmaf(kv.x, kv.x, fmaf(kv.y, kv.y, fmaf(kv.z, kv.z, kv.w * kv.w)));
            float qq = fmaf(qv.x, qv.x, fmaf(qv.y, qv.y, fmaf(qv.z, qv.z, qv.w * qv.w)));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
              kk += __shfl_xor_sync(0xffffffffu, kk, o);
              qq += __shfl_xor_sync(0xffffffffu, qq, o);
            }
            const float rk = rsqrtf(kk + p.l2_eps), rq = rsqrtf(qq + p.l2_eps);
            kv = make_float4(kv.x * rk, kv.y * rk, kv.z * rk, kv.w * rk);
            qv = make_float4(qv.x * rq, qv.y * rq, qv.z * rq, qv.w * rq);
            dot *= rk * rq;
          }
          reinterpret_cast<float4*>(kf)[i4] = kv;
          reinterpret_cast<float4*>(qf)[i4] = qv;
          if (lane == 0) kqs[tk] = dot;
        }
      }
    }
    if (warp == 1 && lane < nt) betas[lane] = beta_next;
    fence_proxy_async_smem();   // generic writes to the stage ordered before its next bulk copies
    __syncthreads();
    if (b + 1 < nblk) {
      issue(b + 1);
      fetch_beta(b + 1);
    }
    for (int i = 0; i < nt; ++i) {
      const int t = t0 + i;
      const float4* kp = reinterpret_cast<const float4*>(kf + i * kD + warp * kRows);
      const float4* qp = reinterpret_cast<const float4*>(qf + i * kD + warp * kRows);
      const float4* ep = reinterpret_cast<const float4*>(e + i * kD + warp * kRows);
      // two accumulators per sum shorten the FMA chains of the one-column shape; with
      // four columns the chains are independent already
      constexpr int kAcc = kCPT == 1 ? 2 : 1;
      float a[kCPT][kAcc], bq[kCPT][kAcc];
#pragma unroll
      for (int c = 0; c < kCPT; ++c)
#pragma unroll
        for (int x = 0; x < kAcc; ++x) a[c][x] = bq[c][x] = 0.f;
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const float4 kv = kp[r4], qv = qp[r4], ev = ep[r4];
        const float kr[4] = {kv.x, kv.y, kv.z, kv.w};
        const float qr[4] = {qv.x, qv.y, qv.z, qv.w};
        const float er[4] = {ev.x, ev.y, ev.z, ev.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = 4 * r4 + j;
#pragma unroll
          for (int c = 0; c < kCPT; ++c) {
            s[r][c] *= er[j];
            a[c][j % kAcc] = fmaf(s[r][c], kr[j], a[c][j % kAcc]);
            bq[c][j % kAcc] = fmaf(s[r][c], qr[j], bq[c][j % kAcc]);
          }
        }
      }
      float* part = reinterpret_cast<float*>(smem + C::kOffPart + (t & 1) * C::kPartBuf);
      {
        float pa[kCPT], pb[kCPT];
#pragma unroll
        for (int c = 0; c < kCPT; ++c) {
          pa[c] = a[c][0];
          pb[c] = bq[c][0];
#pragma unroll
          for (int x = 1; x < kAcc; ++x) {
            pa[c] += a[c][x];
            pb[c] += bq[c][x];
          }
        }
        Vec<kCPT>::store(part + (warp * 32 + lane) * 2 * kCPT, pa);
        Vec<kCPT>::store(part + (warp * 32 + lane) * 2 * kCPT + kCPT, pb);
      }
      __syncthreads();
      float A[kCPT], B[kCPT];
#pragma unroll
      for (int c = 0; c < kCPT; ++c) A[c] = B[c] = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        float pa[kCPT], pb[kCPT];
        Vec<kCPT>::load(part + (w * 32 + lane) * 2 * kCPT, pa);
        Vec<kCPT>::load(part + (w * 32 + lane) * 2 * kCPT + kCPT, pb);
#pragma unroll
        for (int c = 0; c < kCPT; ++c) {
          A[c] += pa[c];
          B[c] += pb[c];
        }
      }
      const float kq = kqs[i], bt = betas[i];
      const uint16_t* vrow = reinterpret_cast<const uint16_t*>(buf + C::kOffV + i * C::kCols * 2);
      float u[kCPT], o[kCPT];
#pragma unroll
      for (int c = 0; c < kCPT; ++c) {
        u[c] = bt * (bf16_to_f32(vrow[lane * kCPT + c]) - A[c]);
        o[c] = p.scale * fmaf(u[c], kq, B[c]);
      }
      if (warp == (t & (kWarps - 1)))
        store_out<kCPT>(p.out + (start + t) * tok_stride + h * kD + col0, o);
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const float4 kv = kp[r4];
        const float kr[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int c = 0; c < kCPT; ++c) s[4 * r4 + j][c] = fmaf(kr[j], u[c], s[4 * r4 + j][c]);
      }
      if (t + 1 == ck) store_slice<kCPT>(p.ckpt + ck_off, s, warp, col0);
      if (p.steps != nullptr)
        store_slice<kCPT>(
            p.steps + ((static_cast<int64_t>(n) * p.fixed_len + t) * p.H + h) * kD * kD, s, warp,
            col0);
    }
    // (the next block's conversion writes kf, qf, k.q and beta only after the barrier
    // that follows its landing, which every thread reaches after this token loop)
  }
  if (ok && p.dst != nullptr) store_slice<kCPT>(p.dst + soff, s, warp, col0);
}

}  // namespace tok

__global__ void __launch_bounds__(tok::kThreads, 3) kda_token_narrow_kernel(const TokenParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  tok::token_body<1, false>(p, smem);
}

__global__ void __launch_bounds__(tok::kThreads, 2) kda_token_wide_kernel(const TokenParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  tok::token_body<4, false>(p, smem);
}

__global__ void __launch_bounds__(tok::kThreads, 3)
kda_token_narrow_fe_kernel(const TokenParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  tok::token_body<1, true>(p, smem);
}

__global__ void __launch_bounds__(tok::kThreads, 2) kda_token_wide_fe_kernel(const TokenParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  tok::token_body<4, true>(p, smem);
}

namespace tok {
extern const uint32_t kSmemNarrow = Cfg<1>::kSmem;
extern const uint32_t kSmemWide = Cfg<4>::kSmem;
extern const int kThreadsPerCta = kThreads;
}  // namespace tok

}  // namespace kda
