// kda_recurrence.cuh — inter-chunk recurrence with the fused output (body shared
// by the split recurrence kernel and the recurrence CTAs of the fused launch).
//
// One CTA per (sequence, head); the chunks of the sequence are walked in order,
// the state S stays in tensor memory from chunk to chunk, tcgen05 UMMAs fed by
// TMA carry it, and the output (intra-chunk causal term plus the read of S by
// q) is formed in the same CTA.  The state is
// kept transposed, S^T[v][k], in TMEM lanes v = 0..127, so every UMMA has M = 128:
//   P_W^T = S0^T W^T                            (N=64, K=128; f16; B = W^T, MN-major)
//   P_Q^T = S0^T (Q Gamma)^T                    (N=64, K=128; f16; B = Q Gamma rows, K-major)
//   Ud^T  = U^T - P_W^T                         (threads; f16 operand)
//   S^T   = S0^T Diag(Gamma_end) + Ud^T Kd      (N=128, K=64; f16; B = Kd rows, MN-major)
//   O^T   = scale (P_Q^T + Ud^T Aqk^T)          (N=64, K=64; f16)
// A checkpoint offset p is a chunk boundary of the schedule, so the checkpoint
// state is S after the chunk that ends at p (h0 for p = 0, the final state for
// p = len).
//
// Serial chain per chunk: S ready -> (state warps) f16 S0^T into TMEM -> P_W
// -> (state warps) f16 Ud^T into TMEM and the decayed S -> S update.  P_Q is
// issued right behind P_W and runs while the state warps form Ud.
// S0^T and Ud^T are the A operands of their UMMAs straight from tensor memory,
// so shared memory only feeds the B tiles.  The state warps and the issuing
// warp meet at two hardware named barriers per chunk (S0^T ready, Ud^T ready):
// an mbarrier hand-off between warps costs several hundred cycles inside this
// kernel, a named barrier a few tens.  [P_W | P_Q/O] alternate between two TMEM
// regions, so the output warps drain chunk j while chunk j+1 proceeds; the
// chunk operands stream through a three-stage TMA ring.
//
// Tensor memory (512 columns):
//   [0, 128)    S^T f32 (lane v, column k)
//   [128, 384)  two regions: P_W^T (64 columns) then P_Q^T / O^T (64 columns)
//   [384, 448)  S0^T f16, two k per column (A operand of P_W and P_Q)
//   [448, 480)  Ud^T f16, two tokens per column (A operand of the update and O)
//
// Warp roles:
//   warps 0-7   state warps: warp w serves TMEM lanes 32 (w % 4) .. + 31 and half
//               w / 4 of every state row (64 columns; 32 tokens of P_W / Ud);
//   warps 8-11  output warps: read O^T out of TMEM and store o;
//   warp 12     issues every UMMA (lane 0) after the named barriers;
//   warp 13     lane 0 streams the operand ring.
//
// Every wait is bounded; a failed wait is combined across the participants of
// the next named barrier (bar.red.or), so all of them leave together.
//
// In-place state update (ht == h0) is safe: each thread reads its part of the h0
// column before writing the same part of ht, and a (sequence, head) pair is
// owned by exactly one CTA (FlashInfer PR #4262 "Physical schedules and true
// in-place state update" describes the same ownership rule).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace rec {
constexpr uint32_t kWQ = 0;          // 16 KB W^T [128 k][64 tok] f16, MN-major B;
                                     // 16 KB Q Gamma [64 tok][128 k] f16, K-major B, 2 panels
constexpr uint32_t kUT = 32768;      // 16 KB U^T  [128 v][64 tok] f16 (128B swizzle)
constexpr uint32_t kKd = 49152;      // 16 KB Kd [64 tok][128 k] f16, MN-major B, 2 panels
constexpr uint32_t kAqk = 65536;     //  8 KB Aqk  [64 r][64 s] f16, K-major B
constexpr uint32_t kGC = 73728;      // 512 B Gamma_end f32 [128]
constexpr uint32_t kStage = 74752;
constexpr int kStages = 3;
constexpr uint32_t kBytes = kStages * kStage;
constexpr uint32_t kSmemAlloc = kBytes + 1024;
constexpr uint32_t kStageTx = 32768 + 16384 + 16384 + 8192 + 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColP = 128;
constexpr uint32_t kColS0 = 384;
constexpr uint32_t kColUd = 448;
constexpr int kRegions = 2;
constexpr int kStateWarps = 8, kOutWarps = 4;
constexpr int kMmaWarp = kStateWarps + kOutWarps;
constexpr int kTmaWarp = kMmaWarp + 1;
constexpr int kThreads = (kTmaWarp + 1) * 32;
constexpr uint32_t kStateThreads = kStateWarps * 32;
constexpr uint32_t kOutThreads = kOutWarps * 32;
constexpr uint32_t kChainThreads = kStateThreads + 32;   // state warps + the issuing warp
constexpr uint32_t kBarS0 = 1, kBarUd = 2, kBarOut = 3, kBarOutOr = 4;   // named barriers
static_assert(kSmemAlloc <= 227 * 1024, "shared memory budget");
static_assert(kColP + kRegions * 128 <= kColS0 && kColUd + 32 <= 512, "tensor memory budget");
}  // namespace rec

__device__ __forceinline__ uint32_t region_col(int j) { return rec::kColP + 128u * (j % rec::kRegions); }

// Acquire the ready flag of a record written by a prepare CTA of the same launch
// (bounded poll), then order this thread's later TMA reads after it.
__device__ __forceinline__ bool wait_record(const KdaParams& p, int64_t rec, long long budget) {
  if (budget < 0) return false;
  const int32_t* flag = reinterpret_cast<const int32_t*>(p.ws + p.lay.ready) + rec;
  const long long t0 = clock64();
  for (;;) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) break;
    if (clock64() - t0 > budget) return false;
    __nanosleep(64);
  }
  asm volatile("fence.proxy.async.global;" ::: "memory");
  return true;
}

// The recurrence of one (sequence, head) unit.  kFused: the chunk records come
// from prepare CTAs of the same launch, so each one is awaited on its flag.
template <bool kFused>
__device__ __forceinline__ void recurrence_body(const KdaParams& p, const SplitMaps& maps,
                                                uint8_t* smem_raw, int unit) {
  using namespace rec;
  uint8_t* sm = smem_align<1024>(smem_raw);
  __shared__ uint64_t full_bar[kStages], empty_bar[kStages], oready_bar[kRegions], ofree_bar[kRegions];
  __shared__ uint64_t mma1_bar, sready_bar, drain_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int32_t s_abort;
  volatile int32_t* abort_flag = &s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;
  const int h = unit % p.H;
  int32_t n = unit / p.H;
  if (p.cu_seqlens != nullptr)
    n = reinterpret_cast<const int32_t*>(p.ws + p.lay.seq_order)[n];
  if (n < 0 || n >= p.N) return;
  const SeqInfo si = seq_info(p, n);
  const int32_t nch = si.nch;
  const int64_t nh = static_cast<int64_t>(n) * p.H + h;
  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 2);   // the issuer's last commit of the chunk + the output store
    }
    for (int i = 0; i < kRegions; ++i) {
      mbar_init(&oready_bar[i], 1);
      mbar_init(&ofree_bar[i], kOutThreads);
    }
    mbar_init(&mma1_bar, 1);
    mbar_init(&sready_bar, 1);
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  if (warp >= kThreads / 32) {
    // no role (the fused launch gives every CTA two more warps than the recurrence uses)
  } else if (warp == kTmaWarp) {
    // =========================== TMA producer ====================================
    if ((tid & 31) == 0) {
      int issued[kStages] = {0, 0, 0};
      bool ok = true;
      auto load = [&](int j) {
        const int st = j % kStages;
        const int64_t slot = si.slot0 + j;
        if (slot < 0 || slot >= p.slots) return;  // corrupt metadata: nothing to load
        const int32_t recr = static_cast<int32_t>(slot * p.H + h);
        if constexpr (kFused) {
          if (j >= p.fused_j0 && !wait_record(p, recr, budget)) {
            ok = false;
            return;
          }
        }
        uint8_t* base = sm + st * kStage;
        mbar_arrive_expect_tx(&full_bar[st], kStageTx);
        tma_load_2d(base + kWQ, &maps.wt, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kWQ + 16384, &maps.qg, &full_bar[st], 0, recr * 64);
        tma_load_2d(base + kWQ + 16384 + 8192, &maps.qg, &full_bar[st], 64, recr * 64);
        tma_load_2d(base + kUT, &maps.ut, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kKd, &maps.kd, &full_bar[st], 0, recr * 64);
        tma_load_2d(base + kKd + 8192, &maps.kd, &full_bar[st], 64, recr * 64);
        tma_load_2d(base + kAqk, &maps.aqk, &full_bar[st], 0, recr * 64);
        bulk_load(base + kGC, p.ws + p.lay.gc + static_cast<size_t>(recr) * kTileGC, 512,
                  &full_bar[st]);
        issued[st]++;
      };
      if (nch > 0) {
        prefetch_tmap(&maps.wt);
        prefetch_tmap(&maps.qg);
        prefetch_tmap(&maps.ut);
        prefetch_tmap(&maps.kd);
        prefetch_tmap(&maps.aqk);
      }
      for (int j = 0; j < nch && j < kStages && ok; ++j) load(j);
      for (int j = 0; j + kStages < nch && ok; ++j) {
        // stage j % kStages is free once every UMMA of chunk j has completed
        ok = mbar_wait_sleep(&empty_bar[j % kStages], (j / kStages) & 1, budget) && !*abort_flag;
        if (ok) load(j + kStages);
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.ws, kStatusTimeout);
      }
      // drain: every TMA load this thread issued completes before exit
      for (int st = 0; st < kStages; ++st)
        if (issued[st] > 0)
          mbar_wait(&full_bar[st], static_cast<uint32_t>((issued[st] - 1) & 1), drain_budget);
    }
  } else if (warp == kMmaWarp) {
    // =========================== UMMA issuer =====================================
    const bool lead = (tid & 31) == 0;
    const uint32_t id_p = idesc_f16(128, 64, kFmtF16, kKMajor, kMNMajor);
    const uint32_t id_q = idesc_f16(128, 64, kFmtF16, kKMajor, kKMajor);
    const uint32_t id_s = idesc_f16(128, 128, kFmtF16, kKMajor, kMNMajor);
    const uint32_t id_o = idesc_f16(128, 64, kFmtF16, kKMajor, kKMajor);
    const uint32_t tS0 = tbase + kColS0, tUd = tbase + kColUd;
    bool ok = true, issued = false;
    for (int j = 0; j < nch; ++j) {
      const int st = j % kStages;
      const int rg = j % kRegions;
      const uint32_t tP = tbase + region_col(j);
      const uint32_t bW = smem_u32(sm + st * kStage + kWQ);
      const uint32_t bKd = smem_u32(sm + st * kStage + kKd);
      const uint32_t bAq = smem_u32(sm + st * kStage + kAqk);
      ok = !named_bar_or(kBarS0, kChainThreads, !ok || *abort_flag);   // S0^T is in TMEM
      if (!ok) break;
      if (lead) {
        // the output warps must have drained this region (chunk j - 2)
        if (j >= kRegions)
          ok = mbar_wait(&ofree_bar[rg], ((j - kRegions) / kRegions) & 1, budget);
        if (ok) {
          tc_fence_after();
          // P_W^T = S0^T W^T (the chain needs it), then P_Q^T = S0^T (Q Gamma)^T
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ta(tP, tS0 + kk * 8, sdesc_sw128(bW + kk * 2048, 16384, 1024), id_p, kk > 0);
          umma_commit(&mma1_bar);
          issued = true;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_f16_ta(tP + 64, tS0 + kk * 8,
                        sdesc_sw128(bW + 16384 + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024), id_q,
                        kk > 0);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      ok = !named_bar_or(kBarUd, kChainThreads, !ok || *abort_flag);   // Ud^T and decayed S are in TMEM
      if (!ok) break;
      if (lead) {
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ta(tbase + kColS, tUd + kk * 8, sdesc_sw128(bKd + kk * 2048, 8192, 1024), id_s, 1);
        umma_commit(&sready_bar);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16_ta(tP + 64, tUd + kk * 8, sdesc_sw128(bAq + kk * 32, 16, 1024), id_o, 1);
        umma_commit(&oready_bar[rg]);
        umma_commit(&empty_bar[st]);
      }
      __syncwarp();
    }
    if (lead) {
      if (!ok) {
        *abort_flag = 1;
        record_status(p.ws, kStatusTimeout);
      }
      // drain: every UMMA this warp issued completes before the CTA frees TMEM
      if (issued) {
        umma_commit(&drain_bar);
        mbar_wait(&drain_bar, 0, drain_budget);
      }
    }
  } else if (warp >= kStateWarps) {
    // =========================== output warps ===================================
    // A full chunk leaves through the stage's [W^T | (Q Gamma)^T] tiles (dead once
    // [P_W | P_Q] has completed) as one TMA tile store; a partial chunk (the end of
    // a sequence, or a checkpoint boundary) uses plain stores so that nothing past
    // the chunk is written.  The stage is released once the store has read it.
    const int qw = warp - kStateWarps;
    const int v = qw * 32 + (tid & 31);
    const bool leader = (tid == kStateWarps * 32);
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32);
    const int64_t ostride = static_cast<int64_t>(p.H) * kD;
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int rg = j % kRegions;
      const int st = j % kStages;
      ok = mbar_wait(&oready_bar[rg], (j / kRegions) & 1, budget) && !*abort_flag;
      ok = !named_bar_or(kBarOutOr, kOutThreads, !ok);   // the same decision in every output thread
      if (!ok) break;
      tc_fence_after();
      int32_t t0, c;
      chunk_span(si, j, t0, c);
      uint32_t a[32], b[32];
      const uint32_t reg = region_col(j);
      tmem_ld32(tmem_addr(tbase, lane_base, reg + 64), a);
      tmem_ld32(tmem_addr(tbase, lane_base, reg + 96), b);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&ofree_bar[rg]);
      if (c == kC) {
        uint8_t* stile = sm + st * kStage + kWQ;   // O [64 tok][128 v] bf16
        uint16_t* so = reinterpret_cast<uint16_t*>(stile) + v;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          so[i * kD] = __bfloat16_as_ushort(__float2bfloat16_rn(p.scale * __uint_as_float(a[i])));
          so[(32 + i) * kD] = __bfloat16_as_ushort(__float2bfloat16_rn(p.scale * __uint_as_float(b[i])));
        }
        fence_proxy_async_smem();
        named_bar_sync(kBarOut, kOutThreads);
        if (leader) {
          tma_store_3d(&maps.o_out, stile, 0, h, si.start + t0);
          bulk_commit();
          bulk_wait_read();
          mbar_arrive(&empty_bar[st]);
        }
      } else {
        uint16_t* orow = p.out + (static_cast<int64_t>(si.start + t0) * p.H + h) * kD + v;
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i < c)
            orow[i * ostride] = __bfloat16_as_ushort(__float2bfloat16_rn(p.scale * __uint_as_float(a[i])));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (32 + i < c)
            orow[(32 + i) * ostride] =
                __bfloat16_as_ushort(__float2bfloat16_rn(p.scale * __uint_as_float(b[i])));
        }
        if (leader) mbar_arrive(&empty_bar[st]);
      }
    }
    if (leader) bulk_wait_all();   // every tile store of this CTA is complete
    if (!ok) {
      *abort_flag = 1;
      record_status(p.ws, kStatusTimeout);
    }
  } else {
    // =========================== state warps ====================================
    const int qw = warp & 3, hw = warp >> 2;   // lane quarter, half of the row
    const int v = qw * 32 + (tid & 31);        // TMEM lane = value channel
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32);
    float* ckc = (p.ckpt != nullptr) ? p.ckpt + nh * (kD * kD) + v : nullptr;
    // copy this thread's half row of S^T (columns k = 64 hw ..) to a state buffer
    auto store_state = [&](float* dst) {
      uint32_t a[32], b[32];
      tmem_ld32(tmem_addr(tbase, lane_base, kColS + hw * 64), a);
      tmem_ld32(tmem_addr(tbase, lane_base, kColS + hw * 64 + 32), b);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        dst[(hw * 64 + i) * kD] = __uint_as_float(a[i]);
        dst[(hw * 64 + 32 + i) * kD] = __uint_as_float(b[i]);
      }
    };
    // initial state: S^T[v][64 hw .. 64 hw + 63] = h0[k][v]
    {
      const float* h0c = p.h0 ? p.h0 + nh * (kD * kD) + v : nullptr;
#pragma unroll
      for (int kc = 0; kc < 2; ++kc) {
        uint32_t r[32];
        const int k0 = hw * 64 + kc * 32;
        // all loads first: a checkpoint store between them (a buffer the compiler cannot
        // prove apart from h0) would make every load wait for the previous one
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(h0c ? h0c[(k0 + i) * kD] : 0.f);
        if (ckc && si.ck == 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) ckc[(k0 + i) * kD] = __uint_as_float(r[i]);
        }
        tmem_st32(tmem_addr(tbase, lane_base, kColS + k0), r);
      }
      tmem_wait_st();
    }
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int st = j % kStages;
      const uint8_t* stg = sm + st * kStage;
      ok = ok && mbar_wait(&full_bar[st], (j / kStages) & 1, budget) && !*abort_flag;
      if (ok && j > 0) ok = mbar_wait(&sready_bar, (j - 1) & 1, budget) && !*abort_flag;
      tc_fence_after();
      uint32_t a[32], b[32];
      if (ok) {
        // checkpoint: the state after the chunk that ends at the offset
        if (ckc && si.nA > 0 && j == si.nA) store_state(ckc);
        // (b) S0^T half row -> f16 A operand in TMEM (FP16: 2^-11 rounding; the state
        // stays far inside the FP16 range for the inputs the header admits)
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + hw * 64), a);
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + hw * 64 + 32), b);
        tmem_wait_ld();
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_f16(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
        tmem_st16(tmem_addr(tbase, lane_base, kColS0 + hw * 32), pk);
#pragma unroll
        for (int i = 0; i < 16; ++i) pk[i] = pack_f16(__uint_as_float(b[2 * i]), __uint_as_float(b[2 * i + 1]));
        tmem_st16(tmem_addr(tbase, lane_base, kColS0 + hw * 32 + 16), pk);
        tmem_wait_st();
      }
      tc_fence_before();
      ok = !named_bar_or(kBarS0, kChainThreads, !ok);
      if (!ok) break;
      // the S half row scaled by Gamma_end goes back to TMEM while [P_W | P_Q]
      // runs (the update that accumulates onto it is issued after the next barrier)
      {
        const float4* gc4 = reinterpret_cast<const float4*>(stg + kGC) + hw * 16;
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4) {
          const float4 ga = gc4[i4], gb = gc4[8 + i4];
          a[4 * i4 + 0] = __float_as_uint(__uint_as_float(a[4 * i4 + 0]) * ga.x);
          a[4 * i4 + 1] = __float_as_uint(__uint_as_float(a[4 * i4 + 1]) * ga.y);
          a[4 * i4 + 2] = __float_as_uint(__uint_as_float(a[4 * i4 + 2]) * ga.z);
          a[4 * i4 + 3] = __float_as_uint(__uint_as_float(a[4 * i4 + 3]) * ga.w);
          b[4 * i4 + 0] = __float_as_uint(__uint_as_float(b[4 * i4 + 0]) * gb.x);
          b[4 * i4 + 1] = __float_as_uint(__uint_as_float(b[4 * i4 + 1]) * gb.y);
          b[4 * i4 + 2] = __float_as_uint(__uint_as_float(b[4 * i4 + 2]) * gb.z);
          b[4 * i4 + 3] = __float_as_uint(__uint_as_float(b[4 * i4 + 3]) * gb.w);
        }
        tmem_st32(tmem_addr(tbase, lane_base, kColS + hw * 64), a);
        tmem_st32(tmem_addr(tbase, lane_base, kColS + hw * 64 + 32), b);
      }
      // (e) Ud^T = U^T - P_W^T (tokens 32 hw .. 32 hw + 31) -> f16 A operand in TMEM
      ok = mbar_wait(&mma1_bar, j & 1, budget) && !*abort_flag;
      tc_fence_after();
      if (ok) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tbase, lane_base, region_col(j) + hw * 32), r);
        tmem_wait_ld();
        const uint8_t* ut = stg + kUT;
        uint32_t ud[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 uq = *reinterpret_cast<const uint4*>(ut + sw128_offset(v, hw * 4 + q));
          const uint32_t uw[4] = {uq.x, uq.y, uq.z, uq.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 uf = __half22float2(*reinterpret_cast<const __half2*>(&uw[e]));
            ud[q * 4 + e] = pack_f16(uf.x - __uint_as_float(r[q * 8 + 2 * e]),
                                     uf.y - __uint_as_float(r[q * 8 + 2 * e + 1]));
          }
        }
        tmem_st16(tmem_addr(tbase, lane_base, kColUd + hw * 16), ud);
      }
      tmem_wait_st();   // Ud^T and the decayed S row are in TMEM
      tc_fence_before();
      ok = !named_bar_or(kBarUd, kChainThreads, !ok);
      if (!ok) break;
    }
    if (ok && nch > 0) ok = mbar_wait(&sready_bar, (nch - 1) & 1, budget) && !*abort_flag;
    if (!ok) {
      *abort_flag = 1;
      record_status(p.ws, kStatusTimeout);
    } else {
      tc_fence_after();
      if (p.ht != nullptr) store_state(p.ht + nh * (kD * kD) + v);
      if (ckc && nch > 0 && si.ck == si.len) store_state(ckc);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace kda
