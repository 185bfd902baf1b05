// kda_recurrence.cu — inter-chunk recurrence with the fused output (split variant).
//
// One CTA per (sequence, head); the chunks of the sequence are walked in order
// (north star subsystems (b) "an inter-chunk recurrence kernel that carries S
// in TMEM/registers across chunks via tcgen05 GEMMs fed by TMA" and (c) "an
// output kernel fusing the intra-chunk causal term with q.S").  The state is
// kept transposed, S^T[v][k], in TMEM lanes v = 0..127, so every UMMA has M = 128:
//   P^T  = S0^T [W | Q*Gamma]^T                (M=128, N=128, K=128; bf16)
//   Ud^T = U^T - P^T[:, 0:64]                   (threads; f16 operand)
//   S^T  = S0^T Diag(Gamma_end) + Ud^T Kd       (M=128, N=128, K=64;  f16)
//   O^T  = scale (P^T[:, 64:128] + Ud^T Aqk^T)  (M=128, N=64,  K=64;  f16)
//   C^T  = S0^T Diag(Gamma_p) + Ud^T Kp         (checkpoint chunk only)
// Warp roles: warps 0-3 own TMEM lanes 0-127 (one state row each); warp 4
// lane 0 issues the TMA ring (2 stages) and every UMMA.
// In-place state update (ht == h0) is safe: each thread reads its whole h0
// column before any thread of any CTA writes ht, and a (sequence, head) pair
// is owned by exactly one CTA (FlashInfer PR #4262 "Physical schedules and
// true in-place state update" describes the same ownership rule).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace rec {
constexpr uint32_t kWQ = 0;          // 32 KB [W^T | (Q Gamma)^T] MN-major B, 2 panels [128 k][64]
constexpr uint32_t kUT = 32768;      // 16 KB U^T  [128 v][64 tok] f16 (128B swizzle)
constexpr uint32_t kKd = 49152;      // 16 KB Kd^T [128 k][64 tok] f16, K-major B
constexpr uint32_t kAqk = 65536;     //  8 KB Aqk  [64 r][64 s] f16, K-major B
constexpr uint32_t kGC = 73728;      // 512 B Gamma_end f32 [128]
constexpr uint32_t kStage = 74752;
constexpr uint32_t kS0T = 2 * kStage;        // 32 KB S0^T bf16, K-major A, 2 panels [128 v][64 k]
constexpr uint32_t kUdT = kS0T + 32768;      // 16 KB Ud^T f16, K-major A [128 v][64 tok]
constexpr uint32_t kKp = kUdT + 16384;       // 16 KB Kp^T f16 (checkpoint chunk)
constexpr uint32_t kGP = kKp + 16384;        // 512 B Gamma_p f32 [128]
constexpr uint32_t kBytes = kGP + 512;
constexpr uint32_t kSmemAlloc = kBytes + 1024;
constexpr uint32_t kStageTx = 32768 + 16384 + 16384 + 8192 + 512;
constexpr uint32_t kColS = 0, kColP = 128, kColO = 192, kColC = 256;
constexpr int kThreads = 160;
extern const uint32_t kSmemAllocBytes = kSmemAlloc;
}  // namespace rec

__global__ void __launch_bounds__(rec::kThreads, 1)
kda_recurrence_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  using namespace rec;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full_bar[2], empty_bar[2], s0_bar, ud_bar, mma1_bar, mma2_bar, ck_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int32_t s_abort;
  volatile int32_t* abort_flag = &s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int unit = blockIdx.x;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;
  const int h = unit % p.H;
  int32_t n = unit / p.H;
  if (p.cu_seqlens != nullptr)
    n = reinterpret_cast<const int32_t*>(p.ws + p.lay.seq_order)[n];
  if (n < 0 || n >= p.N) return;
  const SeqInfo si = seq_info(p, n);
  const int32_t nch = (si.len + kC - 1) / kC;
  int32_t cp_off = -1, cj = -1;
  if (p.ckpt_offsets != nullptr) {
    cp_off = min(max(p.ckpt_offsets[n], 0), si.len);
    cj = cp_off >= 1 ? (cp_off - 1) / kC : -1;
  }
  const int64_t nh = static_cast<int64_t>(n) * p.H + h;
  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full_bar[i], 1);
      mbar_init(&empty_bar[i], 1);
    }
    mbar_init(&s0_bar, 128);
    mbar_init(&ud_bar, 128);
    mbar_init(&mma1_bar, 1);
    mbar_init(&mma2_bar, 1);
    mbar_init(&ck_bar, 1);
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

  if (warp == 4) {
    // =========================== producer + MMA issuer =========================
    if ((tid & 31) == 0) {
      int issued[2] = {0, 0};
      uint64_t* last_commit = nullptr;
      uint32_t last_parity = 0;
      bool ck_issued = false;
      auto load = [&](int j) {
        const int st = j & 1;
        const int64_t slot = si.slot0 + j;
        if (slot < 0 || slot >= p.slots) return;  // corrupt metadata: nothing to load
        const int32_t recr = static_cast<int32_t>(slot * p.H + h);
        uint8_t* base = sm + st * kStage;
        mbar_arrive_expect_tx(&full_bar[st], kStageTx);
        tma_load_2d(base + kWQ, &maps.wt, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kWQ + 16384, &maps.qgt, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kUT, &maps.ut, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kKd, &maps.kdt, &full_bar[st], 0, recr * 128);
        tma_load_2d(base + kAqk, &maps.aqk, &full_bar[st], 0, recr * 64);
        bulk_load(base + kGC, p.ws + p.lay.gc + static_cast<size_t>(recr) * kTileGC, 512,
                  &full_bar[st]);
        issued[st]++;
      };
      if (nch > 0) {
        prefetch_tmap(&maps.wt);
        prefetch_tmap(&maps.qgt);
        prefetch_tmap(&maps.ut);
        prefetch_tmap(&maps.kdt);
        prefetch_tmap(&maps.aqk);
      }
      if (cj >= 0 && cj < nch) {
        mbar_arrive_expect_tx(&ck_bar, 16384 + 512);
        tma_load_2d(sm + kKp, &maps.kpt, &ck_bar, 0, static_cast<int32_t>(nh * 128));
        bulk_load(sm + kGP, p.ws + p.lay.gp + nh * kTileGC, 512, &ck_bar);
        ck_issued = true;
      }
      for (int j = 0; j < nch && j < 2; ++j) load(j);
      const uint32_t id_p = idesc_f16(128, 128, kFmtBF16, kKMajor, kMNMajor);
      const uint32_t id_s = idesc_f16(128, 128, kFmtF16, kKMajor, kKMajor);
      const uint32_t id_o = idesc_f16(128, 64, kFmtF16, kKMajor, kKMajor);
      const uint32_t aS0 = smem_u32(sm + kS0T), aUd = smem_u32(sm + kUdT);
      bool ok = true;
      bool ck_seen = false;
      for (int j = 0; j < nch && ok; ++j) {
        const int st = j & 1;
        const uint32_t bWQ = smem_u32(sm + st * kStage + kWQ);
        const uint32_t bKd = smem_u32(sm + st * kStage + kKd);
        const uint32_t bAq = smem_u32(sm + st * kStage + kAqk);
        ok = mbar_wait(&s0_bar, j & 1, budget) && !*abort_flag;
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16(tbase + kColP, sdesc_sw128(aS0 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(bWQ + kk * 2048, 16384, 1024), id_p, kk > 0);
        umma_commit(&mma1_bar);
        last_commit = &mma1_bar;
        last_parity = j & 1;
        ok = mbar_wait(&ud_bar, j & 1, budget) && !*abort_flag;
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tbase + kColS, sdesc_sw128(aUd + kk * 32, 16, 1024),
                   sdesc_sw128(bKd + kk * 32, 16, 1024), id_s, 1);
        if (j == cj) {
          if (!ck_seen) {
            ck_seen = mbar_wait(&ck_bar, 0, budget);
            if (!ck_seen) { ok = false; }
          }
          if (ok) {
            const uint32_t bKp = smem_u32(sm + kKp);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_f16(tbase + kColC, sdesc_sw128(aUd + kk * 32, 16, 1024),
                       sdesc_sw128(bKp + kk * 32, 16, 1024), id_s, 1);
          }
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_f16(tbase + kColO, sdesc_sw128(aUd + kk * 32, 16, 1024),
                   sdesc_sw128(bAq + kk * 32, 16, 1024), id_o, 1);
        umma_commit(&mma2_bar);
        umma_commit(&empty_bar[st]);
        last_commit = &empty_bar[st];
        last_parity = (j >> 1) & 1;
        if (!ok) break;
        if (j + 2 < nch) {
          ok = mbar_wait(&empty_bar[st], (j >> 1) & 1, budget);
          if (!ok) break;
          load(j + 2);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(p.ws, kStatusTimeout);
      }
      // drain: every TMA load and UMMA this thread issued completes before exit
      for (int st = 0; st < 2; ++st)
        if (issued[st] > 0)
          mbar_wait(&full_bar[st], static_cast<uint32_t>((issued[st] - 1) & 1), drain_budget);
      if (ck_issued) mbar_wait(&ck_bar, 0, drain_budget);
      if (last_commit) mbar_wait(last_commit, last_parity, drain_budget);
    }
  } else {
    // =========================== state warps (lane v = tid) =====================
    const int v = tid;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32);
    // initial state column v of S = row v of S^T
    {
      const float* h0c = p.h0 ? p.h0 + nh * (kD * kD) + v : nullptr;
      float* ckc = (p.ckpt != nullptr && cp_off == 0) ? p.ckpt + nh * (kD * kD) + v : nullptr;
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        uint32_t r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = h0c ? h0c[(kc * 32 + i) * kD] : 0.f;
          r[i] = __float_as_uint(x);
          if (ckc) ckc[(kc * 32 + i) * kD] = x;
        }
        tmem_st32(tmem_addr(tbase, lane_base, kColS + kc * 32), r);
      }
      tmem_wait_st();
    }
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      const int st = j & 1;
      const uint8_t* stg = sm + st * kStage;
      const int32_t t0 = si.start + j * kC;
      const int32_t c = min(kC, si.len - j * kC);
      ok = mbar_wait(&full_bar[st], (j >> 1) & 1, budget) && !*abort_flag;
      if (!ok) break;
      tc_fence_after();
      // (b) S0^T row -> bf16 A operand; S row scaled by Gamma_end (and Gamma_p) back to TMEM
      const float* gcs = reinterpret_cast<const float*>(stg + kGC);
      const float* gps = reinterpret_cast<const float*>(sm + kGP);
      const bool ckj = (j == cj);
      if (ckj) {
        ok = mbar_wait(&ck_bar, 0, budget) && !*abort_flag;
        if (!ok) break;
      }
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + kc * 32), r);
        tmem_wait_ld();
        uint8_t* a_row = sm + kS0T + (kc >> 1) * 16384;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4 o;
          o.x = pack_bf16(__uint_as_float(r[q * 8 + 0]), __uint_as_float(r[q * 8 + 1]));
          o.y = pack_bf16(__uint_as_float(r[q * 8 + 2]), __uint_as_float(r[q * 8 + 3]));
          o.z = pack_bf16(__uint_as_float(r[q * 8 + 4]), __uint_as_float(r[q * 8 + 5]));
          o.w = pack_bf16(__uint_as_float(r[q * 8 + 6]), __uint_as_float(r[q * 8 + 7]));
          *reinterpret_cast<uint4*>(a_row + sw128_offset(v, (kc & 1) * 4 + q)) = o;
        }
        if (ckj) {
          uint32_t cr[32];
#pragma unroll
          for (int i = 0; i < 32; ++i)
            cr[i] = __float_as_uint(__uint_as_float(r[i]) * gps[kc * 32 + i]);
          tmem_st32(tmem_addr(tbase, lane_base, kColC + kc * 32), cr);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * gcs[kc * 32 + i]);
        tmem_st32(tmem_addr(tbase, lane_base, kColS + kc * 32), r);
      }
      tmem_wait_st();
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&s0_bar);
      // (e) Ud^T = U^T - P^T[:, 0:64] -> f16 A operand
      ok = mbar_wait(&mma1_bar, j & 1, budget) && !*abort_flag;
      if (!ok) break;
      tc_fence_after();
      {
        const uint8_t* ut = stg + kUT;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, lane_base, kColP + half * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int chunk = half * 4 + q;
            const uint4 uu = *reinterpret_cast<const uint4*>(ut + sw128_offset(v, chunk));
            const uint32_t uw[4] = {uu.x, uu.y, uu.z, uu.w};
            uint32_t ow[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __half2 u2 = *reinterpret_cast<const __half2*>(&uw[e]);
              const float2 uf = __half22float2(u2);
              ow[e] = pack_f16(uf.x - __uint_as_float(r[q * 8 + 2 * e]),
                               uf.y - __uint_as_float(r[q * 8 + 2 * e + 1]));
            }
            *reinterpret_cast<uint4*>(sm + kUdT + sw128_offset(v, chunk)) =
                make_uint4(ow[0], ow[1], ow[2], ow[3]);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&ud_bar);
      // (g) output rows and the checkpoint state
      ok = mbar_wait(&mma2_bar, j & 1, budget) && !*abort_flag;
      if (!ok) break;
      tc_fence_after();
      {
        uint16_t* orow = p.out + (static_cast<int64_t>(t0) * p.H + h) * kD + v;
        const int64_t ostride = static_cast<int64_t>(p.H) * kD;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, lane_base, kColO + half * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int rr = half * 32 + i;
            if (rr < c)
              orow[rr * ostride] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(p.scale * __uint_as_float(r[i])));
          }
        }
      }
      if (ckj) {
        float* ckc = p.ckpt + nh * (kD * kD) + v;
#pragma unroll
        for (int kc = 0; kc < 4; ++kc) {
          uint32_t r[32];
          tmem_ld32(tmem_addr(tbase, lane_base, kColC + kc * 32), r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) ckc[(kc * 32 + i) * kD] = __uint_as_float(r[i]);
        }
      }
      tc_fence_before();
    }
    if (!ok) {
      *abort_flag = 1;
      record_status(p.ws, kStatusTimeout);
    } else if (p.ht != nullptr) {
      float* htc = p.ht + nh * (kD * kD) + v;
#pragma unroll
      for (int kc = 0; kc < 4; ++kc) {
        uint32_t r[32];
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + kc * 32), r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) htc[(kc * 32 + i) * kD] = __uint_as_float(r[i]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 512);
}

}  // namespace kda
