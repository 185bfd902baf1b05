// kda_chain.cuh — the inter-chunk recurrence of the stream variant (256 threads per
// (sequence, head), half of a CTA whose other half runs a prepare group on the same
// SM: 256 tensor-memory columns and 104 KB of shared memory).
//
// The state S [k][v] (key channel k on TMEM lane k, value channel v on column v)
// stays in tensor memory from chunk to chunk.  Per chunk of c <= 64 tokens, with the
// records the prepare CTAs made for it (W and Q Gamma as token rows, U, Kd, Aqk,
// Gamma_end), the recurrence of the chunked form is
//   [P_Q; P_W] = [Q Gamma; W] S0             (one UMMA: M = 128 rows r', N = 128 v, K = 128 k)
//   Ud         = U - P_W                     (threads; FP16, into shared memory)
//   S1         = Diag(Gamma_end) S0 + Kd^T Ud  (threads scale S row k by Gamma_end[k];
//                                               then one UMMA: M = 128 k, N = 128 v, K = 64 r)
//   O          = scale (P_Q + Aqk Ud)        (one UMMA accumulating onto P_Q: M = 128, K = 64)
// S0 is S rounded to FP16 for the tensor core (FP32 S stays in tensor memory).  The
// same algebra as the split variant's recurrence; only the orientation differs, so
// that every operand is either in shared memory already or written there by the
// threads that own its rows: S0 [k][v] and Ud [r][v] are MN-major B operands, and
// [Q Gamma; W] is the K-major A operand of the first product.
//
// Tensor memory (256 columns):
//   [0, 128)    S  f32 (lane k, column v)
//   [128, 256)  PQ f32: lanes 0..63 P_Q, then O (rows r of the chunk); lanes 64..127 P_W
//
// Threads: warp w serves TMEM lanes 32 (w % 4) .. + 31 and value columns 64 (w / 4)
// .. + 63, so thread (L = lane, h = w / 4) owns S row L, and PQ row L, on that column
// half.  Warps 0, 1, 4, 5 (PQ lanes 0..63) drain and store the output; warps 2, 3, 6, 7
// (PQ lanes 64..127) form Ud.  Thread 64 (warp 2, lane 0) issues every UMMA; thread 32
// (warp 1, lane 0) acquires the records' ready flags and issues their TMA copies.
//
// Per chunk j: [B] every thread waits for S(j) (the previous update), loads its S row
// half, writes S0 into shared memory and the Gamma-scaled S back into tensor memory;
// the output warps also drain and store O(j - 1).  [C] barrier of the 256 threads; the
// issuer starts P; the Ud warps load their U rows of chunk j.  [D] the Ud warps wait
// for P and write Ud; the producer brings chunk j + 1's A tile and acquires record
// j + 2 (two chunks ahead, off the chain).  [E] barrier of the Ud warps; the issuer
// starts the update and O, with separate commits for S and for O.  No register array
// lives across a barrier (spilled registers would put L2 round trips on the chain).
// Every wait is bounded; a failure is ORed across each barrier's participants
// (bar.red.or) so that all of them leave together.
//
// The records are consumed from L2 soon after the prepare CTAs of the same launch made
// them.  Once a record has been read it is dropped from L2 without a write-back
// (discard.global.L2), so the records never cost DRAM bandwidth.
//
// In-place state update (ht == h0) is safe: each thread reads its part of the h0
// rows before writing the same part of ht, and a (sequence, head) pair is owned by
// exactly one CTA (FlashInfer PR #4262 "Physical schedules and true in-place state
// update" describes the same ownership rule).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace chain {
constexpr int kThreads = 256;
constexpr uint32_t kA = 0;          // 32 KB [Q Gamma; W] f16, K-major A of P: 2 panels [128 rows][64 k]
constexpr uint32_t kAqk = 32768;    //  8 KB Aqk [64 r][64 s] f16, K-major A of O (its rows 64..127 read
                                    //        the Kd tile after it, only into PQ lanes no one reads)
constexpr uint32_t kKd = 40960;     // 16 KB Kd [64 r][128 k] f16, MN-major A of the update: 2 panels [64 r][64 k]
constexpr uint32_t kS0 = 57344;     // 32 KB S0 [128 k][128 v] f16, MN-major B of P: 2 panels [128 k][64 v]
constexpr uint32_t kUd = 90112;     // 16 KB U, then Ud = U - P_W in place: [64 r][128 v] f16,
                                    //        MN-major B of the update and O: 2 panels [64 r][64 v]
constexpr uint32_t kBytes = 106496;
constexpr uint32_t kSmemAlloc = kBytes + 1024;
constexpr uint32_t kTxA = 32768, kTxY = 16384 + 8192 + 16384;
constexpr uint32_t kColS = 0, kColPQ = 128;
constexpr int kIssuer = 64;         // warp 2, lane 0
constexpr int kProducer = 32;       // warp 1, lane 0: record flags, A tiles
constexpr int kLoaderY = 96;        // warp 3, lane 0: Kd / Aqk / U tiles
constexpr uint32_t kBarAll = 1, kBarUd = 2;   // named barriers (ids 1, 2)
static_assert(kUd + 16384 == kBytes && kKd + 16384 == kS0, "layout");
}  // namespace chain

// Drop a consumed record's lines from L2 without writing them back (128-byte lines;
// `bytes` a multiple of 128, `base` 128-byte aligned).
__device__ __forceinline__ void discard_l2(const uint8_t* base, uint32_t bytes, int tid, int nthreads) {
  for (uint32_t off = static_cast<uint32_t>(tid) * 128u; off < bytes; off += 128u * nthreads)
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(base + off) : "memory");
}

// Loads of record data written earlier in the same launch by other CTAs: L2 only (the
// L1 of this SM is not coherent with their stores).
__device__ __forceinline__ uint4 ldg_cg_v4(const void* p) {
  uint4 r;
  asm volatile("ld.global.cg.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
__device__ __forceinline__ float ldg_cg_f32(const float* p) {
  float r;
  asm volatile("ld.global.cg.f32 %0, [%1];" : "=f"(r) : "l"(p));
  return r;
}

// Acquire the ready flag of a record written by a prepare CTA of the same launch
// (bounded poll); the caller orders its later TMA reads with fence.proxy.async and the
// other threads' reads with a CTA barrier.
__device__ __forceinline__ bool acquire_record(const KdaParams& p, int64_t rec, long long budget) {
  if (budget < 0) return false;
  const int32_t* flag = reinterpret_cast<const int32_t*>(p.ws + p.lay.ready) + rec;
  const long long t0 = clock64();
  for (;;) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (clock64() - t0 > budget) return false;
    __nanosleep(32);
  }
}

// The recurrence of one (sequence, head) unit of the stream variant, run by threads
// 0..255 of the CTA.  tbase: 256 tensor-memory columns of the caller's allocation.
__device__ __forceinline__ void chain_body(const KdaParams& p, const SplitMaps& maps,
                                           uint8_t* smem_raw, int unit, uint32_t tbase) {
  using namespace chain;
  uint8_t* sm = smem_align<1024>(smem_raw);
  __shared__ uint64_t fullA_bar, fullY_bar, p_bar, s_bar, o_bar, drain_bar;
  __shared__ int32_t s_abort;
  volatile int32_t* abort_flag = &s_abort;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;
  const int hd = unit % p.H;
  int32_t n = unit / p.H;
  if (p.cu_seqlens != nullptr) n = reinterpret_cast<const int32_t*>(p.ws + p.lay.seq_order)[n];
  if (n < 0 || n >= p.N) return;
  const SeqInfo si = seq_info(p, n);
  const int32_t nch = si.nch;
  const int64_t nh = static_cast<int64_t>(n) * p.H + hd;
  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;

  const int qtr = warp & 3, half = warp >> 2;
  const int L = qtr * 32 + lane;                       // TMEM lane: S row k, PQ row r'
  const uint32_t lane_base = static_cast<uint32_t>(qtr * 32);
  const bool out_warp = qtr < 2;                       // PQ lanes 0..63: output rows
  const int v0 = half * 64;                            // this thread's value columns
  const int oi = half * 64 + qtr * 32 + lane;          // index among the 128 output threads

  if (tid == 0) {
    mbar_init(&fullA_bar, 1);
    mbar_init(&fullY_bar, 1);
    mbar_init(&p_bar, 1);
    mbar_init(&s_bar, 1);
    mbar_init(&o_bar, 1);
    mbar_init(&drain_bar, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  named_bar_sync(kBarAll, kThreads);
  const uint32_t sbase = smem_u32(sm);

  auto rec_of = [&](int j) -> int64_t {   // record index of chunk j, or -1 if out of range
    const int64_t slot = si.slot0 + j;
    if (slot < 0 || slot >= p.slots) return -1;
    return slot * p.H + hd;
  };
  // producer: acquire a record's ready flag; TMA of a chunk's A tile and of its Kd / Aqk
  int issuedA = 0, issuedY = 0;
  auto acquire = [&](int j) -> bool {
    if (j >= nch) return true;
    const int64_t r = rec_of(j);
    if (r < 0) return true;
    if (!acquire_record(p, r, budget)) return false;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    return true;
  };
  auto load_A = [&](int j) {
    const int64_t r = rec_of(j);
    if (r < 0) return;
    mbar_arrive_expect_tx(&fullA_bar, kTxA);
    tma_load_2d(sm + kA, &maps.qw, &fullA_bar, 0, static_cast<int32_t>(r * 128));
    tma_load_2d(sm + kA + 16384, &maps.qw, &fullA_bar, 64, static_cast<int32_t>(r * 128));
    ++issuedA;
  };
  auto load_Y = [&](int j) {   // (the loader thread; the record was acquired by the producer)
    const int64_t r = rec_of(j);
    if (r < 0) return;
    asm volatile("fence.proxy.async.global;" ::: "memory");
    mbar_arrive_expect_tx(&fullY_bar, kTxY);
    tma_load_2d(sm + kKd, &maps.kd, &fullY_bar, 0, static_cast<int32_t>(r * 64));
    tma_load_2d(sm + kKd + 8192, &maps.kd, &fullY_bar, 64, static_cast<int32_t>(r * 64));
    tma_load_2d(sm + kAqk, &maps.aqk, &fullY_bar, 0, static_cast<int32_t>(r * 64));
    tma_load_2d(sm + kUd, &maps.u, &fullY_bar, 0, static_cast<int32_t>(r * 64));
    tma_load_2d(sm + kUd + 8192, &maps.u, &fullY_bar, 64, static_cast<int32_t>(r * 64));
    ++issuedY;
  };
  auto load_gamma = [&](int j) -> float {   // Gamma_end[L] of chunk j
    const int64_t r = rec_of(j);
    return r < 0 ? 1.f
                 : ldg_cg_f32(reinterpret_cast<const float*>(p.ws + p.lay.gc + static_cast<size_t>(r) * kTileGC) + L);
  };
  auto discard_record = [&](int j) {        // the 128 output threads drop a read record from L2
    const int64_t rp = rec_of(j);
    if (rp < 0) return;
    discard_l2(p.ws + p.lay.qw + static_cast<size_t>(rp) * kTileQW, static_cast<uint32_t>(kTileQW), oi, 128);
    discard_l2(p.ws + p.lay.u + static_cast<size_t>(rp) * kTileU, static_cast<uint32_t>(kTileU), oi, 128);
    discard_l2(p.ws + p.lay.kd + static_cast<size_t>(rp) * kTileKd, static_cast<uint32_t>(kTileKd), oi, 128);
    discard_l2(p.ws + p.lay.aqk + static_cast<size_t>(rp) * kTileAqk, static_cast<uint32_t>(kTileAqk), oi, 128);
  };
  // an output thread's O row half: scale, round to BF16, store (rows past the chunk skipped)
  auto drain_out = [&](int32_t ot0, int32_t oc) {
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      uint32_t a[32];
      tmem_ld32(tmem_addr(tbase, lane_base, kColPQ + v0 + part * 32), a);
      tmem_wait_ld();
      if (L < oc) {
        uint4* dst = reinterpret_cast<uint4*>(
            p.out + (static_cast<int64_t>(si.start + ot0 + L) * p.H + hd) * kD + v0 + part * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[i] = make_uint4(pack_bf16(p.scale * __uint_as_float(a[8 * i]), p.scale * __uint_as_float(a[8 * i + 1])),
                              pack_bf16(p.scale * __uint_as_float(a[8 * i + 2]), p.scale * __uint_as_float(a[8 * i + 3])),
                              pack_bf16(p.scale * __uint_as_float(a[8 * i + 4]), p.scale * __uint_as_float(a[8 * i + 5])),
                              pack_bf16(p.scale * __uint_as_float(a[8 * i + 6]), p.scale * __uint_as_float(a[8 * i + 7])));
      }
    }
  };

  // producer: records 0 and 1 ready, chunk 0's tiles on their way
  bool ok = true;
  if (tid == kProducer && nch > 0) {
    prefetch_tmap(&maps.qw);
    ok = acquire(0);
    if (ok) {
      load_A(0);
      ok = acquire(1);
    }
  }

  // ---- initial state: S[k = L][v0 .. v0 + 63] = h0 row (or 0); checkpoint at p = 0
  float* ckr = (p.ckpt != nullptr) ? p.ckpt + nh * (kD * kD) + L * kD + v0 : nullptr;
  {
    const float* h0r = p.h0 ? p.h0 + nh * (kD * kD) + L * kD + v0 : nullptr;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      uint32_t r[32];
      // all loads first (a checkpoint store between them would serialise them)
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (h0r) x = *reinterpret_cast<const float4*>(h0r + part * 32 + i4 * 4);
        r[4 * i4 + 0] = __float_as_uint(x.x);
        r[4 * i4 + 1] = __float_as_uint(x.y);
        r[4 * i4 + 2] = __float_as_uint(x.z);
        r[4 * i4 + 3] = __float_as_uint(x.w);
      }
      if (ckr && si.ck == 0) {
#pragma unroll
        for (int i4 = 0; i4 < 8; ++i4)
          *reinterpret_cast<float4*>(ckr + part * 32 + i4 * 4) =
              make_float4(__uint_as_float(r[4 * i4]), __uint_as_float(r[4 * i4 + 1]),
                          __uint_as_float(r[4 * i4 + 2]), __uint_as_float(r[4 * i4 + 3]));
      }
      tmem_st32(tmem_addr(tbase, lane_base, kColS + v0 + part * 32), r);
    }
    tmem_wait_st();
  }

  // records 0 and 1 are visible to every thread after this barrier
  ok = !named_bar_or(kBarAll, kThreads, !ok);
  float gam = 1.f, gam_next = 1.f;   // Gamma_end[k = L] of the current / next chunk
  if (ok && nch > 0) {
    gam_next = load_gamma(0);
    if (tid == kLoaderY) {
      prefetch_tmap(&maps.kd);
      prefetch_tmap(&maps.aqk);
      prefetch_tmap(&maps.u);
      load_Y(0);
    }
  }
  int32_t o_t0 = 0, o_c = 0;          // token span of the chunk whose O is in PQ

  for (int j = 0; j < nch && ok; ++j) {
    int32_t t0, c;
    chunk_span(si, j, t0, c);
    // ===== [B] S(j) ready: S0 into shared memory, Gamma-scaled S back to TMEM
    gam = gam_next;
    if (j > 0) ok = mbar_wait(&s_bar, static_cast<uint32_t>((j - 1) & 1), budget) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);   // tcgen05.ld / st below are warp-collective
    tc_fence_after();
    if (ok) {
      const uint32_t srow = sbase + kS0 + static_cast<uint32_t>(half) * 16384u;
      const bool ck_here = ckr && si.nA > 0 && j == si.nA;
      // (one part at a time: unrolled, the two parts' 64 live values spill)
#pragma unroll 1
      for (int part = 0; part < 2; ++part) {
        uint32_t a[32];
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + v0 + part * 32), a);
        tmem_wait_ld();
        // checkpoint: the state after the chunk that ends at the offset
        if (ck_here) {
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4)
            *reinterpret_cast<float4*>(ckr + part * 32 + i4 * 4) =
                make_float4(__uint_as_float(a[4 * i4]), __uint_as_float(a[4 * i4 + 1]),
                            __uint_as_float(a[4 * i4 + 2]), __uint_as_float(a[4 * i4 + 3]));
        }
        // S0 row k = L, panel `half` (128 B, 128-byte swizzle): 16-byte chunks of 8 values
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          const uint32_t* x = &a[c4 * 8];
          asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(
                           srow + sw128_offset(static_cast<uint32_t>(L), static_cast<uint32_t>(part * 4 + c4))),
                       "r"(pack_f16(__uint_as_float(x[0]), __uint_as_float(x[1]))),
                       "r"(pack_f16(__uint_as_float(x[2]), __uint_as_float(x[3]))),
                       "r"(pack_f16(__uint_as_float(x[4]), __uint_as_float(x[5]))),
                       "r"(pack_f16(__uint_as_float(x[6]), __uint_as_float(x[7])))
                       : "memory");
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = __float_as_uint(__uint_as_float(a[i]) * gam);
        tmem_st32(tmem_addr(tbase, lane_base, kColS + v0 + part * 32), a);
      }
    }
    // update and O of chunk j - 1 complete: the output warps drain and store O(j - 1)
    // (PQ lanes 0..63) before P(j) overwrites it, and a Ud-warp thread (whose warps
    // would otherwise wait at the barrier) brings chunk j's Kd / Aqk / U tiles
    if (j > 0 && (out_warp || tid == kLoaderY)) {
      ok = ok && mbar_wait(&o_bar, static_cast<uint32_t>((j - 1) & 1), budget) && !*abort_flag;
      if (ok && tid == kLoaderY) load_Y(j);
    }
    if (out_warp && j > 0) {
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) drain_out(o_t0, o_c);
    }
    tmem_wait_st();
    fence_proxy_async_smem();
    tc_fence_before();
    // ===== [C] S0 and the scaled S are in place
    ok = !named_bar_or(kBarAll, kThreads, !ok || *abort_flag);
    if (!ok) break;
    if (tid == kIssuer) {
      tc_fence_after();
      ok = mbar_wait(&fullA_bar, static_cast<uint32_t>(j & 1), budget);
      if (ok) {
        const uint32_t idesc = idesc_f16(128, 128, kFmtF16, kKMajor, kMNMajor);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16(tbase + kColPQ, sdesc_sw128(sbase + kA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                   sdesc_sw128(sbase + kS0 + kk * 2048, 16384, 1024), idesc, kk > 0);
        umma_commit(&p_bar);
      } else {
        *abort_flag = 1;
      }
    }
    // the next chunk's Gamma_end (record j + 1 was acquired two chunks ago)
    if (j + 1 < nch) gam_next = load_gamma(j + 1);
    o_t0 = t0;
    o_c = c;
    // ===== [D]
    if (out_warp) {
      if (tid == kProducer && ok) {
        // the A tile is free once P(j) has completed: bring chunk j + 1's; then make sure
        // record j + 2 is ready, two chunks before it is needed
        if (mbar_wait(&p_bar, static_cast<uint32_t>(j & 1), budget)) {
          if (j + 1 < nch) load_A(j + 1);
          ok = acquire(j + 2);
        } else {
          ok = false;
        }
        if (!ok) *abort_flag = 1;
      }
      // the previous record is fully read (its last readers, update and O of chunk
      // j - 1, completed before the drain above): drop it from L2
      if (j > 0 && ok) discard_record(j - 1);
    } else {
      // Ud = U - P_W in place in the B tile: row r = L - 64, value columns v0 .. v0 + 63
      // (U arrived with chunk j's Kd / Aqk tiles)
      ok = ok && mbar_wait(&p_bar, static_cast<uint32_t>(j & 1), budget) && !*abort_flag;
      ok = ok && mbar_wait(&fullY_bar, static_cast<uint32_t>(j & 1), budget) && !*abort_flag;
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) {
        const uint32_t urow = sbase + kUd + static_cast<uint32_t>(half) * 8192u;
        const uint32_t r = static_cast<uint32_t>(L - 64);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          uint32_t a[32];
          tmem_ld32(tmem_addr(tbase, lane_base, kColPQ + v0 + part * 32), a);
          tmem_wait_ld();
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t addr = urow + sw128_offset(r, static_cast<uint32_t>(part * 4 + c4));
            uint32_t uw[4];
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(uw[0]), "=r"(uw[1]), "=r"(uw[2]), "=r"(uw[3])
                         : "r"(addr));
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 uf = __half22float2(*reinterpret_cast<const __half2*>(&uw[e]));
              w[e] = pack_f16(uf.x - __uint_as_float(a[c4 * 8 + 2 * e]),
                              uf.y - __uint_as_float(a[c4 * 8 + 2 * e + 1]));
            }
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                         "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3])
                         : "memory");
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      // ===== [E] Ud is in place: the update and O
      ok = !named_bar_or(kBarUd, 128, !ok || *abort_flag);
      if (ok && tid == kIssuer) {
        tc_fence_after();
        ok = mbar_wait(&fullY_bar, static_cast<uint32_t>(j & 1), budget);
        if (ok) {
          const uint32_t id_s = idesc_f16(128, 128, kFmtF16, kMNMajor, kMNMajor);
          const uint32_t id_o = idesc_f16(128, 128, kFmtF16, kKMajor, kMNMajor);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(tbase + kColS, sdesc_sw128(sbase + kKd + kk * 2048, 8192, 1024),
                     sdesc_sw128(sbase + kUd + kk * 2048, 8192, 1024), id_s, 1);
          umma_commit(&s_bar);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(tbase + kColPQ, sdesc_sw128(sbase + kAqk + kk * 32, 16, 1024),
                     sdesc_sw128(sbase + kUd + kk * 2048, 8192, 1024), id_o, 1);
          umma_commit(&o_bar);
        } else {
          *abort_flag = 1;
        }
      }
    }
  }

  // ---- the last chunk: its O, the final state, the checkpoint at p = len
  ok = __all_sync(0xffffffffu, ok);
  if (ok && nch > 0) {
    if (out_warp) {
      ok = mbar_wait(&o_bar, static_cast<uint32_t>((nch - 1) & 1), budget) && !*abort_flag;
      ok = __all_sync(0xffffffffu, ok);
      tc_fence_after();
      if (ok) {
        drain_out(o_t0, o_c);
        discard_record(nch - 1);
      }
    }
    if (ok) ok = mbar_wait(&s_bar, static_cast<uint32_t>((nch - 1) & 1), budget) && !*abort_flag;
    ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    if (ok) {
      float* dsts[2] = {p.ht ? p.ht + nh * (kD * kD) + L * kD + v0 : nullptr,
                        (ckr && si.ck == si.len) ? ckr : nullptr};
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        uint32_t a[32];
        tmem_ld32(tmem_addr(tbase, lane_base, kColS + v0 + part * 32), a);
        tmem_wait_ld();
#pragma unroll
        for (int d = 0; d < 2; ++d) {
          if (!dsts[d]) continue;
#pragma unroll
          for (int i4 = 0; i4 < 8; ++i4)
            *reinterpret_cast<float4*>(dsts[d] + part * 32 + i4 * 4) =
                make_float4(__uint_as_float(a[4 * i4]), __uint_as_float(a[4 * i4 + 1]),
                            __uint_as_float(a[4 * i4 + 2]), __uint_as_float(a[4 * i4 + 3]));
        }
      }
    }
  } else if (ok && nch == 0 && p.ht != nullptr) {
    // an empty sequence: ht = h0 (an exact alias of h0 is left as it is)
    const float* h0r = p.h0 ? p.h0 + nh * (kD * kD) + L * kD + v0 : nullptr;
    float* htr = p.ht + nh * (kD * kD) + L * kD + v0;
    if (htr != h0r) {
#pragma unroll
      for (int i4 = 0; i4 < 16; ++i4)
        *reinterpret_cast<float4*>(htr + i4 * 4) =
            h0r ? *reinterpret_cast<const float4*>(h0r + i4 * 4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  if (!ok) {
    *abort_flag = 1;
    record_status(p.ws, kStatusTimeout);
  }

  // ---- teardown: every TMA copy and UMMA of this unit completes before the caller frees
  // tensor memory or the CTA exits
  if (tid == kProducer && issuedA > 0)
    mbar_wait(&fullA_bar, static_cast<uint32_t>((issuedA - 1) & 1), drain_budget);
  if (tid == kLoaderY && issuedY > 0)
    mbar_wait(&fullY_bar, static_cast<uint32_t>((issuedY - 1) & 1), drain_budget);
  if (tid == kIssuer) {
    umma_commit(&drain_bar);
    mbar_wait(&drain_bar, 0, drain_budget);
  }
  tc_fence_before();
  named_bar_sync(kBarAll, kThreads);
}

}  // namespace kda
