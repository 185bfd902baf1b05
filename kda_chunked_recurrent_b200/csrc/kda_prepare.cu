// kda_prepare.cu — chunk-local prepare kernel (split variant).
//
// One CTA (256 threads) per (chunk slot, head).  For its 64-token chunk it
// forms the decay-weighted intra-chunk products, solves the unit-lower-
// triangular UT/WY system and writes the per-chunk operands the recurrence
// kernel consumes:
//   W^T, (Q*Gamma)^T (bf16), U^T, Kd^T (f16), Aqk (f16), Gamma_end (f32)
// A checkpoint offset p inside a sequence is a chunk boundary of the schedule
// (the chunks cover [0, p) and [p, len) separately), so the checkpoint state is
// the state after a chunk and needs no extra operands here.
// (north star subsystem (a): "a chunk-local prepare kernel that forms the
// decay-weighted intra-chunk products, solves the unit-lower-triangular UT/WY
// system per chunk and emits W and U"; the split into prepare and recurrence
// launches is the "decomp" variant of FlashInfer PR #4633 "Description").
//
// Thread mapping for the element-wise part: thread t owns the channel pair
// (2p, 2p+1), p = t % 64, in sub-block b = t / 64 (tokens 16b .. 16b+15), so a
// warp writes one full 128-byte swizzled row of one operand panel per store.
//
// Decay factorisation (log2 domain, G = cumsum(g * log2 e), B_b = G at the
// first token of sub-block b, E = G at the chunk end):
//   e_r   = 2^(G_r - B_b)   in [2^-116, 1]        inv_r = 2^(B_b - G_r) in [1, 2^116]
//   K+_r  = k_r e_r,  Q+_r = q_r e_r              (left operand, row r / 64 + r)
//   R^i_r = k_r inv_r 2^(B_i - B_b)  for i >= b   (right operand, segment i)
//   Gamma_r = e_r 2^(B_b),  Kd_r = k_r inv_r 2^(E - B_b)
// so the only per-element MUFU work is e_r and inv_r.  When 2^(B_i - B_b) or
// 2^(E - B_b) underflows, the exact product is below 2^-18 (|G_r - B_b| <= 116),
// an absolute error far under the BF16/FP16 rounding of the operands.
//   A[r, s] = K+_r . R^{b(r)}_s for every s in sub-blocks 0..b(r): inside one
// sub-block the exponents cancel (|.| <= 80 nats); before it both factors are
// <= 1.  One UMMA of M = 128 ([K+; Q+]) by N = 160 (R^0..R^3, 16+32+48+64 rows)
// yields A (strict lower part) and Aqk (lower part with the diagonal).
//
// UT solve: T = (I + M)^-1 with M = diag(beta) A_strict.  The four 16x16
// diagonal blocks are inverted in FP32 by forward substitution; the off-
// diagonal blocks follow level by level, X_ij = -X_ii sum_{k=j}^{i-1} M_ik X_kj,
// as FP16 mma.sync products with FP32 accumulation.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace prep {
constexpr int kThreads = 256;
constexpr uint32_t kV = 0;           // 16 KB  v tile, MN-major A of U^T: 2 panels [64 tok][64 v]
constexpr uint32_t kKG = 16384;      // 16 KB  K*Gamma tile, MN-major A of W^T
constexpr uint32_t kL = 32768;       // 32 KB  [K+; Q+], K-major A: 2 panels [128 rows][64 ch]
constexpr uint32_t kR = 65536;       // 40 KB  R^0..R^3, K-major B: 2 panels [160 rows][64 ch]
constexpr uint32_t kBytes = 65536 + 40960;
// aliases, valid once the first UMMA has completed
constexpr uint32_t kMf = 32768;                 // f32 [4][16][17] diagonal blocks of M
constexpr uint32_t kMh = kMf + 4 * 16 * 17 * 4; // f16 [64][72] off-diagonal blocks of M
constexpr uint32_t kXh = kMh + 64 * 72 * 2;     // f16 [64][72] T = (I + M)^-1
constexpr uint32_t kYh = kXh + 64 * 72 * 2;     // f16 [3][16][24] block products
constexpr uint32_t kTb = 98304;                 // 8 KB T diag(beta) bf16, K-major [64 r][64 s]
constexpr int kLdh = 72;
constexpr uint32_t kSmemAlloc = kBytes + 1024;
extern const uint32_t kSmemAllocBytes = kSmemAlloc;
static_assert(kYh + 3 * 16 * 24 * 2 <= kTb, "solve scratch overlaps the Tb tile");
}  // namespace prep

// Offset of element (row, ch) in a 2-panel, 128B-swizzled [rows][128] 16-bit tile.
__device__ __forceinline__ uint32_t tile_off(uint32_t rows, uint32_t row, uint32_t ch) {
  return (ch >> 6) * (rows * 128u) + sw128_offset(row, (ch & 63u) >> 3) + ((ch & 7u) << 1);
}

// Packed bf16x2 product (round to nearest even), for operands that are rounded
// to bf16 for the tensor core anyway.
__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<const __nv_bfloat162*>(&a),
                             *reinterpret_cast<const __nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

__device__ __forceinline__ float2 bf2_to_f2(uint32_t u) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.x4.m8n8.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.x4.trans.m8n8.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// D(16x8, f32) += A(16x16, f16, row) * B(16x8, f16, col)
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Store a 16x16 f32 accumulator pair (two m16n8 fragments) as f16 into a
// row-major tile (row stride `ld` halves), multiplied by `s`.
__device__ __forceinline__ void store_frag16(__half* base, int ld, const float (&c0)[4],
                                             const float (&c1)[4], float s, int lane) {
  const int g = lane >> 2, q = lane & 3;
  *reinterpret_cast<__half2*>(base + g * ld + 2 * q) = __floats2half2_rn(s * c0[0], s * c0[1]);
  *reinterpret_cast<__half2*>(base + (g + 8) * ld + 2 * q) = __floats2half2_rn(s * c0[2], s * c0[3]);
  *reinterpret_cast<__half2*>(base + g * ld + 8 + 2 * q) = __floats2half2_rn(s * c1[0], s * c1[1]);
  *reinterpret_cast<__half2*>(base + (g + 8) * ld + 8 + 2 * q) =
      __floats2half2_rn(s * c1[2], s * c1[3]);
}

// Write one row of the first UMMA's result.  Row rl lies in sub-block BL and
// `val[s]` holds its products with the right-operand segment of that sub-block
// (s = 0 .. 16 BL + 15).  Key rows feed M = diag(beta) A_strict (diagonal block in
// FP32, earlier blocks in FP16); query rows are Aqk (s <= rl) written as FP16.
template <int BL>
__device__ __forceinline__ void emit_rows(const uint32_t* val, bool is_q, int rl, float br,
                                          uint8_t* sm, __half* aqk_row) {
  using namespace prep;
  constexpr int NV = 16 * (BL + 1);
  if (!is_q) {
    float* Mf = reinterpret_cast<float*>(sm + kMf) + BL * (16 * 17) + (rl & 15) * 17;
#pragma unroll
    for (int s = 16 * BL; s < 16 * BL + 16; ++s)
      Mf[s & 15] = (s < rl) ? br * __uint_as_float(val[s]) : 0.f;
    __half* Mh = reinterpret_cast<__half*>(sm + kMh) + rl * kLdh;
#pragma unroll
    for (int s0 = 0; s0 < 16 * BL; s0 += 8) {
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u)
        pk[u] = pack_f16(br * __uint_as_float(val[s0 + 2 * u]),
                         br * __uint_as_float(val[s0 + 2 * u + 1]));
      *reinterpret_cast<uint4*>(Mh + s0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  } else {
#pragma unroll
    for (int s0 = 0; s0 < kC; s0 += 8) {
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = s0 + 2 * u;
        const float a = (s < NV && s <= rl) ? __uint_as_float(val[s < NV ? s : 0]) : 0.f;
        const float b2 = (s + 1 < NV && s + 1 <= rl) ? __uint_as_float(val[s + 1 < NV ? s + 1 : 0]) : 0.f;
        pk[u] = pack_f16(a, b2);
      }
      *reinterpret_cast<uint4*>(aqk_row + s0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Work item w of the persistent grid: chunk slot w / H, head w % H.  Returns
// false when the slot holds no chunk (past the end of the chunk table).
struct PrepItem {
  int32_t h, c, t0;
  int64_t slot, rec;
};
__device__ __forceinline__ bool locate_item(const KdaParams& p, int64_t w, PrepItem& it) {
  it.slot = w / p.H;
  it.h = static_cast<int32_t>(w % p.H);
  if (it.slot >= p.slots) return false;
  int32_t n = 0, j = 0;
  if (p.cu_seqlens == nullptr && p.ckpt_offsets == nullptr) {
    const int32_t cps = (p.fixed_len + kC - 1) / kC;
    n = static_cast<int32_t>(it.slot / cps);
    j = static_cast<int32_t>(it.slot % cps);
  } else {
    const int32_t* cb = reinterpret_cast<const int32_t*>(p.ws + p.lay.chunk_base);
    if (it.slot >= cb[p.N]) return false;
    int32_t lo = 0, hi = p.N;  // largest n with cb[n] <= slot
    while (hi - lo > 1) {
      const int32_t mid = (lo + hi) >> 1;
      if (cb[mid] <= it.slot) lo = mid; else hi = mid;
    }
    n = lo;
    j = static_cast<int32_t>(it.slot - cb[n]);
  }
  if (n >= p.N) return false;
  const SeqInfo si = seq_info(p, n, false);
  if (j >= si.nch) return false;
  chunk_span(si, j, it.t0, it.c);
  it.t0 += si.start;
  it.rec = it.slot * p.H + it.h;
  return it.c > 0;
}

__global__ void __launch_bounds__(prep::kThreads, 2)
kda_prepare_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  using namespace prep;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ float s_beta[kC];
  __shared__ float2 s_tot[4][64];   // per sub-block totals of g (log2 domain), channel pairs
  __shared__ float2 s_B[4][64];     // B_b per sub-block
  __shared__ float2 s_end[64];      // E (chunk end)

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;
  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;
  const int64_t nitems = p.slots * p.H;

  if (tid == 0) {
    mbar_init(&tma_bar, 1);
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.v_in);
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  bool ok = true;
  int mma_commits = 0;     // UMMA commits issued so far (their mbarrier phases)
  int tma_issued = 0;      // v tiles issued so far (tma_bar phases)

  PrepItem cur;
  bool cur_valid = blockIdx.x < nitems && locate_item(p, blockIdx.x, cur);
  for (int64_t w = blockIdx.x; w < nitems && ok; w += gridDim.x) {
    PrepItem nxt;
    const bool nxt_valid = (w + gridDim.x < nitems) && locate_item(p, w + gridDim.x, nxt);
    if (!cur_valid) {
      cur = nxt;
      cur_valid = nxt_valid;
      continue;
    }
    const int h = cur.h;
    const int32_t t0 = cur.t0, c = cur.c;
    const int64_t rec = cur.rec;

    // ---- loads: g (float2), k, q (bf16x2) for 16 tokens x 2 channels
    const int cp = tid & 63;         // channel pair
    const int blk = tid >> 6;        // sub-block 0..3
    const int ch0 = 2 * cp;
    const int64_t rstride = static_cast<int64_t>(p.H) * kD;
    const int64_t base_el = (static_cast<int64_t>(t0) * p.H + h) * kD + ch0;
    float2 G[16];
    uint32_t kw[16], qw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int r = blk * 16 + i;
      const int64_t el = base_el + r * rstride;
      if (r < c) {
        G[i] = __ldg(reinterpret_cast<const float2*>(p.g + el));
        kw[i] = __ldg(reinterpret_cast<const unsigned int*>(p.k + el));
        qw[i] = __ldg(reinterpret_cast<const unsigned int*>(p.q + el));
      } else {
        G[i] = make_float2(0.f, 0.f);
        kw[i] = 0u;
        qw[i] = 0u;
      }
    }
    if (tid < kC) {
      float b = 0.f;
      if (tid < c) b = bf16_to_f32(p.beta[static_cast<int64_t>(t0 + tid) * p.H + h]);
      s_beta[tid] = b;
    }

    // ---- L2 prefetch of the next item's rows (q, k, v: 256 B, g: 512 B per token)
    if (nxt_valid) {
      const int which = tid >> 6, r = tid & 63;
      if (r < nxt.c) {
        const int64_t row = (static_cast<int64_t>(nxt.t0) + r) * p.H + nxt.h;
        if (which == 0) bulk_prefetch_l2(p.q + row * kD, 256);
        else if (which == 1) bulk_prefetch_l2(p.k + row * kD, 256);
        else if (which == 2) bulk_prefetch_l2(p.v + row * kD, 256);
        else bulk_prefetch_l2(p.g + row * kD, 512);
      }
    }

    // ---- TMA: v tile straight into the MN-major A operand of U^T
    if (tid == 0) {
      mbar_arrive_expect_tx(&tma_bar, 16384);
      tma_load_3d(sm + kV, &maps.v_in, &tma_bar, 0, h, t0);
      tma_load_3d(sm + kV + 8192, &maps.v_in, &tma_bar, 64, h, t0);
    }
    const uint32_t tma_parity = static_cast<uint32_t>(tma_issued & 1);
    ++tma_issued;

  // ---- gate scan within the sub-block, then across sub-blocks
  {
    float2 run = make_float2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      run.x = fmaf(G[i].x, kLog2e, run.x);
      run.y = fmaf(G[i].y, kLog2e, run.y);
      G[i] = run;
    }
    s_tot[blk][cp] = run;
  }
  __syncthreads();
  {
    float2 pre = make_float2(0.f, 0.f);
    for (int b = 0; b < blk; ++b) {
      pre.x += s_tot[b][cp].x;
      pre.y += s_tot[b][cp].y;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      G[i].x += pre.x;
      G[i].y += pre.y;
    }
    s_B[blk][cp] = G[0];
    if (blk == 3) s_end[cp] = G[15];
  }
  __syncthreads();

  // ---- operands
  {
    const float2 B = G[0];
    const float2 E = s_end[cp];
    const float2 cB = make_float2(ex2(B.x), ex2(B.y));                    // 2^B_b
    const float2 cE = make_float2(ex2(E.x - B.x), ex2(E.y - B.y));        // 2^(E - B_b)
    // 2^(B_i - B_b) for the later sub-blocks i = 1, 2, 3 (unused entries never read)
    float2 c1 = make_float2(0.f, 0.f), c2 = c1, c3 = c1;
    if (blk < 1) { const float2 b1 = s_B[1][cp]; c1 = make_float2(ex2(b1.x - B.x), ex2(b1.y - B.y)); }
    if (blk < 2) { const float2 b2 = s_B[2][cp]; c2 = make_float2(ex2(b2.x - B.x), ex2(b2.y - B.y)); }
    if (blk < 3) { const float2 b3 = s_B[3][cp]; c3 = make_float2(ex2(b3.x - B.x), ex2(b3.y - B.y)); }
    const int seg_own = (blk == 0) ? 0 : (blk == 1) ? 16 : (blk == 2) ? 48 : 96;
    // Store addresses.  Row r = 16 blk + i has (r & 7) == (i & 7), so the 128-byte
    // swizzle of every operand row reduces to a per-thread base plus one of eight
    // per-thread XOR terms and a compile-time row offset.
    const uint32_t panel = static_cast<uint32_t>(cp >> 5);
    const uint32_t chunk = static_cast<uint32_t>((cp & 31) >> 2);
    const uint32_t inner = static_cast<uint32_t>((cp & 3) * 4 + blk * 2048);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t bL = sbase + kL + panel * 16384u + inner;
    const uint32_t bR = sbase + kR + panel * 20480u + inner;
    const uint32_t bRo = bR + static_cast<uint32_t>(seg_own) * 128u;
    const uint32_t bKG = sbase + kKG + panel * 8192u + inner;
    const uint32_t cB2 = pack_bf16(cB.x, cB.y);
    const uint32_t c1b = pack_bf16(c1.x, c1.y), c2b = pack_bf16(c2.x, c2.y),
                   c3b = pack_bf16(c3.x, c3.y);
    uint32_t qg_lo[8], qg_hi[8], kd_lo[8], kd_hi[8];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const uint32_t xo = ((chunk ^ static_cast<uint32_t>(i & 7)) << 4) + static_cast<uint32_t>(i) * 128u;
      const float2 g2 = G[i];
      const float e0 = ex2(g2.x - B.x), e1 = ex2(g2.y - B.y);
      const float i0 = ex2(B.x - g2.x), i1 = ex2(B.y - g2.y);
      // bf16 operands: factors rounded to bf16, products in packed bf16 math
      const uint32_t e2 = pack_bf16(e0, e1), inv2 = pack_bf16(i0, i1);
      sts32(bL + xo, hmul2_bf16(kw[i], e2));
      sts32(bL + xo + 64u * 128u, hmul2_bf16(qw[i], e2));
      const uint32_t rd2 = hmul2_bf16(kw[i], inv2);
      sts32(bRo + xo, rd2);
      if (blk < 1) sts32(bR + xo + 16u * 128u, hmul2_bf16(rd2, c1b));
      if (blk < 2) sts32(bR + xo + 48u * 128u, hmul2_bf16(rd2, c2b));
      if (blk < 3) sts32(bR + xo + 96u * 128u, hmul2_bf16(rd2, c3b));
      const uint32_t gm2 = hmul2_bf16(e2, cB2);
      sts32(bKG + xo, hmul2_bf16(kw[i], gm2));
      const uint32_t qg = hmul2_bf16(qw[i], gm2);
      // Kd feeds the FP16 state update: FP32 products, one rounding
      const float2 kf = bf2_to_f2(kw[i]);
      const uint32_t kd = pack_f16(kf.x * i0 * cE.x, kf.y * i1 * cE.y);
      // transpose the channel pairs into per-channel token rows (lo = channel 2p, hi = 2p+1)
      if (i & 1) {
        qg_lo[i >> 1] |= qg << 16;
        qg_hi[i >> 1] |= qg & 0xFFFF0000u;
        kd_lo[i >> 1] |= kd << 16;
        kd_hi[i >> 1] |= kd & 0xFFFF0000u;
      } else {
        qg_lo[i >> 1] = qg & 0xFFFFu;
        qg_hi[i >> 1] = qg >> 16;
        kd_lo[i >> 1] = kd & 0xFFFFu;
        kd_hi[i >> 1] = kd >> 16;
      }
    }
    // (Q Gamma)^T, Kd^T (and Kp^T) rows: channel ch0 / ch0 + 1, tokens 16 blk .. 16 blk + 15
    uint8_t* qgt = p.ws + p.lay.qgt + rec * kTileQGT + (ch0 * 64 + blk * 16) * 2;
    uint8_t* kdt = p.ws + p.lay.kdt + rec * kTileKdT + (ch0 * 64 + blk * 16) * 2;
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      reinterpret_cast<uint4*>(qgt)[hh] =
          make_uint4(qg_lo[4 * hh], qg_lo[4 * hh + 1], qg_lo[4 * hh + 2], qg_lo[4 * hh + 3]);
      reinterpret_cast<uint4*>(qgt + 128)[hh] =
          make_uint4(qg_hi[4 * hh], qg_hi[4 * hh + 1], qg_hi[4 * hh + 2], qg_hi[4 * hh + 3]);
      reinterpret_cast<uint4*>(kdt)[hh] =
          make_uint4(kd_lo[4 * hh], kd_lo[4 * hh + 1], kd_lo[4 * hh + 2], kd_lo[4 * hh + 3]);
      reinterpret_cast<uint4*>(kdt + 128)[hh] =
          make_uint4(kd_hi[4 * hh], kd_hi[4 * hh + 1], kd_hi[4 * hh + 2], kd_hi[4 * hh + 3]);
    }
    if (blk == 0)
      reinterpret_cast<float2*>(p.ws + p.lay.gc + rec * kTileGC)[cp] =
          make_float2(ex2(E.x), ex2(E.y));
  }

  // ---- UMMA 1: D[0:128, 0:160] = [K+; Q+] . R^T   (bf16 -> f32)
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0) {
    tc_fence_after();
    const uint32_t idesc = idesc_f16(128, 160, kFmtBF16, kKMajor, kKMajor);
    const uint32_t aL = smem_u32(sm + kL), aR = smem_u32(sm + kR);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t ad = sdesc_sw128(aL + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
      const uint64_t bd = sdesc_sw128(aR + (kk >> 2) * 20480 + (kk & 3) * 32, 16, 1024);
      umma_f16(tbase, ad, bd, idesc, kk > 0);
    }
    umma_commit(&mma_bar);
  }
  ++mma_commits;
  ok = mbar_wait(&mma_bar, static_cast<uint32_t>((mma_commits - 1) & 1), budget);
  ok = !__syncthreads_or(!ok);
  if (ok) {
    tc_fence_after();
    // ---- extract A (lane quarters 0,1) and Aqk (quarters 2,3): row rl, sub-block bl.
    // Warps w and w + 4 share a lane quarter; warp w reads the column segment of
    // the first sub-block its rows hold, warp w + 4 that of the second, so at most
    // 64 accumulator values are live per thread and all eight warps take part.
    const int qw = warp & 3, phase = warp >> 2;
    const int rl = (qw & 1) * 32 + lane;
    const int bl = rl >> 4;
    const bool is_q = qw >= 2;
    const uint32_t lane_base = static_cast<uint32_t>(qw * 32);
    const float br = s_beta[rl];
    __half* aqk_row = reinterpret_cast<__half*>(p.ws + p.lay.aqk + rec * kTileAqk) + rl * 64;
    if ((qw & 1) == 0) {
      if (phase == 0) {
        uint32_t v[16];
        tmem_ld16(tmem_addr(tbase, lane_base, 0), v);
        tmem_wait_ld();
        if (bl == 0) emit_rows<0>(v, is_q, rl, br, sm, aqk_row);
      } else {
        uint32_t v[32];
        tmem_ld32(tmem_addr(tbase, lane_base, 16), v);
        tmem_wait_ld();
        if (bl == 1) emit_rows<1>(v, is_q, rl, br, sm, aqk_row);
      }
    } else {
      if (phase == 0) {
        uint32_t v[48], t32[32], t16[16];
        tmem_ld32(tmem_addr(tbase, lane_base, 48), t32);
        tmem_ld16(tmem_addr(tbase, lane_base, 80), t16);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = t32[i];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[32 + i] = t16[i];
        if (bl == 2) emit_rows<2>(v, is_q, rl, br, sm, aqk_row);
      } else {
        uint32_t v[64], t0[32], t1[32];
        tmem_ld32(tmem_addr(tbase, lane_base, 96), t0);
        tmem_ld32(tmem_addr(tbase, lane_base, 128), t1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = t0[i];
          v[32 + i] = t1[i];
        }
        if (bl == 3) emit_rows<3>(v, is_q, rl, br, sm, aqk_row);
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  if (ok) {
    __half* Xh = reinterpret_cast<__half*>(sm + kXh);
    // ---- diagonal blocks: forward substitution in FP32, one column per thread
    if (tid < 64) {
      const int bi = tid >> 4, jj = tid & 15;
      const float* Mf = reinterpret_cast<const float*>(sm + kMf) + bi * (16 * 17);
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        float acc0 = 0.f, acc1 = 0.f;  // two partial sums halve the dependent chain
#pragma unroll
        for (int ss = 0; ss < rr; ss += 2) {
          acc0 = fmaf(Mf[rr * 17 + ss], x[ss], acc0);
          if (ss + 1 < rr) acc1 = fmaf(Mf[rr * 17 + ss + 1], x[ss + 1], acc1);
        }
        x[rr] = (rr < jj) ? 0.f : (rr == jj ? 1.f : -(acc0 + acc1));
      }
#pragma unroll
      for (int rr = 0; rr < 16; ++rr)
        Xh[(bi * 16 + rr) * kLdh + bi * 16 + jj] = __float2half_rn(x[rr]);
    }
    __syncthreads();
    // ---- off-diagonal blocks, level by level (one warp per block pair)
    const uint32_t aMh = smem_u32(sm + kMh), aXh = smem_u32(sm + kXh), aYh = smem_u32(sm + kYh);
    for (int d = 1; d <= 3; ++d) {
      if (warp < 4 - d) {
        const int pi = warp, bi = d + pi, bj = pi;
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        for (int kb = bj; kb < bi; ++kb) {
          uint32_t a[4], b[4];
          ldsm_x4(aMh + ((bi * 16 + (lane & 15)) * kLdh + kb * 16 + (lane >> 4) * 8) * 2, a);
          ldsm_x4_t(aXh + ((kb * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * kLdh + bj * 16 +
                           (lane >> 4) * 8) * 2, b);
          mma16816(acc0, a, b[0], b[1]);
          mma16816(acc1, a, b[2], b[3]);
        }
        __half* Y = reinterpret_cast<__half*>(sm + kYh) + pi * (16 * 24);
        store_frag16(Y, 24, acc0, acc1, 1.f, lane);
        __syncwarp();
        float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
        {
          uint32_t a[4], b[4];
          ldsm_x4(aXh + ((bi * 16 + (lane & 15)) * kLdh + bi * 16 + (lane >> 4) * 8) * 2, a);
          ldsm_x4_t(aYh + (pi * (16 * 24) + ((lane & 7) + ((lane >> 3) & 1) * 8) * 24 +
                           (lane >> 4) * 8) * 2, b);
          mma16816(x0, a, b[0], b[1]);
          mma16816(x1, a, b[2], b[3]);
        }
        store_frag16(Xh + (bi * 16) * kLdh + bj * 16, kLdh, x0, x1, -1.f, lane);
      }
      __syncthreads();
    }
    // ---- T diag(beta) -> bf16, K-major [r][s] (the B operand (T diag beta)^T)
    {
      const int r = tid >> 2, part = tid & 3;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int chunk = part * 2 + cc;
        const uint4 xv = *reinterpret_cast<const uint4*>(Xh + r * kLdh + chunk * 8);
        const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = chunk * 8 + 2 * u;
          const float2 xf = __half22float2(*reinterpret_cast<const __half2*>(&xw[u]));
          const float a = (s <= r) ? xf.x * s_beta[s] : 0.f;
          const float b2 = (s + 1 <= r) ? xf.y * s_beta[s + 1] : 0.f;
          pk[u] = pack_bf16(a, b2);
        }
        *reinterpret_cast<uint4*>(sm + kTb + sw128_offset(r, chunk)) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  ok = !__syncthreads_or(!ok);

  // ---- UMMA 2: W^T = (K Gamma)^T (T diag beta)^T -> cols [0,64); U^T = V^T (T diag beta)^T -> [64,128)
  bool tma_seen = false;
  if (ok && tid == 0) {
    tma_seen = mbar_wait(&tma_bar, tma_parity, budget);
    if (tma_seen) {
      tc_fence_after();
      const uint32_t idesc = idesc_f16(128, 64, kFmtBF16, kMNMajor, kKMajor);
      const uint32_t aKG = smem_u32(sm + kKG), aV = smem_u32(sm + kV), bT = smem_u32(sm + kTb);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const uint64_t bd = sdesc_sw128(bT + kk * 32, 16, 1024);
        umma_f16(tbase + 0, sdesc_sw128(aKG + kk * 2048, 8192, 1024), bd, idesc, kk > 0);
        umma_f16(tbase + 64, sdesc_sw128(aV + kk * 2048, 8192, 1024), bd, idesc, kk > 0);
      }
      umma_commit(&mma_bar);
    }
  }
  if (tid == 0 && !tma_seen) ok = false;
  ok = !__syncthreads_or(!ok);
  if (ok) {
    ++mma_commits;
    ok = mbar_wait(&mma_bar, static_cast<uint32_t>((mma_commits - 1) & 1), budget);
  }
  ok = !__syncthreads_or(!ok);
  if (ok) {
    tc_fence_after();
    // warps 0-3: W^T rows (lane = k); warps 4-7: U^T rows (lane = v)
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32);
    const int row = (warp & 3) * 32 + lane;
    const bool is_u = warp >= 4;
    uint8_t* dst = is_u ? p.ws + p.lay.ut + rec * kTileUT + row * 128
                        : p.ws + p.lay.wt + rec * kTileWT + row * 128;
    const uint32_t col0 = is_u ? 64u : 0u;
    uint32_t a[32];
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      tmem_ld32(tmem_addr(tbase, lane_base, col0 + part * 32), a);
      tmem_wait_ld();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint4 o;
        const float* f = reinterpret_cast<const float*>(a) + q8 * 8;
        if (is_u) {
          o = make_uint4(pack_f16(f[0], f[1]), pack_f16(f[2], f[3]), pack_f16(f[4], f[5]),
                         pack_f16(f[6], f[7]));
        } else {
          o = make_uint4(pack_bf16(f[0], f[1]), pack_bf16(f[2], f[3]), pack_bf16(f[4], f[5]),
                         pack_bf16(f[6], f[7]));
        }
        reinterpret_cast<uint4*>(dst)[part * 4 + q8] = o;
      }
    }
  }

    // next item: every thread is done with this item's TMEM and shared tiles
    tc_fence_before();
    ok = !__syncthreads_or(!ok);
    cur = nxt;
    cur_valid = nxt_valid;
  }

  // ---- teardown: on any failure record it, drain what was issued, free TMEM
  if (!ok) {
    if (tid == 0) {
      record_status(p.ws, kStatusTimeout);
      // copies and commits complete in issue order: waiting for the last drains all
      if (tma_issued > 0)
        mbar_wait(&tma_bar, static_cast<uint32_t>((tma_issued - 1) & 1), drain_budget);
      if (mma_commits > 0)
        mbar_wait(&mma_bar, static_cast<uint32_t>((mma_commits - 1) & 1), drain_budget);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 256);
}

}  // namespace kda
