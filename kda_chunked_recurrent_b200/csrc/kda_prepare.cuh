// kda_prepare.cuh — chunk-local prepare (body shared by the split prepare kernel
// and the prepare CTAs of the fused launch).
//
// A persistent grid (two CTAs of 256 threads per SM in the split variant) walks
// the records (chunk slot, head).  For each 64-token chunk it forms the decay-weighted
// intra-chunk products, solves the unit-lower-triangular UT/WY system and
// writes the per-chunk operands the recurrence kernel consumes:
//   W^T [128 k][64 tok] f16, U^T [128 v][64 tok] f16, Aqk [64][64] f16
//   (UMMA results, staged in shared memory and written by TMA tile stores),
//   Q*Gamma [64 tok][128 k] f16, Kd [64 tok][128 k] f16 (token rows, written
//   straight from the element-wise pass with 128-byte warp stores),
//   Gamma_end [128] f32.
// A checkpoint offset p inside a sequence is a chunk boundary of the schedule
// (the chunks cover [0, p) and [p, len) separately), so the checkpoint state is
// the state after a chunk and needs no extra operands here.
// This is the chunk-local step of the method: decay-weighted intra-chunk key
// products, the unit-lower-triangular UT/WY solve and W, U per chunk.  Running it
// as its own launch before the recurrence is the two-launch design FlashInfer PR
// #4633 calls decomp ("Description").
//
// Inputs of a chunk: q, k (bf16) and g (f32) arrive by TMA as whole [64 tok][128 ch]
// tiles into shared memory the previous chunk no longer needs: g into R once that
// chunk's Aqk store has read R (during its off-diagonal solve), q and k into the v and
// K Gamma tiles once its second UMMA has completed; all of them were prefetched into L2
// one chunk earlier.  k and g go to registers before the element-wise pass; q is read
// from its tile row by row during it (fewer live registers), so v follows by TMA into
// its UMMA operand layout only after that pass, and is converted from BF16 to FP16 in
// place during the off-diagonal solve.
//
// Thread mapping for the element-wise part: thread t owns the channel pair
// (2p, 2p+1), p = t % 64, in sub-block b = t / 64 (tokens 16b .. 16b+15), so a
// warp writes one full 128-byte row of one operand per store.
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
// UT solve: T = (I + M)^-1 with M = diag(beta) A_strict, in 16x16 blocks.  The
// diagonal blocks X_ii are inverted in FP32 by right-looking forward substitution;
// then each of three warps walks one block column down, X_ij = -X_ii (sum_{k=j}^{i-1}
// M_ik X_kj), as FP16 mma.sync products with FP32 accumulation, kept in registers (in
// transposed form every accumulator is the next product's A fragment).  Each block of
// T diag(beta), the operand of the W/U UMMA, is written from the accumulator as soon
// as it is final.
//
// Item order: each 256-thread group walks its items (first, first + stride, ...) with
// their chunk spans looked up 64 at a time into shared memory, skipping items that hold
// no chunk, so that the next item's tiles are always requested one item ahead; the
// stream launch's groups claim items from a counter instead.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace prep {
constexpr int kThreads = 256;
constexpr uint32_t kV = 0;           // 16 KB  v tile, MN-major A of U^T: 2 panels [64 tok][64 v]
                                     //        (lands as BF16, converted to FP16 in place)
constexpr uint32_t kKG = 16384;      // 16 KB  K*Gamma tile (f16), MN-major A of W^T
constexpr uint32_t kL = 32768;       // 32 KB  [K+; Q+], K-major A: 2 panels [128 rows][64 ch]
constexpr uint32_t kR = 65536;       // 40 KB  R^0..R^3, K-major B: 2 panels [160 rows][64 ch]
constexpr uint32_t kBytes = 65536 + 40960;
// raw input tiles of a chunk, landed before its element-wise pass (which reads
// them into registers before anything overwrites these regions)
constexpr uint32_t kQraw = kV;                  // q [64 tok][128 ch] bf16 (read row by row
                                                //   by the element-wise pass)
constexpr uint32_t kKraw = kKG;                 // k [64 tok][128 ch] bf16
constexpr uint32_t kGraw = kR;                  // g [64 tok][128 ch] f32 (32 KB)
constexpr uint32_t kRawQKTx = 16384 + 16384;
constexpr uint32_t kRawGTx = 32768;
// the thread that stores Aqk and requests the next g tile (warp 7, idle in the
// off-diagonal solve); thread 0 issues every other copy and UMMA
constexpr int kGThread = 224;
// the thread that prefetches the next item's tiles into L2 (warp 1, idle while thread 0
// issues the first UMMA)
constexpr int kPrefetchThread = 32;
// aliases of [K+; Q+] once the first UMMA has completed: the solve scratch, and
// after the solve the staging tiles of the W^T / U^T TMA stores
constexpr int kLdh = 72;
constexpr int kMfBlk = 272;                     // floats per diagonal block of Mf (16 x 16 + 16 pad)
constexpr uint32_t kMf = kL;                    // f32 [4][16 s][16 r] diagonal blocks of M, column-major
constexpr uint32_t kMh = kMf + 4 * kMfBlk * 4;  // f16 [64][72] off-diagonal blocks of M
constexpr uint32_t kXh = kMh + 64 * kLdh * 2;   // f16 [64][72] T = (I + M)^-1
constexpr uint32_t kWs = kL;                    // W^T staging [128 k][64 tok] f16, 128B swizzle
constexpr uint32_t kUs = kL + 16384;            // U^T staging [128 v][64 tok] f16, 128B swizzle
// aliases of R once the first UMMA has completed
constexpr uint32_t kAqs = kR;                   // Aqk staging [64 r][64 s] f16, 128B swizzle
constexpr uint32_t kTb = 98304;                 // 8 KB T diag(beta) f16, K-major [64 r][64 s]
// small per-group state after the tiles: mbarriers, TMEM slot, beta, gate sums
constexpr uint32_t kAux = kBytes;
constexpr uint32_t kAuxBars = kAux;              // 4 x u64 mbarriers
constexpr uint32_t kAuxTmem = kAux + 32;         // u32 TMEM base
constexpr uint32_t kAuxBeta = kAux + 64;         // f32 [64]
constexpr uint32_t kAuxTot = kAuxBeta + 256;     // float2 [4][64]
constexpr uint32_t kAuxFirst = kAuxTot + 2048;   // float2 [4][64]
constexpr uint32_t kAuxNorm = kAuxFirst + 2048;  // f32 [2][64] inverse norms of k, q rows (front end)
constexpr uint32_t kAuxClaim = kAuxNorm + 512;   // i64 [2] claimed item indices (stream launch)
constexpr uint32_t kAuxSpan = kAuxClaim + 16;    // int4 [kSpanBatch] looked-up items {t0, c, h, rec}
constexpr int kSpanBatch = 64;
constexpr uint32_t kGroupBytes = (kAuxSpan + 16 * kSpanBatch + 1023) / 1024 * 1024;   // one prepare group
constexpr uint32_t kSmemAlloc = kGroupBytes + 1024;
static_assert(kXh + 64 * kLdh * 2 <= kR, "solve scratch overlaps the Aqk staging tile");
static_assert(kAqs + 8192 <= kTb, "Aqk staging overlaps the Tb tile");
static_assert(kUs + 16384 <= kR, "W/U staging overlaps R");
}  // namespace prep

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

// (c0 | c1) += A * B for 16x16 blocks of two row-major [64][72] f16 arrays:
// A at (ar, ac) of the array at shared address aA, B at (br, bc) of aB.
__device__ __forceinline__ void mma_block(float (&c0)[4], float (&c1)[4], uint32_t aA, int ar,
                                          int ac, uint32_t aB, int br, int bc, int lane) {
  using prep::kLdh;
  uint32_t a[4], b[4];
  ldsm_x4(aA + ((ar + (lane & 15)) * kLdh + ac + (lane >> 4) * 8) * 2, a);
  ldsm_x4_t(aB + ((br + (lane & 7) + ((lane >> 3) & 1) * 8) * kLdh + bc + (lane >> 4) * 8) * 2, b);
  mma16816(c0, a, b[0], b[1]);
  mma16816(c1, a, b[2], b[3]);
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

// Store the same 16x16 block of T, scaled by beta of its column, as FP16 into the
// 128B-swizzled K-major Tb tile (rows r0.., columns c0..).
__device__ __forceinline__ void store_tb16(uint32_t tb, const float* beta, int r0, int c0,
                                           const float (&x0)[4], const float (&x1)[4], int lane) {
  const int g = lane >> 2, q = lane & 3;
  {
    const int s = c0 + 2 * q;
    const float b0 = beta[s], b1 = beta[s + 1];
    const uint32_t off = static_cast<uint32_t>((s & 7) * 2);
    sts32(tb + sw128_offset(r0 + g, s >> 3) + off, pack_f16(x0[0] * b0, x0[1] * b1));
    sts32(tb + sw128_offset(r0 + g + 8, s >> 3) + off, pack_f16(x0[2] * b0, x0[3] * b1));
  }
  {
    const int s = c0 + 8 + 2 * q;
    const float b0 = beta[s], b1 = beta[s + 1];
    const uint32_t off = static_cast<uint32_t>((s & 7) * 2);
    sts32(tb + sw128_offset(r0 + g, s >> 3) + off, pack_f16(x1[0] * b0, x1[1] * b1));
    sts32(tb + sw128_offset(r0 + g + 8, s >> 3) + off, pack_f16(x1[2] * b0, x1[3] * b1));
  }
}

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// One block column J of T = (I + M)^-1 below the diagonal, by one warp, in registers.
// The transposed form
//   P_i^T = sum_{k=J}^{i-1} X_kJ^T M_ik^T,   X_iJ^T = -P_i^T X_ii^T,   i = J+1 .. 3,
// makes every product's FP32 accumulator the A fragment of the next product (rounded to
// FP16), so the column's chain never goes through shared memory; the M_ik and X_ii
// blocks it reads (B fragments: their rows, as stored) do not depend on the chain.
// Each finished block is written as FP16 T diag(beta) into the swizzled Tb tile.
template <int J>
__device__ __forceinline__ void offdiag_column(uint32_t aMh, uint32_t aXh, uint32_t aTb,
                                               const float* beta, int lane) {
  using prep::kLdh;
  // lane addresses of a 16x16 block's four 8x8 matrices, in the order (rows 0-7, col 0),
  // (rows 0-7, col 8), (rows 8-15, col 0), (rows 8-15, col 8): the B fragment of the
  // block's transpose, or with .trans the A fragment of it
  const uint32_t lofs =
      static_cast<uint32_t>((((lane & 7) + ((lane >> 4) & 1) * 8) * kLdh + ((lane >> 3) & 1) * 8) * 2);
  auto at = [&](uint32_t base, int r0, int c0) {
    return base + static_cast<uint32_t>((r0 * kLdh + c0) * 2) + lofs;
  };
  const int g = lane >> 2, q = lane & 3;
  uint32_t xa[4 - J][4];   // A fragments of X_kJ^T, k = J .. 3 (FP16)
  ldsm_x4_t(at(aXh, J * 16, J * 16), xa[0]);
#pragma unroll
  for (int i = J + 1; i < 4; ++i) {
    float c0[4] = {0.f, 0.f, 0.f, 0.f}, c1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = J; k < i; ++k) {
      uint32_t b[4];
      ldsm_x4(at(aMh, i * 16, k * 16), b);
      mma16816(c0, xa[k - J], b[0], b[1]);
      mma16816(c1, xa[k - J], b[2], b[3]);
    }
    const uint32_t pa[4] = {pack_f16(-c0[0], -c0[1]), pack_f16(-c0[2], -c0[3]),
                            pack_f16(-c1[0], -c1[1]), pack_f16(-c1[2], -c1[3])};
    uint32_t b[4];
    ldsm_x4(at(aXh, i * 16, i * 16), b);
    float x0[4] = {0.f, 0.f, 0.f, 0.f}, x1[4] = {0.f, 0.f, 0.f, 0.f};
    mma16816(x0, pa, b[0], b[1]);
    mma16816(x1, pa, b[2], b[3]);
    if (i < 3) {
      xa[i - J][0] = pack_f16(x0[0], x0[1]);
      xa[i - J][1] = pack_f16(x0[2], x0[3]);
      xa[i - J][2] = pack_f16(x1[0], x1[1]);
      xa[i - J][3] = pack_f16(x1[2], x1[3]);
    }
    // X_iJ^T[s][r] -> Tb row 16 i + r, column 16 J + s, times beta of the column:
    // x0 holds s = g (r = 2q, 2q+1) and s = g + 8; x1 the same for r + 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int s = J * 16 + g + 8 * h;
      const float bs = beta[s];
      const uint32_t cb = static_cast<uint32_t>(s >> 3), co = static_cast<uint32_t>((s & 7) * 2);
      const float* lo = h ? x0 + 2 : x0;
      const float* hi = h ? x1 + 2 : x1;
      const uint32_t r0 = static_cast<uint32_t>(i * 16 + 2 * q);
      sts16(aTb + sw128_offset(r0, cb) + co, __half_as_ushort(__float2half_rn(lo[0] * bs)));
      sts16(aTb + sw128_offset(r0 + 1, cb) + co, __half_as_ushort(__float2half_rn(lo[1] * bs)));
      sts16(aTb + sw128_offset(r0 + 8, cb) + co, __half_as_ushort(__float2half_rn(hi[0] * bs)));
      sts16(aTb + sw128_offset(r0 + 9, cb) + co, __half_as_ushort(__float2half_rn(hi[1] * bs)));
    }
  }
}

// Write one row of the first UMMA's result.  Row rl lies in sub-block BL and
// `val[s]` holds its products with the right-operand segment of that sub-block
// (s = 0 .. 16 BL + 15).  Key rows feed M = diag(beta) A_strict (diagonal block in
// FP32, earlier blocks in FP16); query rows are Aqk (s <= rl), written as FP16
// into the swizzled staging tile of its TMA store.
template <int BL>
__device__ __forceinline__ void emit_rows(const uint32_t* val, bool is_q, int rl, float br,
                                          uint8_t* sm) {
  using namespace prep;
  constexpr int NV = 16 * (BL + 1);
  if (!is_q) {
    // diagonal block, column-major (entry (r, s) at s * 16 + r) for the column solve
    float* Mf = reinterpret_cast<float*>(sm + kMf) + BL * kMfBlk + (rl & 15);
#pragma unroll
    for (int s = 16 * BL; s < 16 * BL + 16; ++s)
      Mf[(s & 15) * 16] = (s < rl) ? br * __uint_as_float(val[s]) : 0.f;
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
    // columns before the row's sub-block are all kept, those after it are zero; only
    // inside the diagonal block does the row index decide (s <= rl)
    const int d = rl & 15;
#pragma unroll
    for (int s0 = 0; s0 < kC; s0 += 8) {
      uint32_t pk[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int s = s0 + 2 * u;
        float a = 0.f, b2 = 0.f;
        if (s < 16 * BL) {
          a = __uint_as_float(val[s]);
          b2 = __uint_as_float(val[s + 1]);
        } else if (s < NV) {
          a = (s - 16 * BL <= d) ? __uint_as_float(val[s]) : 0.f;
          b2 = (s + 1 - 16 * BL <= d) ? __uint_as_float(val[s + 1]) : 0.f;
        }
        pk[u] = pack_f16(a, b2);
      }
      *reinterpret_cast<uint4*>(sm + kAqs + sw128_offset(rl, s0 >> 3)) =
          make_uint4(pk[0], pk[1], pk[2], pk[3]);
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
  if (w < 0x7fffffff) {   // 32-bit divisions (every realistic grid)
    const uint32_t w32 = static_cast<uint32_t>(w), H = static_cast<uint32_t>(p.H);
    it.slot = w32 / H;
    it.h = static_cast<int32_t>(w32 - static_cast<uint32_t>(it.slot) * H);
  } else {
    it.slot = w / p.H;
    it.h = static_cast<int32_t>(w % p.H);
  }
  if (it.slot >= p.slots) return false;
  it.rec = it.slot * p.H + it.h;
  if (p.cu_seqlens == nullptr && p.ckpt_offsets == nullptr) {
    const uint32_t cps = static_cast<uint32_t>((p.fixed_len + kC - 1) / kC);
    const uint32_t s32 = static_cast<uint32_t>(it.slot);   // slot < slots < 2^31 here
    const int32_t n = static_cast<int32_t>(s32 / cps);
    const int32_t j = static_cast<int32_t>(s32 - static_cast<uint32_t>(n) * cps);
    if (n >= p.N) return false;
    const SeqInfo si = seq_info(p, n, false);
    if (j >= si.nch || j >= p.split_jmax) return false;
    chunk_span(si, j, it.t0, it.c);
    it.t0 += si.start;
    return it.c > 0;
  }
  // packed or checkpointed batches: the schedule kernel's slot span, one load
  const int2 v = reinterpret_cast<const int2*>(p.ws + p.lay.slot_span)[it.slot];
  it.t0 = v.x;
  it.c = v.y & 127;
  return it.c > 0 && (v.y >> 7) < p.split_jmax;
}

// Work item w in chunk-major order, used when prepare CTAs feed recurrence CTAs
// of the same launch: chunk j = fused_j0 + w / R of chain c = w % R (R = N H
// chains, in the recurrence grid's order), so every chain's chunk j is prepared
// before any chain's chunk j + 1.
__device__ __forceinline__ bool locate_item_chunk_major(const KdaParams& p, int64_t w, PrepItem& it) {
  const int64_t R = static_cast<int64_t>(p.N) * p.H;
  const int64_t j = p.fused_j0 + w / R, c = w - (w / R) * R;
  int32_t n = static_cast<int32_t>(c / p.H);
  it.h = static_cast<int32_t>(c - static_cast<int64_t>(n) * p.H);
  if (p.cu_seqlens != nullptr) n = reinterpret_cast<const int32_t*>(p.ws + p.lay.seq_order)[n];
  if (n < 0 || n >= p.N) return false;
  const SeqInfo si = seq_info(p, n);
  if (j >= si.nch) return false;
  it.slot = si.slot0 + j;
  if (it.slot < 0 || it.slot >= p.slots) return false;
  chunk_span(si, static_cast<int32_t>(j), it.t0, it.c);
  it.t0 += si.start;
  it.rec = it.slot * p.H + it.h;
  return it.c > 0;
}

// Group-wide barriers of the prepare body: the whole CTA in the split kernel; in a
// CTA of the fused or stream launch, which runs more than one 256-thread group,
// a named barrier of the group's own (`bar`) over the group's threads.
template <bool kFused>
__device__ __forceinline__ void prep_sync(uint32_t bar) {
  if constexpr (kFused) named_bar_sync(bar, prep::kThreads); else __syncthreads();
}
template <bool kFused>
__device__ __forceinline__ bool prep_sync_or(uint32_t bar, bool pred) {
  if constexpr (kFused) return named_bar_or(bar, prep::kThreads, pred);
  else return __syncthreads_or(pred) != 0;
}

// Where a prepare group's tensor memory and barrier come from: its own 256-column
// allocation and named barrier 1 + grp (split and fused launches), or a part of the
// CTA's allocation and a barrier id the caller assigns (stream launch).
struct PrepGroupRes {
  uint32_t tmem;   // kTmemOwn: the group allocates its own 256 columns
  uint32_t bar;    // named barrier id of the group (fused / stream launches)
};
constexpr uint32_t kTmemOwn = 0xFFFFFFFFu;

// Publish a finished record to the recurrence CTAs of the fused launch: its tile
// stores (issued by this thread) are complete and every thread's plain stores
// were ordered before the last CTA barrier.
__device__ __forceinline__ void publish_record(const KdaParams& p, int64_t rec) {
  bulk_wait_all();
  asm volatile("fence.proxy.async.global;" ::: "memory");
  int32_t* flag = reinterpret_cast<int32_t*>(p.ws + p.lay.ready) + rec;
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}

// The prepare loop of one 256-thread group (grp: its index in the CTA; its shared
// memory is the grp-th kGroupBytes slice).  Items first, first + stride, ... <
// nitems; kFused selects the chunk-major item order, the named barriers and the
// ready flags.
// kFE: the input front end is compiled in (switches in p.fe_flags): the gate is formed
// from the raw BF16 gate tile in the scan, the inverse L2 norms of the k and q rows
// are folded into the FP32 factors that already multiply them (so every operand keeps
// its single rounding), and beta is squashed from its logit in FP32.  T diag(beta) is
// an FP16 operand, so the squashed beta on its diagonal keeps 2^-11 relative precision.
template <bool kFused, bool kFE = false, bool kStream = false>
__device__ __forceinline__ void prepare_body(const KdaParams& p, const SplitMaps& maps,
                                             uint8_t* smem_raw, int grp, int64_t first,
                                             int64_t stride, int64_t nitems,
                                             PrepGroupRes res = PrepGroupRes{kTmemOwn, 0u}) {
  using namespace prep;
  uint8_t* sm = smem_align<1024>(smem_raw) + static_cast<uint32_t>(grp) * kGroupBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kAuxBars);
  uint64_t& tma_bar = bars[0];
  uint64_t& mma_bar = bars[1];
  uint64_t& raw_qk_bar = bars[2];
  uint64_t& raw_g_bar = bars[3];
  uint32_t& tmem_slot = *reinterpret_cast<uint32_t*>(sm + kAuxTmem);
  float* s_beta = reinterpret_cast<float*>(sm + kAuxBeta);
  float2 (*s_tot)[64] = reinterpret_cast<float2 (*)[64]>(sm + kAuxTot);     // per sub-block sums of g
  float2 (*s_first)[64] = reinterpret_cast<float2 (*)[64]>(sm + kAuxFirst); // first token's running sum
  float* s_norm = reinterpret_cast<float*>(sm + kAuxNorm);   // front end: 1/|k_r|, then 1/|q_r|
  const bool fe_gate = kFE && (p.fe_flags & 2u) != 0;
  const bool fe_norm = kFE && (p.fe_flags & 1u) != 0;
  const bool fe_beta = kFE && (p.fe_flags & 4u) != 0;
  const uint32_t raw_g_tx = fe_gate ? 16384u : kRawGTx;   // raw gate tile is BF16

  const int tid = threadIdx.x - grp * kThreads;
  const int warp = tid >> 5, lane = tid & 31;
  // packed FP32 pair arithmetic in the element-wise pass (same bits as the scalar
  // form), where the register budget allows it: the split kernel's
  constexpr bool kPack = !kFused;
  const uint32_t gbar = res.bar != 0u ? res.bar : 1u + static_cast<uint32_t>(grp);
  const bool own_tmem = res.tmem == kTmemOwn;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;
  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;
  auto locate = [&](int64_t w, PrepItem& it) {
    if constexpr (kFused) return locate_item_chunk_major(p, w, it);
    else return locate_item(p, w, it);
  };

  if (tid == 0) {
    mbar_init(&tma_bar, 1);
    mbar_init(&mma_bar, 1);
    mbar_init(&raw_qk_bar, 1);
    mbar_init(&raw_g_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.v_in);
    prefetch_tmap(&maps.q_in);
    prefetch_tmap(&maps.k_in);
    prefetch_tmap(&maps.g_in);
    if constexpr (!kStream) {   // (the stream records are written without these maps)
      prefetch_tmap(&maps.wt);
      prefetch_tmap(&maps.ut);
    }
    prefetch_tmap(&maps.aqk);
  }
  if (own_tmem) {
    if (warp == 0) {
      tmem_alloc(&tmem_slot, 256);
      tmem_relinquish();
    }
  } else if (tid == 0) {
    tmem_slot = res.tmem;
  }
  prep_sync<kFused>(gbar);
  tc_fence_after();
  const uint32_t tbase = tmem_slot;
  const uint32_t sbase = smem_u32(sm);
  bool ok = true;
  // Phase bookkeeping of the four mbarriers in one word (fewer registers live across the
  // item loop): for each, bit `kPh*` is the parity of the phases completed so far, i.e.
  // of the number of copies or commits issued, and bit `kPh* << 4` records that at
  // least one was issued.  A wait for the last one uses the complement of its parity bit.
  uint32_t ph = 0;
  constexpr uint32_t kPhTma = 1, kPhMma = 2, kPhQk = 4, kPhG = 8;
  auto bump = [&](uint32_t b) { ph = (ph ^ b) | (b << 4); };
  auto last_parity = [&](uint32_t b) -> uint32_t { return (ph & b) ? 0u : 1u; };
  bool qk_for_cur = false, g_for_cur = false;  // the current item's tiles are in flight
  auto issue_qk = [&](const PrepItem& it) {  // thread 0 only
    mbar_arrive_expect_tx(&raw_qk_bar, kRawQKTx);
    tma_load_3d(sm + kQraw, &maps.q_in, &raw_qk_bar, 0, it.h, it.t0);
    tma_load_3d(sm + kKraw, &maps.k_in, &raw_qk_bar, 0, it.h, it.t0);
  };
  auto issue_g = [&](const PrepItem& it) {  // thread kGThread only, its Aqk stores read
    mbar_arrive_expect_tx(&raw_g_bar, raw_g_tx);
    tma_load_3d(sm + kGraw, &maps.g_in, &raw_g_bar, 0, it.h, it.t0);
  };

  // Item order.  Static: first, first + stride, ...  Claimed (stream launch): thread 0
  // takes the next valid item from a counter in the workspace one item ahead and
  // publishes its index in shared memory; the other threads read it after the first
  // barrier of the iteration (nothing before that barrier needs it but thread 0).
  const bool claim = kFused && p.claim_items != 0;
  int64_t* s_claim = reinterpret_cast<int64_t*>(sm + kAuxClaim);
  auto claim_next = [&](PrepItem& it) -> int64_t {   // thread 0 only
    unsigned long long* ctr = reinterpret_cast<unsigned long long*>(p.ws + p.lay.claim);
    for (;;) {
      const int64_t w = static_cast<int64_t>(atomicAdd(ctr, 1ull));
      if (w >= nitems) return nitems;
      if (locate(w, it)) return w;
    }
  };
  // Static order: the items' chunk spans are looked up kSpanBatch items at a time, one
  // item per thread, into shared memory (one global round trip per batch instead of one
  // on every item's critical path); an item that holds no chunk reads as c = 0.
  int4* s_span = reinterpret_cast<int4*>(sm + kAuxSpan);
  auto load_batch = [&](int32_t i0) {   // items i0 .. i0 + kSpanBatch - 1 of this group
    if (tid < kSpanBatch) {
      const int64_t w = first + static_cast<int64_t>(i0 + tid) * stride;
      PrepItem it;
      int4 v = make_int4(0, 0, 0, 0);
      if (w < nitems && locate(w, it)) v = make_int4(it.t0, it.c, it.h, static_cast<int32_t>(it.rec));
      s_span[tid] = v;
    }
  };
  auto batch_item = [&](int32_t i, PrepItem& it) -> bool {
    const int4 v = s_span[i % kSpanBatch];
    it.t0 = v.x;
    it.c = v.y;
    it.h = v.z;
    it.rec = v.w;
    return v.y > 0;
  };
  // The next valid item from index i of this group's sequence on (-1: none), refilling
  // the batch where it crosses one; every thread of the group takes the same steps, so
  // the refill's barriers match.  The first barrier of a refill ends the reads of the old
  // batch, the second publishes the new entries.
  // (item indices fit 32 bits: there are fewer than 2^31 records)
  const int32_t first32 = static_cast<int32_t>(first), stride32 = static_cast<int32_t>(stride),
                nitems32 = static_cast<int32_t>(nitems);
  int32_t loaded = 0;   // index of the first item of the batch in shared memory
  auto next_valid = [&](int32_t i, PrepItem& it) -> int32_t {
    for (;; ++i) {
      if (first32 + i * stride32 >= nitems32) return -1;
      if (i - loaded >= kSpanBatch) {
        prep_sync<kFused>(gbar);
        loaded = i - i % kSpanBatch;
        load_batch(loaded);
        prep_sync<kFused>(gbar);
      }
      if (batch_item(i, it)) return i;
    }
  };
  PrepItem cur;
  int64_t w0 = first;
  int32_t i_cur = -1;   // static order: index of the current item in the group's sequence
  bool cur_valid;
  if (claim) {
    if (tid == 0) s_claim[0] = claim_next(cur);
    prep_sync<kFused>(gbar);
    w0 = s_claim[0];
    cur_valid = w0 < nitems && locate(w0, cur);
  } else {
    load_batch(0);
    prep_sync<kFused>(gbar);
    i_cur = next_valid(0, cur);
    cur_valid = i_cur >= 0;
    w0 = cur_valid ? first32 + i_cur * stride32 : nitems;
  }
  int64_t pending = -1;   // fused launch: record whose ready flag is still to be raised
  int iter = 0;
  for (int64_t w = w0, w_next = 0; w < nitems && ok; w = w_next, ++iter) {
    PrepItem nxt;
    bool nxt_valid = false;
    if (claim) {
      if (tid == 0) {
        w_next = claim_next(nxt);
        s_claim[(iter + 1) & 1] = w_next;
        nxt_valid = w_next < nitems;
      }
    } else {
      // items that hold no chunk (past the chunk table, or the hybrid's tail rows) are
      // skipped here, so the next item's tiles are always requested one item ahead
      const int32_t i_nxt = next_valid(i_cur + 1, nxt);
      nxt_valid = i_nxt >= 0;
      w_next = nxt_valid ? first32 + i_nxt * stride32 : nitems;
      i_cur = i_nxt;
    }
    if (!cur_valid) {
      cur = nxt;
      cur_valid = nxt_valid;
      continue;
    }
    const int h = cur.h;
    const int32_t t0 = cur.t0, c = cur.c;
    const int64_t rec = cur.rec;

    const int cp = tid & 63;         // channel pair
    const int blk = tid >> 6;        // sub-block 0..3
    if (!qk_for_cur) {
      if (tid == 0) issue_qk(cur);
      bump(kPhQk);
    }
    if (!g_for_cur) {
      if (tid == kGThread) {
        bulk_wait_read();
        issue_g(cur);
      }
      bump(kPhG);
    }
    qk_for_cur = g_for_cur = false;
    uint16_t beta_raw = 0;   // consumed only after the operand pass, so its latency hides
    if (tid < c) beta_raw = p.beta[static_cast<int64_t>(t0 + tid) * p.H + h];
    // front end: the gate's exponent -log2(e) exp(A_log[h]) (a + dt_bias) as a * cz + cb,
    // one FMA per lane of the channel pair
    float2 fe_cz = make_float2(0.f, 0.f), fe_cb = make_float2(0.f, 0.f);
    if constexpr (kFE) {
      if (fe_gate) {
        const float cz = -kLog2e * expf(__ldg(p.A_log + h));
        const float2 dtb =
            __ldg(reinterpret_cast<const float2*>(p.dt_bias + static_cast<int64_t>(h) * kD) + cp);
        fe_cz = make_float2(cz, cz);
        fe_cb = make_float2(cz * dtb.x, cz * dtb.y);
      }
    }

    // ---- raw tiles -> registers: g (float2), k, q (bf16x2) for 16 tokens x 2 channels.
    // One thread waits for the copies; the others sleep in the barrier instead of polling
    // (their polls would take issue slots from the other group on the SM).
    if (tid == 0) {
      ok = mbar_wait(&raw_g_bar, last_parity(kPhG), budget);
      ok = ok && mbar_wait(&raw_qk_bar, last_parity(kPhQk), budget);
    }
    ok = !prep_sync_or<kFused>(gbar, !ok);
    float2 G[16];
    uint32_t kw[16];
    {
      const float2* gs = reinterpret_cast<const float2*>(sm + kGraw) + blk * 16 * 64 + cp;
      const uint32_t* ks = reinterpret_cast<const uint32_t*>(sm + kKraw) + blk * 16 * 64 + cp;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool in = ok && blk * 16 + i < c;   // rows past the chunk read as zero
        if (fe_gate) {
          // g = lower_bound * sigmoid(exp(A_log) (a + dt_bias)) from the raw BF16 gate a
          const uint32_t a2 = in ? reinterpret_cast<const uint32_t*>(sm + kGraw)[(blk * 16 + i) * 64 + cp] : 0u;
          const float2 z = fma2<kPack>(bf2_to_f2(a2), fe_cz, fe_cb);
          // (approximate reciprocal: 1 + 2^z is at least 1, and an infinite denominator
          // gives 0, the limit of the logistic)
          const float2 den = add2<kPack>(make_float2(ex2(z.x), ex2(z.y)), make_float2(1.f, 1.f));
          G[i] = in ? mul2<kPack>(make_float2(rcp_approx(den.x), rcp_approx(den.y)),
                                  make_float2(p.lower_bound, p.lower_bound))
                    : make_float2(0.f, 0.f);
        } else {
          G[i] = in ? gs[i * 64] : make_float2(0.f, 0.f);
        }
        kw[i] = in ? ks[i * 64] : 0u;
      }
    }
    if constexpr (kFE) {
      if (fe_norm) {   // (warp-uniform; on a failed wait the values are never used)
        // inverse L2 norms of the chunk's k and q rows: warp w takes rows 8 w .. 8 w + 7,
        // two rows at a time, half-warp h = lane / 16 one row, lane channels 8 (lane % 16)
        // .. + 7 (the raw tiles are intact until the barrier below)
        const uint4* kr = reinterpret_cast<const uint4*>(sm + kKraw);
        const uint4* qr = reinterpret_cast<const uint4*>(sm + kQraw);
        const int hl = lane & 15;
        // (the partial sums of all four row pairs first, so that no store to s_norm
        // sits between the loads and keeps the later ones waiting)
        float sk[4], sq[4];
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int row = warp * 8 + rr * 2 + (lane >> 4);
          const uint4 kv = kr[row * 16 + hl], qv = qr[row * 16 + hl];
          sk[rr] = 0.f;
          sq[rr] = 0.f;
          const uint32_t kx[4] = {kv.x, kv.y, kv.z, kv.w}, qx[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float2 a = bf2_to_f2(kx[j]), b = bf2_to_f2(qx[j]);
            sk[rr] = fmaf(a.x, a.x, fmaf(a.y, a.y, sk[rr]));
            sq[rr] = fmaf(b.x, b.x, fmaf(b.y, b.y, sq[rr]));
          }
        }
#pragma unroll
        for (int rr = 0; rr < 4; ++rr) {
          const int row = warp * 8 + rr * 2 + (lane >> 4);
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) {
            sk[rr] += __shfl_xor_sync(0xffffffffu, sk[rr], o);
            sq[rr] += __shfl_xor_sync(0xffffffffu, sq[rr], o);
          }
          if (hl == 0) {
            s_norm[row] = rsqrtf(sk[rr] + p.l2_eps);
            s_norm[64 + row] = rsqrtf(sq[rr] + p.l2_eps);
          }
        }
      }
    }
    // ---- gate scan within the sub-block; one exchange gives every sub-block start
    {
      float2 run = make_float2(0.f, 0.f);
      const float2 l2e = make_float2(kLog2e, kLog2e);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        run = fma2<kPack>(G[i], l2e, run);
        G[i] = run;
      }
      s_first[blk][cp] = G[0];
      s_tot[blk][cp] = run;
    }
    // the previous item's TMA stores have finished reading their staging tiles
    if (tid == 0) bulk_wait_read();
    ok = !prep_sync_or<kFused>(gbar, !ok);
    if (!ok) break;
    if (claim && tid != 0) {
      w_next = s_claim[(iter + 1) & 1];
      nxt_valid = w_next < nitems && locate(w_next, nxt);
    }
    float2 Bs[4];   // B_i: G at the first token of sub-block i
    float2 E;       // G at the chunk end
    {
      float2 acc = make_float2(0.f, 0.f), pre = acc;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float2 f = s_first[b][cp], t = s_tot[b][cp];
        Bs[b] = make_float2(acc.x + f.x, acc.y + f.y);
        if (b == blk) pre = acc;
        acc.x += t.x;
        acc.y += t.y;
      }
      E = acc;
#pragma unroll
      for (int i = 0; i < 16; ++i) G[i] = add2<kPack>(G[i], pre);
    }

    // ---- operands
    {
      const float2 B = G[0];
      const float2 cB = make_float2(ex2(B.x), ex2(B.y));                    // 2^B_b
      const float2 cE = make_float2(ex2(E.x - B.x), ex2(E.y - B.y));        // 2^(E - B_b)
      // 2^(B_i - B_b) for the later sub-blocks i = 1, 2, 3 (unused entries never read)
      float2 c1 = make_float2(0.f, 0.f), c2 = c1, c3 = c1;
      if (blk < 1) c1 = make_float2(ex2(Bs[1].x - B.x), ex2(Bs[1].y - B.y));
      if (blk < 2) c2 = make_float2(ex2(Bs[2].x - B.x), ex2(Bs[2].y - B.y));
      if (blk < 3) c3 = make_float2(ex2(Bs[3].x - B.x), ex2(Bs[3].y - B.y));
      const int seg_own = (blk == 0) ? 0 : (blk == 1) ? 16 : (blk == 2) ? 48 : 96;
      // Store addresses.  Row r = 16 blk + i has (r & 7) == (i & 7), so the 128-byte
      // swizzle of every operand row reduces to a per-thread base plus one of eight
      // per-thread XOR terms and a compile-time row offset.
      const uint32_t panel = static_cast<uint32_t>(cp >> 5);
      const uint32_t chunk = static_cast<uint32_t>((cp & 31) >> 2);
      const uint32_t inner = static_cast<uint32_t>((cp & 3) * 4 + blk * 2048);
      const uint32_t bL = sbase + kL + panel * 16384u + inner;
      const uint32_t bR = sbase + kR + panel * 20480u + inner;
      const uint32_t bRo = bR + static_cast<uint32_t>(seg_own) * 128u;
      const uint32_t bKG = sbase + kKG + panel * 8192u + inner;
      const uint32_t c1b = pack_bf16(c1.x, c1.y), c2b = pack_bf16(c2.x, c2.y),
                     c3b = pack_bf16(c3.x, c3.y);
      // Q Gamma and Kd token rows: this thread's channel pair of rows 16 blk + i
      // (the stream records keep Q Gamma as rows 0..63 of the [Q Gamma; W] tile)
      uint32_t* qg_out = reinterpret_cast<uint32_t*>(
                             kStream ? p.ws + p.lay.qw + rec * kTileQW : p.ws + p.lay.qg + rec * kTileQG) +
                         blk * 16 * 64 + cp;
      uint32_t* kd_out = reinterpret_cast<uint32_t*>(p.ws + p.lay.kd + rec * kTileKd) + blk * 16 * 64 + cp;
      const float2 nB = make_float2(-B.x, -B.y);
      // the raw q tile, row by row (rows past the chunk read as zero)
      const uint32_t* qs = reinterpret_cast<const uint32_t*>(sm + kQraw) + blk * 16 * 64 + cp;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t xo = ((chunk ^ static_cast<uint32_t>(i & 7)) << 4) + static_cast<uint32_t>(i) * 128u;
        const uint32_t qv = (blk * 16 + i < c) ? qs[i * 64] : 0u;
        const float2 d = add2<kPack>(G[i], nB);                 // G_r - B_b
        const float2 e = make_float2(ex2(d.x), ex2(d.y));       // e_r
        float2 inv = make_float2(ex2(-d.x), ex2(-d.y));         // 1 / e_r
        const float2 kf = bf2_to_f2(kw[i]), qf = bf2_to_f2(qv);
        const float2 gam = mul2<kPack>(e, cB);                  // Gamma_r, FP32
        if (kFE && fe_norm) {
          // front end: the row's inverse norms ride on the FP32 factors (one rounding each)
          const float rk = s_norm[blk * 16 + i], rq = s_norm[64 + blk * 16 + i];
          const float2 rk2 = make_float2(rk, rk), rq2 = make_float2(rq, rq);
          const uint32_t e2k = pack_bf16(mul2<kPack>(e, rk2)), e2q = pack_bf16(mul2<kPack>(e, rq2));
          sts32(bL + xo, hmul2_bf16(kw[i], e2k));
          sts32(bL + xo + 64u * 128u, hmul2_bf16(qv, e2q));
          const uint32_t rd2 = hmul2_bf16(kw[i], pack_bf16(mul2<kPack>(inv, rk2)));
          sts32(bRo + xo, rd2);
          if (blk < 1) sts32(bR + xo + 16u * 128u, hmul2_bf16(rd2, c1b));
          if (blk < 2) sts32(bR + xo + 48u * 128u, hmul2_bf16(rd2, c2b));
          if (blk < 3) sts32(bR + xo + 96u * 128u, hmul2_bf16(rd2, c3b));
          sts32(bKG + xo, pack_f16(mul2<kPack>(kf, mul2<kPack>(gam, rk2))));
          qg_out[i * 64] = pack_f16(mul2<kPack>(qf, mul2<kPack>(gam, rq2)));
          inv = mul2<kPack>(inv, rk2);
        } else {
          // bf16 operands: factors rounded to bf16, products in packed bf16 math
          const uint32_t e2 = pack_bf16(e), inv2 = pack_bf16(inv);
          sts32(bL + xo, hmul2_bf16(kw[i], e2));
          sts32(bL + xo + 64u * 128u, hmul2_bf16(qv, e2));
          const uint32_t rd2 = hmul2_bf16(kw[i], inv2);
          sts32(bRo + xo, rd2);
          if (blk < 1) sts32(bR + xo + 16u * 128u, hmul2_bf16(rd2, c1b));
          if (blk < 2) sts32(bR + xo + 48u * 128u, hmul2_bf16(rd2, c2b));
          if (blk < 3) sts32(bR + xo + 96u * 128u, hmul2_bf16(rd2, c3b));
          // K Gamma (A of the W UMMA) and Q Gamma (B of the state read): FP16 products of
          // FP32 factors, one rounding each
          sts32(bKG + xo, pack_f16(mul2<kPack>(kf, gam)));
          qg_out[i * 64] = pack_f16(mul2<kPack>(qf, gam));
        }
        // Kd feeds the FP16 state update: FP32 products, one rounding
        kd_out[i * 64] = pack_f16(mul2<kPack>(mul2<kPack>(kf, inv), cE));
      }
      if (blk == 0)
        reinterpret_cast<float2*>(p.ws + p.lay.gc + rec * kTileGC)[cp] =
            make_float2(ex2(E.x), ex2(E.y));
    }
    if (tid < kC) {
      // beta (or, from raw projections, sigmoid of its BF16 logit, in FP32): it scales M
      // in FP32 and reaches the tensor core only through the FP16 T diag(beta)
      const float b = bf16_to_f32(beta_raw);
      s_beta[tid] = fe_beta ? 1.f / (1.f + ex2(-b * kLog2e)) : b;
    }

    // ---- UMMA 1: D[0:128, 0:160] = [K+; Q+] . R^T   (bf16 -> f32)
    fence_proxy_async_smem();
    tc_fence_before();
    prep_sync<kFused>(gbar);
    // every thread has read the raw q tile: the v tile goes there now, by TMA straight
    // into the MN-major A operand of U^T
    if (tid == 0) {
      mbar_arrive_expect_tx(&tma_bar, 16384);
      tma_load_3d(sm + kV, &maps.v_in, &tma_bar, 0, h, t0);
      tma_load_3d(sm + kV + 8192, &maps.v_in, &tma_bar, 64, h, t0);
    }
    bump(kPhTma);
    const uint32_t tma_parity = last_parity(kPhTma);
    if (tid == 0) {
      tc_fence_after();
      const uint32_t idesc = idesc_f16(128, 160, kFmtBF16, kKMajor, kKMajor);
      const uint32_t aL = sbase + kL, aR = sbase + kR;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint64_t ad = sdesc_sw128(aL + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        const uint64_t bd = sdesc_sw128(aR + (kk >> 2) * 20480 + (kk & 3) * 32, 16, 1024);
        umma_f16(tbase, ad, bd, idesc, kk > 0);
      }
      umma_commit(&mma_bar);
      if constexpr (kFused) {
        // the previous record's tile stores were issued a whole element-wise pass
        // ago and are long complete: publish it while this UMMA runs
        if (pending >= 0) publish_record(p, pending);
      }
    }
    if constexpr (kFused) pending = -1;
    // While the first UMMA runs, one otherwise idle thread prefetches the next item's
    // tiles (q, k, g, v) and beta rows into L2.
    if (tid == kPrefetchThread && nxt_valid) {
        tma_prefetch_3d(&maps.q_in, 0, nxt.h, nxt.t0);
        tma_prefetch_3d(&maps.k_in, 0, nxt.h, nxt.t0);
        tma_prefetch_3d(&maps.g_in, 0, nxt.h, nxt.t0);
        tma_prefetch_3d(&maps.v_in, 0, nxt.h, nxt.t0);
        tma_prefetch_3d(&maps.v_in, 64, nxt.h, nxt.t0);
        // beta rows of the next chunk, all heads: 16-byte aligned and inside the tensor
        const uintptr_t lo =
            reinterpret_cast<uintptr_t>(p.beta + static_cast<int64_t>(nxt.t0) * p.H) & ~uintptr_t(15);
        uintptr_t hi = (reinterpret_cast<uintptr_t>(p.beta + static_cast<int64_t>(nxt.t0 + nxt.c) * p.H) + 15) &
                       ~uintptr_t(15);
        const uintptr_t lim =
            reinterpret_cast<uintptr_t>(p.beta + static_cast<int64_t>(p.T) * p.H) & ~uintptr_t(15);
        hi = hi < lim ? hi : lim;
        if (hi > lo) bulk_prefetch_l2(reinterpret_cast<const void*>(lo), static_cast<uint32_t>(hi - lo));
      }
    bump(kPhMma);
    if (tid == 0) ok = mbar_wait(&mma_bar, last_parity(kPhMma), budget);
    ok = !prep_sync_or<kFused>(gbar, !ok);
    if (ok) {
      tc_fence_after();
      // ---- extract A (lane quarters 0,1) and Aqk (quarters 2,3): row rl, sub-block bl.
      // Warps w and w + 4 share a lane quarter; warp w reads the column segment of
      // the first sub-block its rows hold, warp w + 4 that of the second, so at most
      // 64 accumulator values are live per thread and all eight warps take part.
      const int qw4 = warp & 3, phase = warp >> 2;
      const int rl = (qw4 & 1) * 32 + lane;
      const int bl = rl >> 4;
      const bool is_q = qw4 >= 2;
      const uint32_t lane_base = static_cast<uint32_t>(qw4 * 32);
      const float br = s_beta[rl];
      if ((qw4 & 1) == 0) {
        if (phase == 0) {
          uint32_t v[16];
          tmem_ld16(tmem_addr(tbase, lane_base, 0), v);
          tmem_wait_ld();
          if (bl == 0) emit_rows<0>(v, is_q, rl, br, sm);
        } else {
          uint32_t v[32];
          tmem_ld32(tmem_addr(tbase, lane_base, 16), v);
          tmem_wait_ld();
          if (bl == 1) emit_rows<1>(v, is_q, rl, br, sm);
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
          if (bl == 2) emit_rows<2>(v, is_q, rl, br, sm);
        } else {
          uint32_t v[64], ta[32], tb[32];
          tmem_ld32(tmem_addr(tbase, lane_base, 96), ta);
          tmem_ld32(tmem_addr(tbase, lane_base, 128), tb);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            v[i] = ta[i];
            v[32 + i] = tb[i];
          }
          if (bl == 3) emit_rows<3>(v, is_q, rl, br, sm);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    prep_sync<kFused>(gbar);
    if (ok && tid == kGThread) {
      tma_store_2d(&maps.aqk, sm + kAqs, 0, static_cast<int32_t>(rec * 64));
      bulk_commit();
    }
    // R (UMMA1's operand, then the Aqk staging tile) is free once that store has read
    // it: kGThread requests the next item's g tile there during the off-diagonal solve,
    // where its warp is idle (so waiting for the store does not hold up the diagonal
    // phase), a whole UMMA 2 early
    const bool g_next = ok && nxt_valid;
    if (g_next) {
      bump(kPhG);
      g_for_cur = true;   // (for the next iteration)
    }

    if (ok) {
      __half* Xh = reinterpret_cast<__half*>(sm + kXh);
      const uint32_t aMh = sbase + kMh, aXh = sbase + kXh, aTb = sbase + kTb;
      if (tid < 64) {
        // ---- diagonal blocks X_bb = (I + M_bb)^-1 in FP32, one column per thread,
        // right-looking: once x[ss] is final it is folded into every later row, so the
        // dependent chain is one FMA per row (the later rows' updates are independent)
        const int bi = tid >> 4, jj = tid & 15;
        const float* Mc = reinterpret_cast<const float*>(sm + kMf) + bi * kMfBlk;   // [s][r]
        const float4* Mc4 = reinterpret_cast<const float4*>(Mc);   // 16-byte aligned columns
        float x[16];
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) x[rr] = (rr == jj) ? 1.f : 0.f;
#pragma unroll
        for (int ss = 0; ss < 15; ++ss) {
          const float xs = x[ss];
#pragma unroll
          for (int q4 = (ss + 1) >> 2; q4 < 4; ++q4) {
            const float4 m = Mc4[ss * 4 + q4];
            const float mv[4] = {m.x, m.y, m.z, m.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (4 * q4 + e > ss) x[4 * q4 + e] = fmaf(-mv[e], xs, x[4 * q4 + e]);
          }
        }
        const int col = bi * 16 + jj;
        const float bcol = s_beta[col];
        __half* tbp = reinterpret_cast<__half*>(sm + kTb + (col & 7) * 2);
#pragma unroll
        for (int rr = 0; rr < 16; ++rr) {
          Xh[(bi * 16 + rr) * kLdh + col] = __float2half_rn(x[rr]);
          tbp[sw128_offset(bi * 16 + rr, col >> 3) >> 1] = __float2half_rn(x[rr] * bcol);
        }
      } else {
        // ---- strictly upper blocks of Tb are zero
        for (int slot = tid - 64; slot < 64 * 8; slot += kThreads - 64) {
          const int r = slot >> 3, ch = slot & 7;
          if (ch >= 2 * ((r >> 4) + 1))
            *reinterpret_cast<uint4*>(sm + kTb + sw128_offset(r, ch)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      prep_sync<kFused>(gbar);
      // ---- off-diagonal blocks, one block column j per warp, down the column:
      //   X_ij = -X_ii (sum_{k=j}^{i-1} M_ik X_kj),  i = j+1 .. 3,
      // FP16 mma.sync with FP32 accumulation.  Column j only reads its own earlier
      // blocks (held in registers) and the diagonal blocks, so the warps need no
      // barrier between levels.
      if (warp < 3) {
        if (warp == 0) offdiag_column<0>(aMh, aXh, aTb, s_beta, lane);
        else if (warp == 1) offdiag_column<1>(aMh, aXh, aTb, s_beta, lane);
        else offdiag_column<2>(aMh, aXh, aTb, s_beta, lane);
      } else if (warp == 7) {
        if (tid == kGThread && g_next) {
          bulk_wait_read();
          issue_g(nxt);
        }
      } else {
        // ---- warps 3-6: the v tile (BF16, landed by TMA in its operand layout) becomes FP16 in
        // place: the U UMMA multiplies it by the FP16 T diag(beta), and both operands of
        // one UMMA share a type (BF16 -> FP16 is exact for |v| in the FP16 normal range)
        if (mbar_wait(&tma_bar, tma_parity, budget)) {
          uint4* vt = reinterpret_cast<uint4*>(sm + kV);
          for (int i = tid - 96; i < 16384 / 16; i += 128) {
            const uint4 x = vt[i];
            const float2 a = bf2_to_f2(x.x), b = bf2_to_f2(x.y), c2 = bf2_to_f2(x.z),
                         d = bf2_to_f2(x.w);
            vt[i] = make_uint4(pack_f16(a.x, a.y), pack_f16(b.x, b.y), pack_f16(c2.x, c2.y),
                               pack_f16(d.x, d.y));
          }
        } else {
          ok = false;
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = !prep_sync_or<kFused>(gbar, !ok);

    // ---- UMMA 2: W^T = (K Gamma)^T (T diag beta)^T -> cols [0,64); U^T = V^T (T diag beta)^T -> [64,128)
    bool tma_seen = false;
    if (ok && tid == 0) {
      tma_seen = mbar_wait(&tma_bar, tma_parity, budget);
      if (tma_seen) {
        tc_fence_after();
        if constexpr (kStream) {
          // token rows [U | W] = (T diag beta) [V | K Gamma]: A = T diag(beta) as rows
          // 64..127 of an M = 128 operand (rows 0..63 read the 8 KB below it; their
          // products land in TMEM lanes 0..63, which no one reads); B = [V | K Gamma],
          // MN-major, four 64-column panels 8 KB apart (V, then K Gamma); N = 256
          const uint32_t idesc = idesc_f16(128, 256, kFmtF16, kKMajor, kMNMajor);
          const uint32_t aT = sbase + kTb - 8192, bVK = sbase + kV;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_f16(tbase, sdesc_sw128(aT + kk * 32, 16, 1024), sdesc_sw128(bVK + kk * 2048, 8192, 1024),
                     idesc, kk > 0);
        } else {
          const uint32_t idesc = idesc_f16(128, 64, kFmtF16, kMNMajor, kKMajor);
          const uint32_t aKG = sbase + kKG, aV = sbase + kV, bT = sbase + kTb;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = sdesc_sw128(bT + kk * 32, 16, 1024);
            umma_f16(tbase + 0, sdesc_sw128(aKG + kk * 2048, 8192, 1024), bd, idesc, kk > 0);
            umma_f16(tbase + 64, sdesc_sw128(aV + kk * 2048, 8192, 1024), bd, idesc, kk > 0);
          }
        }
        umma_commit(&mma_bar);
      }
    }
    if (tid == 0 && !tma_seen) ok = false;
    if (tid == 0 && ok) {
      bump(kPhMma);
      ok = mbar_wait(&mma_bar, last_parity(kPhMma), budget);
    }
    ok = !prep_sync_or<kFused>(gbar, !ok);
    // the next item's q and k tiles go into v / K Gamma, free now that the second
    // UMMA has completed
    if (ok && nxt_valid) {
      if (tid == 0) issue_qk(nxt);
      bump(kPhQk);
      qk_for_cur = true;
    }
    if (ok && kStream) {
      tc_fence_after();
      // TMEM lanes 64..127 hold token row r = lane - 64 of [U | W]: warps 2, 3 write the
      // U row, warps 6, 7 the W row (into rows 64..127 of the [Q Gamma; W] tile), each
      // 128 FP16 values = 256 contiguous bytes
      if ((warp & 3) >= 2) {
        const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32);
        const int r = ((warp & 3) - 2) * 32 + lane;
        const bool is_w = warp >= 4;
        uint4* dst = reinterpret_cast<uint4*>(
            is_w ? p.ws + p.lay.qw + rec * kTileQW + static_cast<int64_t>(64 + r) * 256
                 : p.ws + p.lay.u + rec * kTileU + static_cast<int64_t>(r) * 256);
        const uint32_t col0 = is_w ? 128u : 0u;
        uint32_t a[32];
#pragma unroll
        for (int part = 0; part < 4; ++part) {
          tmem_ld32(tmem_addr(tbase, lane_base, col0 + part * 32), a);
          tmem_wait_ld();
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const float* f = reinterpret_cast<const float*>(a) + q8 * 8;
            dst[part * 4 + q8] = make_uint4(pack_f16(f[0], f[1]), pack_f16(f[2], f[3]),
                                            pack_f16(f[4], f[5]), pack_f16(f[6], f[7]));
          }
        }
      }
    } else if (ok) {
      tc_fence_after();
      // warps 0-3: W^T rows (lane = k); warps 4-7: U^T rows (lane = v), into the
      // swizzled staging tiles of the TMA stores
      const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32);
      const int row = (warp & 3) * 32 + lane;
      const bool is_u = warp >= 4;
      uint8_t* dst = sm + (is_u ? kUs : kWs);
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
          o = make_uint4(pack_f16(f[0], f[1]), pack_f16(f[2], f[3]), pack_f16(f[4], f[5]),
                         pack_f16(f[6], f[7]));
          *reinterpret_cast<uint4*>(dst + sw128_offset(row, part * 4 + q8)) = o;
        }
      }
    }

    // next item: every thread is done with this item's TMEM and shared tiles
    if constexpr (kFused) {
      // the record is published by thread 0 after this barrier: the Aqk store of
      // kGThread has to be complete by then
      if (tid == kGThread) {
        bulk_wait_all();
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    ok = !prep_sync_or<kFused>(gbar, !ok);
    if (ok && tid == 0 && !kStream) {
      tma_store_2d(&maps.wt, sm + kWs, 0, static_cast<int32_t>(rec * 128));
      tma_store_2d(&maps.ut, sm + kUs, 0, static_cast<int32_t>(rec * 128));
      bulk_commit();
    }
    if (ok) pending = rec;
    cur = nxt;
    cur_valid = nxt_valid;
  }

  // ---- teardown: on any failure record it, drain what was issued, free TMEM
  if (tid == 0) {
    if (!ok) {
      record_status(p.ws, kStatusTimeout);
      // copies and commits complete in issue order: waiting for the last drains all
      if (ph & (kPhTma << 4)) mbar_wait(&tma_bar, last_parity(kPhTma), drain_budget);
      if (ph & (kPhMma << 4)) mbar_wait(&mma_bar, last_parity(kPhMma), drain_budget);
      if (ph & (kPhQk << 4)) mbar_wait(&raw_qk_bar, last_parity(kPhQk), drain_budget);
    }
    bulk_wait_all();   // the tile stores this thread issued are complete
    if constexpr (kFused) {
      if (ok && pending >= 0) publish_record(p, pending);
    }
  }
  if (tid == kGThread) {
    if (!ok && (ph & (kPhG << 4))) mbar_wait(&raw_g_bar, last_parity(kPhG), drain_budget);
    bulk_wait_all();
  }
  tc_fence_before();
  prep_sync<kFused>(gbar);
  if (own_tmem && warp == 0) tmem_dealloc(tbase, 256);
}

}  // namespace kda
