// kda_prepare.cu — chunk-local prepare kernel (split variant).
//
// One CTA per (chunk slot, head).  For its 64-token chunk it forms the
// decay-weighted intra-chunk products, solves the unit-lower-triangular UT/WY
// system and writes the per-chunk operands the recurrence kernel consumes:
//   W^T, (Q*Gamma)^T (bf16), U^T, Kd^T (f16), Aqk (f16), Gamma_end (f32)
// (north star subsystem (a): "a chunk-local prepare kernel that forms the
// decay-weighted intra-chunk products, solves the unit-lower-triangular UT/WY
// system per chunk and emits W and U"; the split into prepare and recurrence
// launches is the "decomp" variant of FlashInfer PR #4633 "Description").
//
// Decay factorisation (all in the log2 domain, G2 = cumsum(g * log2 e)):
//   sub-block b = r / 16, reference B_b = G2 at the first token of block b.
//   Left operand   L_r    = k_r * 2^(G2_r - B_b)       (<= 1, >= 2^-116)
//   Right operand  R^i_s  = k_s * 2^(B_i - G2_s)       for s <= 16 i + 15
//   A[r, s] = L_r . R^{b(r)}_s   for every s in blocks 0..b(r):
//     s in block b(r): exponents cancel exactly within one sub-block (|.| <= 80 nats);
//     s before block b(r): both factors are <= 1 (monotone G), underflow harmless.
// The query rows use the same right operand, so one UMMA of M = 128
// ([K+; Q+]) by N = 160 (R^0..R^3 stacked: 16 + 32 + 48 + 64 rows) yields both
// A (strict lower part) and Aqk (lower part including the diagonal).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kda_common.cuh"
#include "sm100_primitives.cuh"

namespace kda {

namespace prep {
constexpr uint32_t kV = 0;           // 16 KB  v tile, MN-major A of U^T: 2 panels [64 tok][64 v]
constexpr uint32_t kKG = 16384;      // 16 KB  K*Gamma tile, MN-major A of W^T
constexpr uint32_t kL = 32768;       // 32 KB  [K+; Q+], K-major A: 2 panels [128 rows][64 ch]
constexpr uint32_t kR = 65536;       // 40 KB  R^0..R^3, K-major B: 2 panels [160 rows][64 ch]
constexpr uint32_t kBytes = 65536 + 40960;
// aliases, valid once the first UMMA has completed
constexpr uint32_t kM = 32768;               // f32 [64][65]  beta_r * A[r][s] (s < r)
constexpr uint32_t kX = kM + 64 * 65 * 4;    // f32 [64][65]  T = (I + M)^-1
constexpr uint32_t kY = kX + 64 * 65 * 4;    // f32 [3][16][17] block products
constexpr uint32_t kTb = 98304;              // 8 KB  T diag(beta) bf16, K-major [64 r][64 s]
constexpr int kLd = 65;
constexpr uint32_t kSmemAlloc = kBytes + 1024;
extern const uint32_t kSmemAllocBytes = kSmemAlloc;
}  // namespace prep

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float x) {
  *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(x);
}

// Offset of element (row, ch) in a 2-panel, 128B-swizzled [rows][128] 16-bit tile.
__device__ __forceinline__ uint32_t tile_off(uint32_t rows, uint32_t row, uint32_t ch) {
  return (ch >> 6) * (rows * 128u) + sw128_offset(row, (ch & 63u) >> 3) + ((ch & 7u) << 1);
}

__global__ void __launch_bounds__(128, 2)
kda_prepare_kernel(const KdaParams p, const __grid_constant__ SplitMaps maps) {
  using namespace prep;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t tma_bar, mma_bar;
  __shared__ uint32_t tmem_slot;
  __shared__ float s_beta[kC];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.y;
  const int64_t slot = blockIdx.x;
  if ((p.flags & kFlagValidate) && reinterpret_cast<const WsHeader*>(p.ws)->call_ok == 0) return;

  // ---- which chunk is this?  (uniform per CTA)
  int32_t n = 0, j = 0;
  if (p.cu_seqlens == nullptr) {
    const int32_t cps = (p.fixed_len + kC - 1) / kC;
    n = static_cast<int32_t>(slot / cps);
    j = static_cast<int32_t>(slot % cps);
  } else {
    const int32_t* cb = reinterpret_cast<const int32_t*>(p.ws + p.lay.chunk_base);
    if (slot >= cb[p.N]) return;
    int32_t lo = 0, hi = p.N;  // largest n with cb[n] <= slot
    while (hi - lo > 1) {
      const int32_t mid = (lo + hi) >> 1;
      if (cb[mid] <= slot) lo = mid; else hi = mid;
    }
    n = lo;
    j = static_cast<int32_t>(slot - cb[n]);
  }
  if (n >= p.N) return;
  const SeqInfo si = seq_info(p, n);
  const int32_t t0 = si.start + j * kC;
  const int32_t c = min(kC, si.len - j * kC);  // valid tokens in this chunk
  if (c <= 0) return;
  const int64_t rec = slot * p.H + h;
  if (slot >= p.slots) return;

  // checkpoint inside this chunk?  local prefix length rp in [1, 64]
  int32_t rp = 0;
  if (p.ckpt_offsets != nullptr) {
    const int32_t off = p.ckpt_offsets[n];
    if (off >= 1 && off <= si.len && (off - 1) / kC == j) rp = off - j * kC;
  }

  const long long budget = p.wait_budget;
  const long long drain_budget = 4000000000LL;

  if (tid == 0) {
    mbar_init(&tma_bar, 1);
    mbar_init(&mma_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_slot, 256);
    tmem_relinquish();
  }
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = tmem_slot;

  // ---- TMA: v tile straight into the MN-major A operand of U^T
  if (tid == 0) {
    prefetch_tmap(&maps.v_in);
    mbar_arrive_expect_tx(&tma_bar, 16384);
    tma_load_3d(sm + kV, &maps.v_in, &tma_bar, 0, h, t0);
    tma_load_3d(sm + kV + 8192, &maps.v_in, &tma_bar, 64, h, t0);
  }

  // ---- beta (zero beyond the valid tokens masks their rows and columns)
  if (tid < kC) {
    float b = 0.f;
    if (tid < c) {
      const uint16_t raw = p.beta[static_cast<int64_t>(t0 + tid) * p.H + h];
      b = bf16_to_f32(raw);
    }
    s_beta[tid] = b;
  }

  // ---- pass 1: gate cumsum for channel ch = tid over the chunk (log2 domain)
  const int ch = tid;
  float G2[kC];
  {
    const float* gp = p.g + (static_cast<int64_t>(t0) * p.H + h) * kD + ch;
    const int64_t stride = static_cast<int64_t>(p.H) * kD;
    float run = 0.f;
#pragma unroll
    for (int r = 0; r < kC; ++r) {
      const float gv = (r < c) ? __ldg(gp + r * stride) : 0.f;
      run = fmaf(gv, kLog2e, run);
      G2[r] = run;
    }
  }
  float Gp = 0.f;  // G2 at the checkpoint's last token
#pragma unroll
  for (int r = 0; r < kC; ++r)
    if (r == rp - 1) Gp = G2[r];

  const float Gend = G2[kC - 1];
  const float B0 = G2[0], B1 = G2[16], B2 = G2[32], B3 = G2[48];

  // ---- pass 2: operands for every token
  {
    const uint16_t* kp = p.k + (static_cast<int64_t>(t0) * p.H + h) * kD + ch;
    const uint16_t* qp = p.q + (static_cast<int64_t>(t0) * p.H + h) * kD + ch;
    const int64_t stride = static_cast<int64_t>(p.H) * kD;
    uint8_t* wsb = p.ws;
    __half* kdt_row = reinterpret_cast<__half*>(wsb + p.lay.kdt + rec * kTileKdT) + ch * 64;
    __nv_bfloat16* qgt_row =
        reinterpret_cast<__nv_bfloat16*>(wsb + p.lay.qgt + rec * kTileQGT) + ch * 64;
    __half* kpt_row = nullptr;
    if (rp > 0)
      kpt_row = reinterpret_cast<__half*>(wsb + p.lay.kpt +
                                          (static_cast<int64_t>(n) * p.H + h) * kTileKdT) +
                ch * 64;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      float kv[16], qv[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = b * 16 + i;
        kv[i] = (r < c) ? bf16_to_f32(__ldg(kp + r * stride)) : 0.f;
        qv[i] = (r < c) ? bf16_to_f32(__ldg(qp + r * stride)) : 0.f;
      }
      const float Bb = (b == 0) ? B0 : (b == 1) ? B1 : (b == 2) ? B2 : B3;
      uint32_t qg_pack[8], kd_pack[8], kp_pack[8];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const int r = b * 16 + i;
        const float G = G2[r];
        const float e = ex2(G - Bb);
        const float inv = ex2(Bb - G);
        // [K+; Q+]
        st_bf16(sm + kL, tile_off(128, r, ch), kv[i] * e);
        st_bf16(sm + kL, tile_off(128, 64 + r, ch), qv[i] * e);
        // right operand rows of segments i' >= b: R^{i'}_r = k_r 2^(B_{i'} - G_r)
        st_bf16(sm + kR, tile_off(160, (b == 0 ? 0 : b == 1 ? 16 : b == 2 ? 48 : 96) + r, ch),
                kv[i] * inv);
        if (b < 1) st_bf16(sm + kR, tile_off(160, 16 + r, ch), kv[i] * ex2(B1 - G));
        if (b < 2) st_bf16(sm + kR, tile_off(160, 48 + r, ch), kv[i] * ex2(B2 - G));
        if (b < 3) st_bf16(sm + kR, tile_off(160, 96 + r, ch), kv[i] * ex2(B3 - G));
        // K * Gamma (MN-major A of W^T) and (Q * Gamma)^T, Kd^T, Kp^T rows
        const float gam = ex2(G);
        st_bf16(sm + kKG, tile_off(64, r, ch), kv[i] * gam);
        const float qg = qv[i] * gam;
        const float kd = kv[i] * ex2(Gend - G);
        const float kpv = (r < rp) ? kv[i] * ex2(Gp - G) : 0.f;
        if (i & 1) {
          qg_pack[i >> 1] |= static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(qg))) << 16;
          kd_pack[i >> 1] |= static_cast<uint32_t>(__half_as_ushort(__float2half_rn(kd))) << 16;
          kp_pack[i >> 1] |= static_cast<uint32_t>(__half_as_ushort(__float2half_rn(kpv))) << 16;
        } else {
          qg_pack[i >> 1] = __bfloat16_as_ushort(__float2bfloat16_rn(qg));
          kd_pack[i >> 1] = __half_as_ushort(__float2half_rn(kd));
          kp_pack[i >> 1] = __half_as_ushort(__float2half_rn(kpv));
        }
      }
      uint4* qd = reinterpret_cast<uint4*>(qgt_row + b * 16);
      qd[0] = make_uint4(qg_pack[0], qg_pack[1], qg_pack[2], qg_pack[3]);
      qd[1] = make_uint4(qg_pack[4], qg_pack[5], qg_pack[6], qg_pack[7]);
      uint4* kd4 = reinterpret_cast<uint4*>(kdt_row + b * 16);
      kd4[0] = make_uint4(kd_pack[0], kd_pack[1], kd_pack[2], kd_pack[3]);
      kd4[1] = make_uint4(kd_pack[4], kd_pack[5], kd_pack[6], kd_pack[7]);
      if (rp > 0) {
        uint4* kq = reinterpret_cast<uint4*>(kpt_row + b * 16);
        kq[0] = make_uint4(kp_pack[0], kp_pack[1], kp_pack[2], kp_pack[3]);
        kq[1] = make_uint4(kp_pack[4], kp_pack[5], kp_pack[6], kp_pack[7]);
      }
    }
    reinterpret_cast<float*>(wsb + p.lay.gc + rec * kTileGC)[ch] = ex2(Gend);
    if (rp > 0)
      reinterpret_cast<float*>(wsb + p.lay.gp + (static_cast<int64_t>(n) * p.H + h) * kTileGC)[ch] =
          ex2(Gp);
  }

  // ---- UMMA 1: D[0:128, 0:160] = [K+; Q+] . R^T   (bf16 -> f32)
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  bool ok = true;
  int mma_commits = 0;
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
  mma_commits = 1;
  ok = mbar_wait(&mma_bar, 0, budget);
  ok = !__syncthreads_or(!ok);
  if (ok) {
    tc_fence_after();
    // ---- extract A (warps 0,1) and Aqk (warps 2,3): row rl, block bl
    const int rl = (warp & 1) * 32 + lane;
    const int bl = rl >> 4;
    const bool is_q = warp >= 2;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32);
    float row[kC];
    if ((warp & 1) == 0) {
      uint32_t w[48];
      uint32_t a32[32], a16[16];
      tmem_ld32(tmem_addr(tbase, lane_base, 0), a32);
      tmem_ld16(tmem_addr(tbase, lane_base, 32), a16);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) w[i] = a32[i];
#pragma unroll
      for (int i = 0; i < 16; ++i) w[32 + i] = a16[i];
#pragma unroll
      for (int s = 0; s < kC; ++s) {
        float x = 0.f;
        if (s < 16 && bl == 0) x = __uint_as_float(w[s]);
        if (s < 32 && bl == 1) x = __uint_as_float(w[16 + s]);
        row[s] = x;
      }
    } else {
      uint32_t w[112];
      uint32_t a32[32], a16[16];
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        tmem_ld32(tmem_addr(tbase, lane_base, 48 + part * 32), a32);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) w[part * 32 + i] = a32[i];
      }
      tmem_ld16(tmem_addr(tbase, lane_base, 144), a16);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 16; ++i) w[96 + i] = a16[i];
#pragma unroll
      for (int s = 0; s < kC; ++s) {
        float x = 0.f;
        if (s < 48 && bl == 2) x = __uint_as_float(w[s]);
        if (bl == 3) x = __uint_as_float(w[48 + s]);
        row[s] = x;
      }
    }
    if (!is_q) {
      float* M = reinterpret_cast<float*>(sm + kM);
      const float br = s_beta[rl];
#pragma unroll
      for (int s = 0; s < kC; ++s) M[rl * kLd + s] = (s < rl) ? br * row[s] : 0.f;
    } else {
      __half* dst = reinterpret_cast<__half*>(p.ws + p.lay.aqk + rec * kTileAqk) + rl * 64;
#pragma unroll
      for (int s0 = 0; s0 < kC; s0 += 8) {
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = s0 + 2 * u;
          const float a = (s <= rl) ? row[s] : 0.f;
          const float b2 = (s + 1 <= rl) ? row[s + 1] : 0.f;
          pk[u] = pack_f16(a, b2);
        }
        *reinterpret_cast<uint4*>(dst + s0) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();

  if (ok) {
    // ---- blocked inverse of the unit lower triangular I + M (M strictly lower)
    const float* M = reinterpret_cast<const float*>(sm + kM);
    float* X = reinterpret_cast<float*>(sm + kX);
    float* Y = reinterpret_cast<float*>(sm + kY);
    if (tid < 64) {
      const int bi = tid >> 4, jj = tid & 15;
      const int o = bi * 16;
      float x[16];
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) {
        float acc = 0.f;
#pragma unroll
        for (int ss = 0; ss < rr; ++ss) acc = fmaf(M[(o + rr) * kLd + o + ss], x[ss], acc);
        x[rr] = (rr < jj) ? 0.f : (rr == jj ? 1.f : -acc);
      }
#pragma unroll
      for (int rr = 0; rr < 16; ++rr) X[(o + rr) * kLd + o + jj] = x[rr];
    }
    __syncthreads();
    for (int d = 1; d <= 3; ++d) {
      const int npairs = 4 - d;
      for (int e = tid; e < npairs * 256; e += 128) {
        const int pi = e >> 8, a = (e >> 4) & 15, bcol = e & 15;
        const int i = d + pi, jb = pi;
        float acc = 0.f;
        for (int kb = jb; kb < i; ++kb)
#pragma unroll
          for (int s = 0; s < 16; ++s)
            acc = fmaf(M[(i * 16 + a) * kLd + kb * 16 + s], X[(kb * 16 + s) * kLd + jb * 16 + bcol],
                       acc);
        Y[pi * 16 * 17 + a * 17 + bcol] = acc;
      }
      __syncthreads();
      for (int e = tid; e < npairs * 256; e += 128) {
        const int pi = e >> 8, a = (e >> 4) & 15, bcol = e & 15;
        const int i = d + pi, jb = pi;
        float acc = 0.f;
#pragma unroll
        for (int s = 0; s < 16; ++s)
          acc = fmaf(X[(i * 16 + a) * kLd + i * 16 + s], Y[pi * 16 * 17 + s * 17 + bcol], acc);
        X[(i * 16 + a) * kLd + jb * 16 + bcol] = -acc;
      }
      __syncthreads();
    }
    // ---- T diag(beta) -> bf16, K-major [r][s] (the B operand (T diag beta)^T)
    {
      const int r = tid >> 1, half = tid & 1;
#pragma unroll
      for (int cch = 0; cch < 4; ++cch) {
        const int chunk = half * 4 + cch;
        uint32_t pk[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int s = chunk * 8 + 2 * u;
          const float a = (s <= r) ? X[r * kLd + s] * s_beta[s] : 0.f;
          const float b2 = (s + 1 <= r) ? X[r * kLd + s + 1] * s_beta[s + 1] : 0.f;
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
    tma_seen = mbar_wait(&tma_bar, 0, budget);
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
    mma_commits = 2;
    ok = mbar_wait(&mma_bar, 1, budget);
  }
  ok = !__syncthreads_or(!ok);
  if (ok) {
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32);
    const int row = tid;  // lane == k for W^T, == v for U^T
    uint32_t a[32];
    __nv_bfloat16* wt = reinterpret_cast<__nv_bfloat16*>(p.ws + p.lay.wt + rec * kTileWT) + row * 64;
    __half* ut = reinterpret_cast<__half*>(p.ws + p.lay.ut + rec * kTileUT) + row * 64;
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      tmem_ld32(tmem_addr(tbase, lane_base, part * 32), a);
      tmem_wait_ld();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint4 o;
        o.x = pack_bf16(__uint_as_float(a[q8 * 8 + 0]), __uint_as_float(a[q8 * 8 + 1]));
        o.y = pack_bf16(__uint_as_float(a[q8 * 8 + 2]), __uint_as_float(a[q8 * 8 + 3]));
        o.z = pack_bf16(__uint_as_float(a[q8 * 8 + 4]), __uint_as_float(a[q8 * 8 + 5]));
        o.w = pack_bf16(__uint_as_float(a[q8 * 8 + 6]), __uint_as_float(a[q8 * 8 + 7]));
        *reinterpret_cast<uint4*>(wt + part * 32 + q8 * 8) = o;
      }
    }
#pragma unroll
    for (int part = 0; part < 2; ++part) {
      tmem_ld32(tmem_addr(tbase, lane_base, 64 + part * 32), a);
      tmem_wait_ld();
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint4 o;
        o.x = pack_f16(__uint_as_float(a[q8 * 8 + 0]), __uint_as_float(a[q8 * 8 + 1]));
        o.y = pack_f16(__uint_as_float(a[q8 * 8 + 2]), __uint_as_float(a[q8 * 8 + 3]));
        o.z = pack_f16(__uint_as_float(a[q8 * 8 + 4]), __uint_as_float(a[q8 * 8 + 5]));
        o.w = pack_f16(__uint_as_float(a[q8 * 8 + 6]), __uint_as_float(a[q8 * 8 + 7]));
        *reinterpret_cast<uint4*>(ut + part * 32 + q8 * 8) = o;
      }
    }
  }

  // ---- teardown: on any failure record it, drain what was issued, free TMEM
  if (!ok) {
    if (tid == 0) {
      record_status(p.ws, kStatusTimeout);
      // commits complete in issue order: waiting for the last one drains all
      mbar_wait(&tma_bar, 0, drain_budget);
      if (mma_commits > 0)
        mbar_wait(&mma_bar, static_cast<uint32_t>((mma_commits - 1) & 1), drain_budget);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) tmem_dealloc(tbase, 256);
}

}  // namespace kda
