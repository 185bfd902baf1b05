// kda_schedule.cu — per-call metadata for packed batches (one CTA).
//
// From cu_seqlens (and the checkpoint offsets, which add one chunk boundary each)
// it builds the chunk table chunk_base[n] = sum_{m<n} chunks_m (so every
// (chunk, head) gets a workspace slot), the span of every slot (first token, token
// count, chunk index), so that a prepare CTA finds its chunk with one load, and a
// longest-first order of the sequences for the recurrence grid, the tail-
// utilisation ordering FlashInfer PR #4262 "Dispatch contract" exposes as
// seq_order.  In validate mode it checks the metadata the host never reads
// (cu_seqlens starts at 0, is non-decreasing and ends at T: FlashInfer PR
// #4633 review of validate_packed_offsets; checkpoint offsets inside their
// sequence: lmdeploy PR #5050 "Motivation") and records the first violation
// in the workspace status word.
#include "kda_common.cuh"

namespace kda {

constexpr int kSchedThreads = 1024;
constexpr int kLptMax = 1024;  // longest-first ordering up to this many sequences

__global__ void __launch_bounds__(kSchedThreads) kda_schedule_kernel(const KdaParams p) {
  __shared__ int32_t warp_tot[32];
  __shared__ int32_t carry;
  __shared__ int32_t bad_cu, bad_ck;
  __shared__ int32_t s_len[kLptMax];
  int32_t* cb = reinterpret_cast<int32_t*>(p.ws + p.lay.chunk_base);
  int32_t* order = reinterpret_cast<int32_t*>(p.ws + p.lay.seq_order);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(p.ws);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const bool validate = (p.flags & kFlagValidate) != 0;
  if (tid == 0) {
    carry = 0;
    bad_cu = 0;
    bad_ck = 0;
  }
  // INT64 cu_seqlens: check (validate mode) and narrow into the workspace copy that
  // every kernel of this call reads (values clamped to [0, T]; T < 2^31)
  if (p.cu_seqlens64 != nullptr) {
    int32_t* cu32 = const_cast<int32_t*>(p.cu_seqlens);
    for (int n = tid; n <= p.N; n += kSchedThreads) {
      const int64_t a = p.cu_seqlens64[n];
      if (validate) {
        const int64_t prev = n > 0 ? p.cu_seqlens64[n - 1] : 0;
        if (a < 0 || a > p.T || a < prev || (n == 0 && a != 0) || (n == p.N && a != p.T) ||
            (n > 0 && p.max_len > 0 && a - prev > p.max_len))
          atomicExch(&bad_cu, 1);
      }
      cu32[n] = static_cast<int32_t>(a < 0 ? 0 : (a > p.T ? p.T : a));
    }
    __threadfence_block();
  }
  __syncthreads();
  for (int base = 0; base < p.N; base += kSchedThreads) {
    const int n = base + tid;
    int32_t cnt = 0, len = 0;
    if (n < p.N) {
      if (validate) {
        int32_t a = n * p.fixed_len, b = a + p.fixed_len;
        if (p.cu_seqlens != nullptr) {
          a = p.cu_seqlens[n];
          b = p.cu_seqlens[n + 1];
          if (b < a || (n == 0 && a != 0) || (n == p.N - 1 && b != p.T) ||
              (p.max_len > 0 && b - a > p.max_len))
            atomicExch(&bad_cu, 1);
        }
        if (p.ckpt_offsets != nullptr) {
          const int32_t o = p.ckpt_offsets[n];
          if (o < 0 || o > b - a) atomicExch(&bad_ck, 1);
        }
      }
      const SeqInfo si = seq_info(p, n, false);  // clamped geometry, checkpoint split included
      len = si.len;
      cnt = si.nch;
      if (p.N <= kLptMax) s_len[n] = len;
    }
    // block-wide exclusive scan of cnt
    int32_t x = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
      int32_t w = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int32_t y = __shfl_up_sync(0xffffffffu, w, o);
        if (lane >= o) w += y;
      }
      warp_tot[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    const int32_t incl = x + (warp > 0 ? warp_tot[warp - 1] : 0);
    if (n < p.N) cb[n] = carry + incl - cnt;
    __syncthreads();
    if (tid == kSchedThreads - 1) carry += incl;
    __syncthreads();
  }
  if (tid == 0) cb[p.N] = carry;
  __syncthreads();
  // slot spans: the sequence holding slot s is the largest n with cb[n] <= s (empty
  // sequences share their successor's base); slots past the last chunk get count 0
  {
    int2* span = reinterpret_cast<int2*>(p.ws + p.lay.slot_span);
    const int32_t total = cb[p.N];
    for (int64_t s = tid; s < p.slots; s += kSchedThreads) {
      int2 v = make_int2(0, 0);
      if (s < total) {
        int32_t lo = 0, hi = p.N;
        while (hi - lo > 1) {
          const int32_t mid = (lo + hi) >> 1;
          if (cb[mid] <= s) lo = mid; else hi = mid;
        }
        const SeqInfo si = seq_info(p, lo, false);
        const int32_t j = static_cast<int32_t>(s) - cb[lo];
        int32_t t0 = 0, c = 0;
        if (j < si.nch) chunk_span(si, j, t0, c);
        v = make_int2(si.start + t0, c | (j << 7));
      }
      span[s] = v;
    }
  }
  // longest-first order (stable on ties); identity beyond kLptMax sequences
  if (p.N <= kLptMax) {
    __syncthreads();
    for (int n = tid; n < p.N; n += kSchedThreads) {
      const int32_t ln = s_len[n];
      int32_t rank = 0;
      for (int m = 0; m < p.N; ++m) {
        const int32_t lm = s_len[m];
        rank += (lm > ln) || (lm == ln && m < n);
      }
      order[rank] = n;
    }
  } else {
    for (int n = tid; n < p.N; n += kSchedThreads) order[n] = n;
  }
  __syncthreads();
  if (tid == 0) {
    const int ok = !(bad_cu || bad_ck);
    hdr->call_ok = ok;
    if (bad_cu) record_status(p.ws, kStatusBadCuSeqlens);
    else if (bad_ck) record_status(p.ws, kStatusBadCkptOffset);
  }
}

}  // namespace kda
