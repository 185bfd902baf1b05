/*
 * KDA per-token recurrence in FP64 — the ORACLE.
 *
 * Test infrastructure only: tests, the smoke check and the CPU-baseline leg of
 * the benchmark may call it; the library product never does.  It shares no
 * code, header or constant with the CUDA path.
 *
 * What it computes (Kimi Delta Attention, a gated delta rule with one decay
 * per key channel).  The pages quoted for this method (lmdeploy PR #5050
 * "Motivation"; FlashInfer PR #4262 "Dispatch contract"; FlashInfer PR #4633
 * "Description") fix the interface — K = V = 128, BF16 inputs, an FP32
 * K x V state per (sequence, head), ragged packing through cu_seqlens, an
 * optional initial state, the final state and a state exported at a caller
 * offset — but print no formula.  The definition written out here is the
 * plain reading of the method statement: for each (sequence n, head h),
 * S = h0[n,h] (or 0), and for every token t of the sequence
 *
 *     S  <- Diag(exp(g_t)) S                   decay each key row k by exp(g_t[k])
 *     u  <- beta_t (v_t - S^T k_t)             prediction error, S already decayed
 *     S  <- S + k_t u^T                        rank-one delta update
 *     o_t = scale * S^T q_t                    read-out after the update
 *
 * The state after the first p tokens of a sequence (0 <= p <= len) is the
 * checkpoint for offset p: p = 0 gives h0, p = len gives the final state.
 *
 * Layouts (row-major, element counts):
 *   q, k, g : [T_total][H][K]     v, out : [T_total][H][V]     beta : [T_total][H]
 *   h0, ht, ckpt : [N][H][K][V]  (S[k][v], key index first)
 *   cu_seqlens : [N+1] int64, 0 = cu[0] <= cu[1] <= ... <= cu[N] = T_total
 *   ckpt_offsets : [N] int64, 0 <= p_n <= len_n
 *
 * `mutation` plants one known mistake (tests use it to show that the pins of
 * this oracle catch such mistakes); 0 means the definition above.
 *   1: u uses the state before the decay      2: read-out before the update
 *   3: decay applied to value columns          4: sign of the correction flipped
 *   5: beta ignored in the update              6: decay uses g of the next token
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static void kda_one_head(int64_t n, int64_t h, int64_t T0, int64_t L, int64_t H,
                         int64_t K, int64_t V, const double* q, const double* k,
                         const double* v, const double* g, const double* beta,
                         double scale, const double* h0, int64_t ckpt_p,
                         double* out, double* ht, double* ckpt, int mutation,
                         double* S, double* Sold, double* u) {
  const int64_t KV = K * V;
  if (h0)
    memcpy(S, h0 + (n * H + h) * KV, sizeof(double) * KV);
  else
    memset(S, 0, sizeof(double) * KV);
  if (ckpt && ckpt_p == 0) memcpy(ckpt + (n * H + h) * KV, S, sizeof(double) * KV);

  for (int64_t t = 0; t < L; ++t) {
    const int64_t row = (T0 + t) * H + h;
    const double* qt = q + row * K;
    const double* kt = k + row * K;
    const double* vt = v + row * V;
    const double* gt = g + row * K;
    if (mutation == 6 && t + 1 < L) gt = g + ((T0 + t + 1) * H + h) * K;
    const double bt = (mutation == 5) ? 1.0 : beta[row];

    if (mutation == 1) memcpy(Sold, S, sizeof(double) * KV);
    /* S <- Diag(exp g_t) S */
    if (mutation == 3) {
      for (int64_t a = 0; a < K; ++a)
        for (int64_t b = 0; b < V; ++b) S[a * V + b] *= exp(gt[b % K]);
    } else {
      for (int64_t a = 0; a < K; ++a) {
        const double d = exp(gt[a]);
        for (int64_t b = 0; b < V; ++b) S[a * V + b] *= d;
      }
    }
    /* read-out before the update (planted mistake) */
    if (mutation == 2) {
      for (int64_t b = 0; b < V; ++b) {
        double acc = 0.0;
        for (int64_t a = 0; a < K; ++a) acc += S[a * V + b] * qt[a];
        out[row * V + b] = scale * acc;
      }
    }
    /* u = beta (v - S^T k) */
    const double* Sp = (mutation == 1) ? Sold : S;
    for (int64_t b = 0; b < V; ++b) {
      double pred = 0.0;
      for (int64_t a = 0; a < K; ++a) pred += Sp[a * V + b] * kt[a];
      u[b] = (mutation == 4) ? bt * (vt[b] + pred) : bt * (vt[b] - pred);
    }
    /* S <- S + k u^T */
    for (int64_t a = 0; a < K; ++a)
      for (int64_t b = 0; b < V; ++b) S[a * V + b] += kt[a] * u[b];
    /* o_t = scale S^T q_t */
    if (mutation != 2) {
      for (int64_t b = 0; b < V; ++b) {
        double acc = 0.0;
        for (int64_t a = 0; a < K; ++a) acc += S[a * V + b] * qt[a];
        out[row * V + b] = scale * acc;
      }
    }
    if (ckpt && ckpt_p == t + 1) memcpy(ckpt + (n * H + h) * KV, S, sizeof(double) * KV);
  }
  if (ht) memcpy(ht + (n * H + h) * KV, S, sizeof(double) * KV);
}

/* Returns 0 on success, -1 on an invalid argument (nothing is written then). */
int kda_oracle_prefill(int64_t N, const int64_t* cu_seqlens, int64_t H, int64_t K,
                       int64_t V, const double* q, const double* k, const double* v,
                       const double* g, const double* beta, double scale,
                       const double* h0, const int64_t* ckpt_offsets, double* out,
                       double* ht, double* ckpt, int num_threads, int mutation) {
  if (N < 0 || H <= 0 || K <= 0 || V <= 0 || !cu_seqlens) return -1;
  if (cu_seqlens[0] != 0) return -1;
  for (int64_t n = 0; n < N; ++n) {
    if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    if (ckpt_offsets && (ckpt_offsets[n] < 0 || ckpt_offsets[n] > cu_seqlens[n + 1] - cu_seqlens[n]))
      return -1;
  }
  if ((ckpt == NULL) != (ckpt_offsets == NULL)) return -1;
  const int64_t units = N * H;
  int rc = 0;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel
#endif
  {
    double* S = (double*)malloc(sizeof(double) * K * V);
    double* Sold = (double*)malloc(sizeof(double) * K * V);
    double* u = (double*)malloc(sizeof(double) * V);
    if (!S || !Sold || !u) rc = -2;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
    for (int64_t w = 0; w < units; ++w) {
      if (!S || !Sold || !u) continue;
      const int64_t n = w / H, h = w % H;
      const int64_t T0 = cu_seqlens[n], L = cu_seqlens[n + 1] - cu_seqlens[n];
      kda_one_head(n, h, T0, L, H, K, V, q, k, v, g, beta, scale, h0,
                   ckpt_offsets ? ckpt_offsets[n] : -1, out, ht, ckpt, mutation, S, Sold,
                   u);
    }
    free(S);
    free(Sold);
    free(u);
  }
  return rc;
}

int kda_oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
