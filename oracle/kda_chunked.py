"""Chunked (UT/WY) form of the KDA recurrence in NumPy FP64 (test infrastructure).

Derived by hand from the per-token recurrence of kda_oracle.c and used only as
an independent check of it: the chunked and the per-token forms must agree.
Splitting a chunk-wise form into a prepare pass and a recurrence pass is what
FlashInfer PR #4633 ("Description") does in its two-launch design; the algebra
below is derived here.

For one (sequence, head), one chunk of c tokens (local r = 0..c-1), state S0
(K x V) entering the chunk, G_r = sum_{s<=r} g_s (per key channel),
Gamma_r = exp(G_r):

  A[r, s]   = sum_k k_r[k] k_s[k] exp(G_r[k] - G_s[k])           (s < r)
  T         = (I + diag(beta) A)^-1                              (unit lower triangular)
  W         = T diag(beta) (K * Gamma)          U = T diag(beta) V
  U_delta   = U - W S0
  Aqk[r, s] = sum_k q_r[k] k_s[k] exp(G_r[k] - G_s[k])           (s <= r)
  O         = scale [ (Q * Gamma) S0 + Aqk U_delta ]
  S1        = Diag(Gamma_{c-1}) S0 + (K * exp(G_{c-1} - G))^T U_delta

Induction on r gives S_r = Diag(Gamma_r) S0 + sum_{s<=r} Diag(Gamma_r / Gamma_s) k_s u_s^T;
inserting it in u_r = beta_r (v_r - S'_r^T k_r) yields (I + diag(beta) A) U_delta =
diag(beta) (V - (K * Gamma) S0), which is the triangular system above.  The
state after the first p tokens of the chunk is the same expression as S1 with
the sum cut at p.
"""
from __future__ import annotations

import numpy as np
from scipy.linalg import solve_triangular


def _chunk(q, k, v, g, beta, scale, S0, ckpt_local=None):
    """One chunk.  q,k,g: [c,K]; v: [c,V]; beta: [c]; S0: [K,V].  Returns (O, S1, S_ckpt)."""
    c = q.shape[0]
    G = np.cumsum(g, axis=0)                                  # [c, K]
    diff = G[:, None, :] - G[None, :, :]                      # [r, s, K] = G_r - G_s
    lower_incl = np.tril(np.ones((c, c), dtype=bool))
    # exp only where s <= r; elsewhere the entry is masked out of the definition
    dec = np.where(lower_incl[:, :, None], np.exp(np.where(lower_incl[:, :, None], diff, 0.0)),
                   0.0)
    A = np.einsum("rk,sk,rsk->rs", k, k, dec)
    A = np.tril(A, -1)
    Aqk = np.einsum("rk,sk,rsk->rs", q, k, dec)               # already zero for s > r
    M = np.eye(c) + beta[:, None] * A
    Tm = solve_triangular(M, np.eye(c), lower=True, unit_diagonal=True)
    Gam = np.exp(G)
    W = Tm @ (beta[:, None] * (k * Gam))
    U = Tm @ (beta[:, None] * v)
    Ud = U - W @ S0
    O = scale * ((q * Gam) @ S0 + Aqk @ Ud)
    Kd = k * np.exp(G[-1][None, :] - G)
    S1 = np.exp(G[-1])[:, None] * S0 + Kd.T @ Ud
    Sc = None
    if ckpt_local is not None:
        p = int(ckpt_local)
        if p == 0:
            Sc = S0.copy()
        else:
            Kp = k[:p] * np.exp(G[p - 1][None, :] - G[:p])
            Sc = np.exp(G[p - 1])[:, None] * S0 + Kp.T @ Ud[:p]
    return O, S1, Sc


def chunked_prefill_f64(q, k, v, g, beta, scale, cu_seqlens, h0=None, ckpt_offsets=None,
                        chunk: int = 64):
    """Chunked form over a packed batch; same shapes and return values as prefill_f64."""
    q, k, v, g, beta = (np.asarray(x, np.float64) for x in (q, k, v, g, beta))
    cu = np.asarray(cu_seqlens, np.int64)
    T, H, K = q.shape
    V = v.shape[2]
    N = cu.shape[0] - 1
    out = np.zeros((T, H, V))
    ht = np.zeros((N, H, K, V))
    ck = None if ckpt_offsets is None else np.asarray(ckpt_offsets, np.int64)
    ckpt = None if ck is None else np.zeros((N, H, K, V))
    for n in range(N):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        for h in range(H):
            S = np.zeros((K, V)) if h0 is None else np.asarray(h0, np.float64)[n, h].copy()
            if ck is not None and ck[n] == 0:
                ckpt[n, h] = S
            for c0 in range(t0, t1, chunk):
                c1 = min(c0 + chunk, t1)
                local = None
                if ck is not None and c0 - t0 < ck[n] <= c1 - t0:
                    local = int(ck[n]) - (c0 - t0)
                O, S1, Sc = _chunk(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], g[c0:c1, h],
                                   beta[c0:c1, h], scale, S, local)
                out[c0:c1, h] = O
                if Sc is not None:
                    ckpt[n, h] = Sc
                S = S1
            ht[n, h] = S
    return out, ht, ckpt
