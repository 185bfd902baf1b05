"""Rounding model of the chunked KDA form (test infrastructure, CPU).

It replays the chunked factorisation of one (sequence, head) in FP64 and rounds each
operand where the tensor-core path stores it, so that the effect of an operand
precision on the final state can be measured against the FP64 per-token oracle
before (or without) running a kernel.  Nothing here is shared with the CUDA path; it
models its choices:

  A, Aqk   from [K+; Q+] R^T, operands rounded to BF16 per 16-token sub-block
  T        (I + diag(beta) A)^-1, then T diag(beta) rounded to `tb` (FP16 or BF16)
  W, U     T diag(beta) (K Gamma), T diag(beta) V; K Gamma and v in the type of `tb`
           (both operands of one tensor-core product share a type)
  S0       the state read by the tensor core, rounded to `s0` (FP16 or BF16), and
           with it W and Q Gamma, its partners in the same products
  Ud       U - W S0, rounded to FP16 (the state update operand)
  Kd       K exp(G_end - G), rounded to FP16
  Aqk      rounded to FP16 for the output product

The kernels' plan is the default (tb = s0 = FP16).  tb = s0 = BF16 is the earlier plan,
which misses the 1e-3 state gate when nothing decays (g = 0): with Gamma = 1 every
chunk's rounding error stays in the state.

``beta_split`` applies the split-beta scheme: T diag(bf16(beta)) is the rounded
operand and diag(beta - bf16(beta)) is added unrounded-enough (a second BF16 tile of a
value 2^-9 smaller), dropping (T - I) diag(beta - bf16(beta)).
"""
from __future__ import annotations

import numpy as np
import torch
from scipy.linalg import solve_triangular

SB = 16     # sub-block of the decay factorisation
C = 64      # chunk length


def to_bf16(x):
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.float32)
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def to_f16(x):
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)


def to_f32(x):
    return np.asarray(x, np.float32).astype(np.float64)


ROUND = {"bf16": to_bf16, "f16": to_f16, "f32": to_f32, "exact": lambda x: x}


def chunk_step(q, k, v, g, beta, scale, S0, *, tb="f16", s0="f16", ud="f16", kd="f16",
               aqk="f16", beta_split=False):
    """One chunk: returns (O [c, V], S1 [K, V])."""
    c = q.shape[0]
    G = to_f32(np.cumsum(to_f32(g), axis=0))
    A = np.zeros((c, c))
    Aq = np.zeros((c, c))
    for i in range(0, c, SB):
        B = G[i]
        rows = slice(i, min(i + SB, c))
        end = min(i + SB, c)
        lk = to_bf16(k[rows] * to_f32(np.exp(G[rows] - B)))
        lq = to_bf16(q[rows] * to_f32(np.exp(G[rows] - B)))
        r = to_bf16(k[:end] * to_f32(np.exp(B - G[:end])))
        A[rows, :end] = lk @ r.T
        Aq[rows, :end] = lq @ r.T
    A = to_f32(np.tril(A, -1))
    Aq = to_f32(np.tril(Aq))
    T = solve_triangular(np.eye(c) + beta[:, None] * A, np.eye(c), lower=True,
                         unit_diagonal=True)
    gam = to_f32(np.exp(G))
    kg = ROUND[tb](k * gam)
    v = ROUND[tb](v)
    if beta_split:
        hi = to_bf16(beta)
        lo = beta - hi
        tbm = ROUND[tb](to_f32(T * hi[None, :]))
        w = to_f32(tbm @ kg + to_bf16(lo)[:, None] * kg)
        u = to_f32(tbm @ v + to_bf16(lo)[:, None] * v)
    else:
        tbm = ROUND[tb](to_f32(T * beta[None, :]))
        w = to_f32(tbm @ kg)
        u = to_f32(tbm @ v)
    s0r = ROUND[s0](S0)
    d = ROUND[ud](to_f32(to_f16(u) - ROUND[s0](w) @ s0r))
    o = scale * (to_f32(ROUND[s0](q * gam) @ s0r) + to_f32(ROUND[aqk](Aq) @ d))
    kdm = ROUND[kd](k * to_f32(np.exp(G[-1][None, :] - G)))
    s1 = to_f32(to_f32(np.exp(G[-1]))[:, None] * S0) + to_f32(kdm.T @ d)
    return o, s1


def final_states(q, k, v, g, beta, scale, cu, h0=None, **opts):
    """Chunked model over a packed batch: q, k, v, g [T, H, 128], beta [T, H] (float64),
    cu [N+1]; returns the final states [N, H, 128, 128]."""
    N = len(cu) - 1
    H = q.shape[1]
    out = np.zeros((N, H, 128, 128))
    for n in range(N):
        for h in range(H):
            S = np.zeros((128, 128)) if h0 is None else np.asarray(h0[n, h], np.float64)
            for c0 in range(cu[n], cu[n + 1], C):
                c1 = min(c0 + C, cu[n + 1])
                _, S = chunk_step(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], g[c0:c1, h],
                                  beta[c0:c1, h], scale, S, **opts)
            out[n, h] = S
    return out
