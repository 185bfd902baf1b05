"""Pins for the oracle: facts fixed by the method statement and by mathematics.

Each pin takes an implementation ``f(q, k, v, g, beta, scale, cu, h0=None, ck=None)
-> (o, ht, ckpt)`` (NumPy float64) and returns ``(ok, detail)``.  The same
pins run against the oracle (all must pass) and against oracle builds with a
planted mistake (at least one must fail for every mistake), which shows the
pins can tell a right oracle from a plausibly wrong one.

Where a pin is not simply an evaluation of the definition it says what makes
it independent: exact rational arithmetic on a rearranged transition form,
automatic differentiation of the delta rule's loss, closed forms, invariants.
"""
from __future__ import annotations

import json
import math
import os
from fractions import Fraction

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def random_case(seed, lens, H=2, K=4, V=3, h0=False, gmin=-5.0):
    r = _rng(seed)
    T = int(sum(lens))
    q = _unit_rows(r.standard_normal((T, H, K)))
    k = _unit_rows(r.standard_normal((T, H, K)))
    v = r.standard_normal((T, H, V))
    g = gmin * r.uniform(0.0, 1.0, (T, H, K))
    beta = r.uniform(0.05, 1.0, (T, H))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    S0 = 0.3 * r.standard_normal((len(lens), H, K, V)) if h0 else None
    return q, k, v, g, beta, cu, S0


def _close(a, b, tol):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    den = max(1.0, float(np.abs(b).max()) if b.size else 1.0)
    err = float(np.abs(a - b).max()) / den if a.size else 0.0
    return err <= tol, err


# ---------------------------------------------------------------- exact / golden

def pin_golden_handworked(f):
    """Hand-worked K=V=2 example (tests/golden/kda_k2_handworked.json)."""
    d = json.load(open(os.path.join(GOLDEN, "kda_k2_handworked.json")))
    q = np.array(d["q"])[:, None, :]
    k = np.array(d["k"])[:, None, :]
    v = np.array(d["v"])[:, None, :]
    g = np.log(np.array(d["decay"]))[:, None, :]
    beta = np.array(d["beta"])[:, None]
    cu = np.array([0, 2], np.int64)
    o, ht, ck = f(q, k, v, g, beta, d["scale"], cu, None, np.array([1], np.int64))
    ok1, e1 = _close(o[:, 0], d["o"], 1e-13)
    ok2, e2 = _close(ht[0, 0], d["S_final"], 1e-13)
    ok3, e3 = _close(ck[0, 0], d["S_after_1"], 1e-13)
    return ok1 and ok2 and ok3, f"o {e1:.2e} S {e2:.2e} ckpt {e3:.2e}"


def _exact_transition_form(q, k, v, dec, beta, scale, S0):
    """Exact rational evaluation of S_t = (I - b k k^T) D_t S_{t-1} + b k v^T.

    This is the recurrence rearranged into its transition-matrix form, evaluated
    with Fractions (no rounding at all); it does not reuse the oracle's order of
    operations.
    """
    T, K, V = len(k), len(k[0]), len(v[0])
    S = [[Fraction(S0[a][b]) for b in range(V)] for a in range(K)]
    outs = []
    for t in range(T):
        DS = [[dec[t][a] * S[a][b] for b in range(V)] for a in range(K)]
        M = [[(Fraction(1) if a == c else Fraction(0)) - beta[t] * k[t][a] * k[t][c]
              for c in range(K)] for a in range(K)]
        S = [[sum(M[a][c] * DS[c][b] for c in range(K)) + beta[t] * k[t][a] * v[t][b]
              for b in range(V)] for a in range(K)]
        outs.append([scale * sum(S[a][b] * q[t][a] for a in range(K)) for b in range(V)])
    return outs, S


def pin_bruteforce_rational(f, seed=11, T=6, K=3, V=2):
    """Oracle vs exact rational arithmetic on tiny inputs (decays chosen rational)."""
    r = _rng(seed)

    def frac(x, den=16):
        return Fraction(int(round(x * den)), den)

    q = [[frac(r.uniform(-1, 1)) for _ in range(K)] for _ in range(T)]
    k = [[frac(r.uniform(-0.6, 0.6)) for _ in range(K)] for _ in range(T)]
    v = [[frac(r.uniform(-2, 2)) for _ in range(V)] for _ in range(T)]
    dec = [[Fraction(int(r.integers(1, 17)), 16) for _ in range(K)] for _ in range(T)]
    beta = [Fraction(int(r.integers(1, 9)), 8) for _ in range(T)]
    S0 = [[frac(r.uniform(-1, 1)) for _ in range(V)] for _ in range(K)]
    scale = Fraction(1, 4)
    outs, S = _exact_transition_form(q, k, v, dec, beta, scale, S0)
    A = lambda m: np.array([[float(x) for x in row] for row in m])
    o, ht, _ = f(A(q)[:, None], A(k)[:, None], A(v)[:, None], np.log(A(dec))[:, None],
                 A([[b] for b in beta]), float(scale), np.array([0, T], np.int64),
                 A(S0)[None, None], None)
    ok1, e1 = _close(o[:, 0], A(outs), 1e-12)
    ok2, e2 = _close(ht[0, 0], A(S), 1e-12)
    return ok1 and ok2, f"o {e1:.2e} S {e2:.2e}"


# ---------------------------------------------------------------- closed forms

def pin_beta_zero_pure_decay(f, seed=3):
    """beta = 0: S_t = Diag(exp(G_t)) S0 and o_t = scale (Diag(exp G_t) S0)^T q_t."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [7, 5], h0=True)
    beta = np.zeros_like(beta)
    o, ht, _ = f(q, k, v, g, beta, 0.5, cu, S0, None)
    ok = True
    err = 0.0
    for n in range(2):
        G = np.cumsum(g[cu[n]:cu[n + 1]], axis=0)              # [L, H, K]
        for h in range(q.shape[1]):
            St = np.exp(G[:, h, :])[:, :, None] * S0[n, h][None]  # [L, K, V]
            exp_o = 0.5 * np.einsum("tkv,tk->tv", St, q[cu[n]:cu[n + 1], h])
            a, e1 = _close(o[cu[n]:cu[n + 1], h], exp_o, 1e-12)
            b, e2 = _close(ht[n, h], St[-1], 1e-12)
            ok &= a and b
            err = max(err, e1, e2)
    return ok, f"{err:.2e}"


def pin_identity_when_nothing_happens(f, seed=4):
    """beta = 0 and g = 0: the state never changes and o_t = scale h0^T q_t."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [9], h0=True)
    o, ht, _ = f(q, k, v, np.zeros_like(g), np.zeros_like(beta), 0.25, cu, S0, None)
    a, e1 = _close(ht, S0, 0.0)
    b, e2 = _close(o, 0.25 * np.einsum("hkv,thk->thv", S0[0], q), 1e-13)
    return a and b, f"{e1:.2e} {e2:.2e}"


def pin_single_token_is_one_sgd_step(f, seed=5):
    """T = 1: the update is one gradient step, rate beta, on 1/2 ||S'^T k - v||^2.

    The gradient comes from torch.autograd in float64, so the sign and the
    operand order of the correction are fixed by differentiation, not retyped.
    """
    import torch
    q, k, v, g, beta, cu, S0 = random_case(seed, [1], H=1, K=5, V=4, h0=True)
    o, ht, _ = f(q, k, v, g, beta, 0.7, cu, S0, None)
    Sd = torch.tensor(np.exp(g[0, 0])[:, None] * S0[0, 0], dtype=torch.float64,
                      requires_grad=True)
    kt = torch.tensor(k[0, 0])
    vt = torch.tensor(v[0, 0])
    loss = 0.5 * ((Sd.T @ kt - vt) ** 2).sum()
    (grad,) = torch.autograd.grad(loss, Sd)
    S1 = (Sd - float(beta[0, 0]) * grad).detach().numpy()
    a, e1 = _close(ht[0, 0], S1, 1e-13)
    b, e2 = _close(o[0, 0], 0.7 * S1.T @ q[0, 0], 1e-13)
    return a and b, f"{e1:.2e} {e2:.2e}"


def pin_basis_keys_overwrite_rows(f, seed=6):
    """g = 0, beta = 1, k_t = e_{i_t}: row i_t of S becomes v_t exactly, others stay."""
    r = _rng(seed)
    K, V, T = 6, 4, 5
    idx = r.permutation(K)[:T]
    k = np.zeros((T, 1, K))
    k[np.arange(T), 0, idx] = 1.0
    v = r.standard_normal((T, 1, V))
    q = _unit_rows(r.standard_normal((T, 1, K)))
    S0 = r.standard_normal((1, 1, K, V))
    o, ht, _ = f(q, k, v, np.zeros((T, 1, K)), np.ones((T, 1)), 1.0,
                 np.array([0, T], np.int64), S0, None)
    exp = S0[0, 0].copy()
    exp[idx] = v[:, 0]
    return _close(ht[0, 0], exp, 1e-15)[0], "rows overwritten"


# ---------------------------------------------------------------- invariants

def pin_delta_rule_retrieval(f, seed=7):
    """beta = 1 and unit-norm k: right after token t, S_t^T k_t = v_t."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [11], H=2, K=5, V=3, h0=True)
    beta = np.ones_like(beta)
    err = 0.0
    ok = True
    for p in (1, 4, 11):
        _, _, ck = f(q, k, v, g, beta, 1.0, cu, S0, np.array([p], np.int64))
        for h in range(2):
            a, e = _close(ck[0, h].T @ k[p - 1, h], v[p - 1, h], 1e-12)
            ok &= a
            err = max(err, e)
    return ok, f"{err:.2e}"


def pin_linearity(f, seed=8):
    """For fixed q, k, g, beta the map (V, h0) -> (o, ht) is linear."""
    q, k, v1, g, beta, cu, S1 = random_case(seed, [6, 9], h0=True)
    _, _, v2, _, _, _, S2 = random_case(seed + 100, [6, 9], h0=True)
    a, b = 0.7, -1.3
    o1, h1, _ = f(q, k, v1, g, beta, 0.3, cu, S1, None)
    o2, h2, _ = f(q, k, v2, g, beta, 0.3, cu, S2, None)
    o3, h3, _ = f(q, k, a * v1 + b * v2, g, beta, 0.3, cu, a * S1 + b * S2, None)
    x, e1 = _close(o3, a * o1 + b * o2, 1e-12)
    y, e2 = _close(h3, a * h1 + b * h2, 1e-12)
    return x and y, f"{e1:.2e} {e2:.2e}"


def pin_scale_linearity(f, seed=9):
    """o is proportional to scale; the states do not depend on it."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [8], h0=True)
    o1, h1, _ = f(q, k, v, g, beta, 1.0, cu, S0, None)
    o2, h2, _ = f(q, k, v, g, beta, 0.125, cu, S0, None)
    x, e1 = _close(o2, 0.125 * o1, 1e-14)
    y, e2 = _close(h2, h1, 0.0)
    return x and y, f"{e1:.2e} {e2:.2e}"


def pin_chunked_equals_per_token(f, seed=10, chunks=(1, 3, 16, 64, 128)):
    """The hand-derived chunked (UT/WY) form equals the per-token form."""
    import oracle
    lens = [200, 67, 1, 0, 130]
    q, k, v, g, beta, cu, S0 = random_case(seed, lens, H=2, K=8, V=6, h0=True)
    ck = np.array([57, 67, 1, 0, 129], np.int64)
    o, ht, c = f(q, k, v, g, beta, 0.2, cu, S0, ck)
    ok = True
    err = 0.0
    for C in chunks:
        o2, h2, c2 = oracle.chunked_prefill_f64(q, k, v, g, beta, 0.2, cu, S0, ck, chunk=C)
        for a, b in ((o, o2), (ht, h2), (c, c2)):
            x, e = _close(a, b, 1e-10)
            ok &= x
            err = max(err, e)
    return ok, f"{err:.2e}"


def pin_ragged_equals_separate(f, seed=12):
    """A packed ragged batch gives each sequence's own result."""
    lens = [13, 0, 1, 29, 4]
    q, k, v, g, beta, cu, S0 = random_case(seed, lens, h0=True)
    ck = np.array([5, 0, 1, 29, 2], np.int64)
    o, ht, c = f(q, k, v, g, beta, 0.4, cu, S0, ck)
    ok = True
    err = 0.0
    for n, L in enumerate(lens):
        sl = slice(cu[n], cu[n + 1])
        o1, h1, c1 = f(q[sl], k[sl], v[sl], g[sl], beta[sl], 0.4, np.array([0, L], np.int64),
                       S0[n:n + 1], ck[n:n + 1])
        for a, b in ((o[sl], o1), (ht[n], h1[0]), (c[n], c1[0])):
            x, e = _close(a, b, 0.0)
            ok &= x
            err = max(err, e)
    return ok, f"{err:.2e}"


def pin_checkpoint_is_prefix_state(f, seed=13):
    """The checkpoint at offset p equals the final state of the first p tokens."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [23], h0=True)
    ok = True
    err = 0.0
    for p in (0, 1, 9, 22, 23):
        _, _, c = f(q, k, v, g, beta, 0.4, cu, S0, np.array([p], np.int64))
        _, hp, _ = f(q[:p], k[:p], v[:p], g[:p], beta[:p], 0.4, np.array([0, p], np.int64),
                     S0, None)
        x, e = _close(c, hp, 0.0)
        ok &= x
        err = max(err, e)
    return ok, f"{err:.2e}"


def pin_prefix_resume(f, seed=14):
    """prefill(prefix) -> h0 -> prefill(suffix) equals one prefill of the whole."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [31], h0=True)
    p = 12
    o, ht, c = f(q, k, v, g, beta, 0.4, cu, S0, np.array([p], np.int64))
    sl = slice(p, 31)
    o2, h2, _ = f(q[sl], k[sl], v[sl], g[sl], beta[sl], 0.4, np.array([0, 31 - p], np.int64),
                  c, None)
    x, e1 = _close(o2, o[sl], 1e-13)
    y, e2 = _close(h2, ht, 1e-13)
    return x and y, f"{e1:.2e} {e2:.2e}"


def pin_zero_length_keeps_h0(f, seed=15):
    """A zero-length sequence returns h0 as its final state and as its checkpoint."""
    q, k, v, g, beta, cu, S0 = random_case(seed, [0, 3, 0], h0=True)
    _, ht, c = f(q, k, v, g, beta, 0.4, cu, S0, np.array([0, 3, 0], np.int64))
    x, _ = _close(ht[0], S0[0], 0.0)
    y, _ = _close(ht[2], S0[2], 0.0)
    z, _ = _close(c[0], S0[0], 0.0)
    return x and y and z, "h0 kept"


ALL_PINS = [
    pin_golden_handworked, pin_bruteforce_rational, pin_beta_zero_pure_decay,
    pin_identity_when_nothing_happens, pin_single_token_is_one_sgd_step,
    pin_basis_keys_overwrite_rows, pin_delta_rule_retrieval, pin_linearity,
    pin_scale_linearity, pin_chunked_equals_per_token, pin_ragged_equals_separate,
    pin_checkpoint_is_prefix_state, pin_prefix_resume, pin_zero_length_keeps_h0,
]
