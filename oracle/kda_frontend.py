"""FP64 oracle of the KDA input front end (test infrastructure only).

Serving code calls the KDA kernels on raw projections and lets the kernel form
the recurrence inputs.  The pages fix the interface of that front end but print
no formula for it:

* FlashInfer PR #4262, "Dispatch contract": the fast path takes ``A_log``
  (FP32, one value per head) and ``dt_bias`` (FP32, one value per head and key
  channel), the switches ``use_qk_l2norm_in_kernel``, ``use_gate_in_kernel`` and
  ``beta_is_logit``, and a finite, negative ``lower_bound``;
* lmdeploy PR #5050, "Motivation": the gate lower bound lies in [-5, 0];
* FlashInfer PR #4633, review of the SM120 validator: ``lower_bound`` ranges of
  [-5, 0) and [-5, 0] in two places of one codebase.

Reading adopted here (stated as this library's definition, per (token, head)):

    q_hat = q / sqrt(sum_c q_c^2 + eps)                   (use_qk_l2norm_in_kernel)
    k_hat = k / sqrt(sum_c k_c^2 + eps)
    g_c   = lower_bound * sigmoid(exp(A_log) * (a_c + dt_bias_c))   (use_gate_in_kernel)
    beta  = sigmoid(b)                                    (beta_is_logit)
    sigmoid(x) = 1 / (1 + exp(-x))

``a`` is the raw gate projection and ``b`` the raw beta logit.  The gate form is
the plainest one that uses every named parameter and puts every log-decay
inside (lower_bound, 0), the interval the lower bound names; the L2 norm is the
textbook one with a small ``eps`` against zero rows.
"""
from __future__ import annotations

import numpy as np

QK_L2NORM = 1
GATE_IN_KERNEL = 2
BETA_IS_LOGIT = 4


def _sigmoid(x):
    return 1.0 / (1.0 + np.exp(-x))


def frontend_f64(q, k, a, b, A_log, dt_bias, lower_bound: float, eps: float, flags: int,
                 mutation: int = 0):
    """Front end in FP64.

    q, k, a: [T, H, 128]; b: [T, H]; A_log: [H]; dt_bias: [H, 128].  Each output
    passes its input through unchanged when its switch is off (a then is g).
    Returns (q_hat, k_hat, g, beta) as float64 arrays.  ``mutation`` plants a
    known mistake (for the pin tests only).
    """
    q, k, a, b = (np.asarray(x, np.float64) for x in (q, k, a, b))
    A_log = np.asarray(A_log, np.float64)
    dt_bias = np.asarray(dt_bias, np.float64)
    if flags & QK_L2NORM:
        def norm(x):
            s = (x * x).sum(-1, keepdims=True) + eps
            return x / (s if mutation == 4 else np.sqrt(s))
        q, k = norm(q), norm(k)
    g = a
    if flags & GATE_IN_KERNEL:
        rate = A_log if mutation == 2 else np.exp(A_log)
        shift = -dt_bias if mutation == 1 else dt_bias
        x = rate[None, :, None] * (a + shift[None])
        g = lower_bound * _sigmoid(-x if mutation == 3 else x)
    beta = b
    if flags & BETA_IS_LOGIT and mutation != 5:
        beta = _sigmoid(b)
    return q, k, g, beta
