"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the FP64 oracle on the same seeded inputs.

Tolerances (fixed by the method statement this library implements):
  * output o (BF16):            max |o_gpu - o_ref| <= 2e-2
  * final / checkpoint states:  ||S_gpu - S_ref||_F / ||S_ref||_F <= 1e-3 per (sequence, head)
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

O_TOL = 2e-2
S_TOL = 1e-3


def to_dev(inp):
    d = {}
    for name in ("q", "k", "v", "g", "beta", "cu_seqlens", "h0", "ckpt_offsets"):
        t = getattr(inp, name)
        d[name] = None if t is None else t.cuda()
    return d


def run_gpu(inp, *, inplace=False, flags=0, variant=0, fixed=None, workspace=None,
            h0_override=None, frontend=None):
    """Run kda_prefill on inp; returns dict of CPU tensors and the device status word."""
    import kda_chunked_recurrent_b200 as K
    d = to_dev(inp)
    fixed = inp.fixed_layout if fixed is None else fixed
    h0 = d["h0"] if h0_override is None else h0_override
    N = inp.num_seqs
    ht = None
    if inplace:
        assert h0 is not None
        h0 = h0.clone()
        ht = h0
    out, ht, ck = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=h0,
                            cu_seqlens=None if fixed else d["cu_seqlens"], num_seqs=N,
                            max_seqlen=max(inp.seqlens) if inp.seqlens else 0,
                            ckpt_offsets=d["ckpt_offsets"], ht=ht, workspace=workspace,
                            variant=variant, flags=flags,
                            frontend=None if frontend is None else dict(
                                frontend, A_log=frontend["A_log"].cuda(),
                                dt_bias=frontend["dt_bias"].cuda()))
    torch.cuda.synchronize()
    ws = workspace
    return {"o": out.float().cpu(), "ht": None if ht is None else ht.cpu(),
            "ckpt": None if ck is None else ck.cpu()}


def rel_fro(a, b):
    a = np.asarray(a, np.float64).reshape(a.shape[0], a.shape[1], -1)
    b = np.asarray(b, np.float64).reshape(b.shape[0], b.shape[1], -1)
    num = np.linalg.norm(a - b, axis=-1)
    den = np.maximum(np.linalg.norm(b, axis=-1), 1e-30)
    return num / den


def frontend_reference_inputs(inp, fe):
    """The recurrence inputs the FP64 front-end oracle forms from raw projections
    (fe: dict(flags, lower_bound, l2_eps, A_log, dt_bias) with CPU tensors), as a
    KDAInputs of float64 tensors for oracle.prefill."""
    import copy
    q, k, g, beta = oracle.frontend_f64(inp.q.double().numpy(), inp.k.double().numpy(),
                                        inp.g.double().numpy(), inp.beta.double().numpy(),
                                        fe["A_log"].double().numpy(), fe["dt_bias"].double().numpy(),
                                        fe["lower_bound"], fe["l2_eps"], fe["flags"])
    ref = copy.copy(inp)
    ref.q, ref.k, ref.g, ref.beta = (torch.from_numpy(np.ascontiguousarray(x))
                                     for x in (q, k, g, beta))
    return ref


def compare(inp, res, seqs=None, heads=None, threads=0, frontend=None):
    """Oracle on the selected (sequence, head) pairs vs the GPU result; returns metrics.
    With ``frontend`` the inputs are raw projections and the FP64 front end runs first."""
    if frontend is not None:
        inp = frontend_reference_inputs(inp, frontend)
    ref = oracle.prefill(inp, threads=threads, heads=heads, seqs=seqs)
    seqs, heads, rows = ref["seqs"], ref["heads"], ref["rows"]
    m = {}
    if rows.size:
        o_gpu = res["o"].double().numpy()[rows][:, heads]
        m["o_maxabs"] = float(np.abs(o_gpu - ref["o"]).max())
    else:
        m["o_maxabs"] = 0.0
    if res["ht"] is not None:
        ht_gpu = res["ht"].double().numpy()[seqs][:, heads]
        m["ht_rel"] = float(rel_fro(ht_gpu, ref["ht"]).max()) if ht_gpu.size else 0.0
        m["ht_zero_ok"] = bool(np.all(np.isfinite(ht_gpu)))
    if res.get("ckpt") is not None and ref["ckpt"] is not None:
        ck_gpu = res["ckpt"].double().numpy()[seqs][:, heads]
        m["ckpt_rel"] = float(rel_fro(ck_gpu, ref["ckpt"]).max())
    return m


def assert_parity(m):
    assert m["o_maxabs"] <= O_TOL, m
    if "ht_rel" in m:
        assert m["ht_rel"] <= S_TOL, m
    if "ckpt_rel" in m:
        assert m["ckpt_rel"] <= S_TOL, m


def decode_oracle(dinp, steps: bool = False, frontend=None):
    """FP64 oracle for kda_decode: every live sequence (slot in [0, P)) is a prefill
    of T tokens from its pool slot.  Returns dict with "live" (sequence indices),
    "o" [L, T, H, V], "ht" [L, H, K, V] and, with ``steps``, "steps" [L, T, H, K, V]
    (the oracle's checkpoint at every prefix length 1..T)."""
    N, T, H = (int(x) for x in dinp.q.shape[:3])
    P = int(dinp.pool.shape[0])
    idx = list(range(N)) if dinp.state_indices is None else dinp.state_indices.tolist()
    live = [n for n in range(N) if 0 <= idx[n] < P]
    L = len(live)
    res = {"live": live}
    if L == 0:
        return res
    sel = lambda x: np.ascontiguousarray(x.double().numpy()[live].reshape(L * T, H, -1))
    q, k, v, g = sel(dinp.q), sel(dinp.k), sel(dinp.v), sel(dinp.g)
    beta = np.ascontiguousarray(dinp.beta.double().numpy()[live].reshape(L * T, H))
    if frontend is not None:
        # frontend: dict(flags, lower_bound, l2_eps, A_log, dt_bias) with oracle switch values
        q, k, g, beta = oracle.frontend_f64(q, k, g, beta, frontend["A_log"].double().numpy(),
                                            frontend["dt_bias"].double().numpy(),
                                            frontend["lower_bound"], frontend["l2_eps"],
                                            frontend["flags"])
        q, k, g, beta = (np.ascontiguousarray(x) for x in (q, k, g, beta))
    h0 = np.ascontiguousarray(dinp.pool.double().numpy()[[idx[n] for n in live]])
    cu = np.arange(L + 1, dtype=np.int64) * T
    o, ht, _ = oracle.prefill_f64(q, k, v, g, beta, dinp.scale, cu, h0)
    res["o"] = o.reshape(L, T, H, -1)
    res["ht"] = ht
    if steps:
        st = np.zeros((L, T, H, 128, 128))
        for tau in range(1, T + 1):
            _, _, ck = oracle.prefill_f64(q, k, v, g, beta, dinp.scale, cu, h0,
                                          np.full(L, tau, np.int64))
            st[:, tau - 1] = ck
        res["steps"] = st
    return res
