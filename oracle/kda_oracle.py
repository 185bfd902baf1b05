"""ctypes front end of the FP64 per-token oracle (kda_oracle.c).

Test infrastructure only (see the package docstring).  The C source is
compiled with gcc on first use into ``oracle/_build/`` with -O3 -march=native.
No flag that changes the IEEE semantics is used: no -ffast-math, and -std=c99
keeps floating-point contraction off, so the host's FMA units never fuse a
product into a sum and the results do not depend on the machine.  The library
name carries a hash of the host's native target flags, so a build made on one
machine is never loaded on another CPU.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_lock = threading.Lock()
_lib = None


CFLAGS = ["-O3", "-march=native", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-Wall"]


def _native_tag() -> str:
    """Short hash of the target flags gcc picks for -march=native on this host."""
    import hashlib
    r = subprocess.run(["gcc", "-march=native", "-Q", "--help=target"], capture_output=True,
                       text=True, check=True)
    return hashlib.sha1(r.stdout.encode()).hexdigest()[:10]


_TAG = None


def oracle_library_path() -> str:
    global _TAG
    if _TAG is None:
        _TAG = _native_tag()
    return os.path.join(_BUILD, f"libkda_oracle_{_TAG}.so")


def build_oracle(force: bool = False) -> str:
    """Compile kda_oracle.c into a shared library (gcc -O3 -march=native, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    lib = oracle_library_path()
    stale = (not os.path.exists(lib)) or os.path.getmtime(lib) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = lib + f".tmp{os.getpid()}"
        cmd = ["gcc"] + CFLAGS + ["-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, lib)
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_oracle())
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.kda_oracle_prefill.restype = ctypes.c_int
            lib.kda_oracle_prefill.argtypes = [I64, P, I64, I64, I64, P, P, P, P, P,
                                               ctypes.c_double, P, P, P, P, P, ctypes.c_int,
                                               ctypes.c_int]
            lib.kda_oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f64(x) -> np.ndarray:
    """Exact widening of a torch/numpy array (bf16, fp32, ...) to contiguous fp64."""
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _i64(x) -> np.ndarray:
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.int64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int64))


def prefill_f64(q, k, v, g, beta, scale: float, cu_seqlens, h0=None, ckpt_offsets=None,
                threads: int = 0, mutation: int = 0):
    """Run the per-token FP64 oracle.

    Shapes: q, k, g [T, H, K]; v [T, H, V]; beta [T, H]; h0 [N, H, K, V] or None;
    cu_seqlens [N+1]; ckpt_offsets [N] or None.  Returns (o [T,H,V], ht [N,H,K,V],
    ckpt [N,H,K,V] or None), all float64.
    """
    q, k, v, g, beta, h0 = map(_f64, (q, k, v, g, beta, h0))
    cu = _i64(cu_seqlens)
    ck = _i64(ckpt_offsets)
    T, H, K = q.shape
    V = v.shape[2]
    N = cu.shape[0] - 1
    assert k.shape == (T, H, K) and g.shape == (T, H, K) and v.shape[:2] == (T, H)
    assert beta.shape == (T, H) and int(cu[-1]) == T
    if h0 is not None:
        assert h0.shape == (N, H, K, V)
    out = np.zeros((T, H, V), np.float64)
    ht = np.zeros((N, H, K, V), np.float64)
    ckpt = np.zeros((N, H, K, V), np.float64) if ck is not None else None

    def p(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    rc = _load().kda_oracle_prefill(N, p(cu), H, K, V, p(q), p(k), p(v), p(g), p(beta),
                                    float(scale), p(h0), p(ck), p(out), p(ht), p(ckpt),
                                    int(threads), int(mutation))
    if rc != 0:
        raise ValueError(f"kda_oracle_prefill rejected its arguments (rc={rc})")
    return out, ht, ckpt


def prefill(inp, threads: int = 0, heads: Optional[list] = None, seqs: Optional[list] = None):
    """Oracle on a KDAInputs batch; optionally restricted to some heads/sequences.

    Restricting builds a smaller packed problem from the selected (sequence, head)
    pairs; since (sequence, head) units are independent by definition, the result
    for each selected pair is the full problem's.  Returns a dict with "o"
    [T_sel, H_sel, V] (rows of the selected sequences, in order), "ht", "ckpt",
    "seqs", "heads", and "rows" (the global token rows of o).
    """
    cu = inp.cu_seqlens.to(torch_int64()).tolist()
    N = len(cu) - 1
    seqs = list(range(N)) if seqs is None else list(seqs)
    heads = list(range(inp.num_heads)) if heads is None else list(heads)
    rows = np.concatenate([np.arange(cu[n], cu[n + 1]) for n in seqs]) if seqs else \
        np.zeros(0, np.int64)
    lens = [cu[n + 1] - cu[n] for n in seqs]
    sub_cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)

    def sel(x):
        a = _f64(x)
        return np.ascontiguousarray(a[rows][:, heads])

    h0 = None
    if inp.h0 is not None:
        h0 = np.ascontiguousarray(_f64(inp.h0)[seqs][:, heads])
    ck = None
    if inp.ckpt_offsets is not None:
        ck = _i64(inp.ckpt_offsets)[seqs]
    o, ht, ckpt = prefill_f64(sel(inp.q), sel(inp.k), sel(inp.v), sel(inp.g), sel(inp.beta),
                              inp.scale, sub_cu, h0, ck, threads=threads)
    return {"o": o, "ht": ht, "ckpt": ckpt, "seqs": seqs, "heads": heads, "rows": rows}


def torch_int64():
    import torch
    return torch.int64
