"""KDA (Kimi Delta Attention) multi-token recurrent prefill for NVIDIA B200 (sm_100a).

The compute lives in libkda_prefill.so (hand-written CUDA behind the C ABI of
include/kda_prefill.h).  This package only marshals arguments: ``capi`` is
the ctypes binding with the C entry points' names, ``prefill`` a convenience
call that allocates outputs and the workspace with torch and launches on the
current CUDA stream.
"""
from __future__ import annotations

import importlib
from typing import Optional

# The ctypes binding (and with it libkda_prefill.so) is loaded on first use, so
# that the input generators can be imported on machines without the library;
# any use of the CUDA path without the built library raises ImportError.
_CAPI_NAMES = {"kda_prefill", "kda_prefill_describe", "kda_prefill_status",
               "kda_prefill_workspace_size", "kda_status_string", "kda_version",
               "kda_workspace_init", "make_shape", "kda_decode", "make_decode_shape"}
KDA_OK = 0
KDA_VARIANT_AUTO, KDA_VARIANT_SPLIT, KDA_VARIANT_FUSED = 0, 1, 2
KDA_VARIANT_HYBRID, KDA_VARIANT_TOKEN, KDA_VARIANT_STREAM = 3, 4, 5
KDA_DECODE_KEEP_STATE, KDA_DECODE_NARROW, KDA_DECODE_WIDE = 1, 2, 4
KDA_FE_QK_L2NORM, KDA_FE_GATE, KDA_FE_BETA_LOGIT = 1, 2, 4
KDA_FLAG_VALIDATE, KDA_FLAG_TEST_FORCE_TIMEOUT, KDA_FLAG_CU_SEQLENS_I64 = 1, 2, 4


def __getattr__(name):
    if name == "capi":
        return importlib.import_module(".capi", __name__)
    if name in _CAPI_NAMES:
        return getattr(importlib.import_module(".capi", __name__), name)
    raise AttributeError(name)

__all__ = ["capi", "prefill", "decode", "Workspace", "KDAError", "kda_prefill",
           "kda_prefill_describe", "kda_prefill_status", "kda_prefill_workspace_size",
           "kda_status_string", "kda_version", "kda_workspace_init", "make_shape", "kda_decode",
           "make_decode_shape"]


class KDAError(RuntimeError):
    def __init__(self, code: int, where: str = "kda_prefill"):
        from . import capi
        super().__init__(f"{where}: {capi.kda_status_string(code)} (code {code})")
        self.code = code


def _ptr(t):
    return None if t is None else int(t.data_ptr())


class Workspace:
    """A device workspace for kda_prefill, initialised once (status word cleared)."""

    def __init__(self, nbytes: int, device=None, stream=None):
        import torch
        self.nbytes = int(max(nbytes, 1024))
        self.buf = torch.empty(self.nbytes + 256, dtype=torch.uint8, device=device or "cuda")
        base = self.buf.data_ptr()
        self.ptr = (base + 255) // 256 * 256
        from . import capi
        s = stream if stream is not None else torch.cuda.current_stream(self.buf.device)
        rc = capi.kda_workspace_init(self.ptr, self.nbytes, s.cuda_stream)
        if rc != KDA_OK:
            raise KDAError(rc, "kda_workspace_init")

    def status(self, stream=None, clear: bool = True) -> int:
        import torch
        from . import capi
        s = stream if stream is not None else torch.cuda.current_stream(self.buf.device)
        rc, val = capi.kda_prefill_status(self.ptr, s.cuda_stream, clear)
        if rc != KDA_OK:
            raise KDAError(rc, "kda_prefill_status")
        return val


def prefill(q, k, v, g, beta, scale: float, *, h0=None, cu_seqlens=None, num_seqs=None,
            max_seqlen: int = 0, ckpt_offsets=None, out=None, ht=None, ckpt_state=None,
            output_final_state: bool = True, workspace: Optional[Workspace] = None,
            variant: int = KDA_VARIANT_AUTO, flags: int = 0, frontend: Optional[dict] = None,
            stream=None):
    """Launch KDA prefill on device tensors.

    q, k, v: [T, H, 128] bf16; g: [T, H, 128] fp32; beta: [T, H] bf16;
    h0/ht/ckpt_state: [N, H, 128, 128] fp32; cu_seqlens: int32 or int64;
    ckpt_offsets: int32.
    Without cu_seqlens, ``num_seqs`` (default 1) equal-length sequences are assumed.
    ``frontend``: dict(flags=KDA_FE_*, lower_bound=..., l2_eps=..., A_log=[H] fp32,
    dt_bias=[H, 128] fp32) to start from raw projections (with KDA_FE_GATE, ``g`` is the
    raw gate in bf16).
    Returns (out, ht, ckpt_state).
    """
    import torch
    from . import capi
    T, H = int(q.shape[0]), int(q.shape[1])
    N = int(cu_seqlens.numel() - 1) if cu_seqlens is not None else int(num_seqs or 1)
    dev = q.device
    if out is None:
        out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
    if ht is None and output_final_state:
        ht = torch.empty(N, H, 128, 128, dtype=torch.float32, device=dev)
    if ckpt_offsets is not None and ckpt_state is None:
        ckpt_state = torch.empty(N, H, 128, 128, dtype=torch.float32, device=dev)
    shape = capi.make_shape(N, T, H, max_seqlen)
    if cu_seqlens is not None and cu_seqlens.dtype == torch.int64:
        flags |= KDA_FLAG_CU_SEQLENS_I64   # INT64 offsets, narrowed on the device
    opts = {"variant": variant, "flags": flags}
    if frontend is not None:
        opts["frontend"] = capi.make_frontend(
            frontend.get("flags", 0), frontend.get("lower_bound", 0.0),
            frontend.get("l2_eps", 0.0), _ptr(frontend.get("A_log")),
            _ptr(frontend.get("dt_bias")))
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    need = capi.kda_prefill_workspace_size(shape, ckpt_offsets is not None, opts)
    if need == 0:
        raise KDAError(capi.KDA_ERR_BAD_SHAPE, "kda_prefill_workspace_size")
    if workspace is None or workspace.nbytes < need:
        workspace = Workspace(need, dev, s)
    rc = capi.kda_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale), _ptr(h0),
                          _ptr(cu_seqlens), shape, _ptr(out), _ptr(ht), _ptr(ckpt_state),
                          _ptr(ckpt_offsets), workspace.ptr, workspace.nbytes, opts,
                          s.cuda_stream)
    if rc != KDA_OK:
        raise KDAError(rc)
    return out, ht, ckpt_state


def decode(q, k, v, g, beta, scale: float, state, *, state_indices=None, out=None,
           step_states=None, return_step_states: bool = False, keep_state: bool = False,
           device_status=None, flags: int = 0, frontend: Optional[dict] = None, stream=None):
    """Decode / draft verification over a state pool (kda_decode).

    q, k, v: [N, T, H, 128] bf16; g: [N, T, H, 128] fp32; beta: [N, T, H] bf16;
    state: [P, H, 128, 128] fp32 pool, updated in place unless ``keep_state``;
    state_indices: [N] int32 slots (negative = padding row) or None (slot n).
    ``flags`` may add KDA_DECODE_NARROW / KDA_DECODE_WIDE (kernel shape).
    ``frontend``: dict(flags=KDA_FE_*, lower_bound=..., l2_eps=..., A_log=[H] fp32,
    dt_bias=[H, 128] fp32); with KDA_FE_GATE, ``g`` is the raw gate in bf16.
    Returns (out, step_states); step_states [N, T, H, 128, 128] when requested.
    """
    import torch
    from . import capi
    N, T, H = int(q.shape[0]), int(q.shape[1]), int(q.shape[2])
    P = int(state.shape[0])
    dev = q.device
    if out is None:
        out = torch.empty(N, T, H, 128, dtype=torch.bfloat16, device=dev)
    if step_states is None and return_step_states:
        step_states = torch.empty(N, T, H, 128, 128, dtype=torch.float32, device=dev)
    shape = capi.make_decode_shape(N, T, H, P)
    s = stream if stream is not None else torch.cuda.current_stream(dev)
    fe = None
    if frontend is not None:
        fe = capi.make_frontend(frontend.get("flags", 0), frontend.get("lower_bound", 0.0),
                                frontend.get("l2_eps", 0.0), _ptr(frontend.get("A_log")),
                                _ptr(frontend.get("dt_bias")))
    rc = capi.kda_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), float(scale),
                         _ptr(state), _ptr(state_indices), shape, _ptr(out), _ptr(step_states),
                         _ptr(device_status),
                         int(flags) | (KDA_DECODE_KEEP_STATE if keep_state else 0),
                         s.cuda_stream, fe)
    if rc != KDA_OK:
        raise KDAError(rc, "kda_decode")
    return out, step_states
