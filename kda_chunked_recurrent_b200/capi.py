"""ctypes binding of libkda_prefill.so (the C ABI of include/kda_prefill.h).

Argument marshalling only: every step of the prefill runs in the library's
CUDA kernels.  The names match the C entry points.  There is no CPU fallback:
importing this module fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda_prefill.so")

# status codes (kda_status_t)
KDA_OK = 0
KDA_ERR_NULL_ARG = 1
KDA_ERR_BAD_SHAPE = 2
KDA_ERR_MISALIGNED = 3
KDA_ERR_UNPAIRED_CKPT = 4
KDA_ERR_PARTIAL_ALIAS = 5
KDA_ERR_OUT_ALIAS = 6
KDA_ERR_WORKSPACE_TOO_SMALL = 7
KDA_ERR_UNSUPPORTED_DEVICE = 8
KDA_ERR_LAUNCH_FAILED = 9
KDA_ERR_BAD_OPTION = 10
KDA_ERR_SCRATCH_UNAVAILABLE = 11
KDA_ERR_BAD_CU_SEQLENS = 16
KDA_ERR_BAD_CKPT_OFFSET = 17
KDA_ERR_TIMEOUT = 18
KDA_ERR_BAD_STATE_INDEX = 19

KDA_VARIANT_AUTO = 0
KDA_VARIANT_SPLIT = 1
KDA_VARIANT_FUSED = 2
KDA_VARIANT_HYBRID = 3
KDA_VARIANT_TOKEN = 4
KDA_VARIANT_STREAM = 5
KDA_DECODE_KEEP_STATE = 1
KDA_FE_QK_L2NORM = 1
KDA_FE_GATE = 2
KDA_FE_BETA_LOGIT = 4
KDA_DECODE_NARROW = 2
KDA_DECODE_WIDE = 4
KDA_FLAG_VALIDATE = 1
KDA_FLAG_TEST_FORCE_TIMEOUT = 2
KDA_FLAG_CU_SEQLENS_I64 = 4


class kda_shape_t(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("total_tokens", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("max_seqlen", ctypes.c_int32)]


class kda_decode_shape_t(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("tokens_per_seq", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("pool_size", ctypes.c_int32)]


class kda_frontend_t(ctypes.Structure):
    _fields_ = [("flags", ctypes.c_uint32), ("lower_bound", ctypes.c_float),
                ("l2_eps", ctypes.c_float), ("A_log", ctypes.c_void_p),
                ("dt_bias", ctypes.c_void_p)]


class kda_options_t(ctypes.Structure):
    _fields_ = [("variant", ctypes.c_int32), ("flags", ctypes.c_uint32),
                ("events", ctypes.c_void_p * 3), ("frontend", ctypes.POINTER(kda_frontend_t)),
                ("reserved", ctypes.c_int32 * 2)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m kda_chunked_recurrent_b200.build`"
            " (there is no fallback implementation)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    lib.kda_version.restype = ctypes.c_int
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [ctypes.c_int]
    lib.kda_prefill_workspace_size.restype = ctypes.c_size_t
    lib.kda_prefill_workspace_size.argtypes = [ctypes.POINTER(kda_shape_t), ctypes.c_int,
                                               ctypes.POINTER(kda_options_t)]
    lib.kda_workspace_init.restype = ctypes.c_int
    lib.kda_workspace_init.argtypes = [P, ctypes.c_size_t, P]
    lib.kda_prefill.restype = ctypes.c_int
    lib.kda_prefill.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, ctypes.POINTER(kda_shape_t),
                                P, P, P, P, P, ctypes.c_size_t, ctypes.POINTER(kda_options_t), P]
    lib.kda_prefill_status.restype = ctypes.c_int
    lib.kda_prefill_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32), ctypes.c_int]
    lib.kda_prefill_describe.restype = ctypes.c_int
    lib.kda_prefill_describe.argtypes = [ctypes.POINTER(kda_shape_t), ctypes.c_int,
                                         ctypes.POINTER(kda_options_t), ctypes.c_char_p,
                                         ctypes.c_size_t]
    lib.kda_decode.restype = ctypes.c_int
    lib.kda_decode.argtypes = [P, P, P, P, P, ctypes.c_float, P, P,
                               ctypes.POINTER(kda_decode_shape_t), P, P, P, ctypes.c_uint32,
                               ctypes.POINTER(kda_frontend_t), P]
    return lib


lib = _load()


def _opt(options):
    if options is None:
        return None
    if isinstance(options, kda_options_t):
        return ctypes.byref(options)
    o = kda_options_t()
    o.variant = int(options.get("variant", 0))
    o.flags = int(options.get("flags", 0))
    for i, ev in enumerate(options.get("events") or ()):
        o.events[i] = ev
    fe = options.get("frontend")
    if fe is not None:
        o._fe = fe if isinstance(fe, kda_frontend_t) else make_frontend(**fe)
        o.frontend = ctypes.pointer(o._fe)
    return ctypes.byref(o)


def make_shape(num_seqs, total_tokens, num_heads, max_seqlen=0) -> kda_shape_t:
    return kda_shape_t(int(num_seqs), int(total_tokens), int(num_heads), int(max_seqlen))


def kda_version() -> int:
    return int(lib.kda_version())


def kda_status_string(code: int) -> str:
    return lib.kda_status_string(int(code)).decode()


def kda_prefill_workspace_size(shape: kda_shape_t, has_ckpt: bool, options=None) -> int:
    return int(lib.kda_prefill_workspace_size(ctypes.byref(shape), int(bool(has_ckpt)),
                                              _opt(options)))


def kda_workspace_init(workspace: int, workspace_bytes: int, stream: int) -> int:
    return int(lib.kda_workspace_init(workspace, workspace_bytes, stream))


def kda_prefill(q, k, v, g, beta, scale, h0, cu_seqlens, shape, out, ht, ckpt_state,
                ckpt_offsets, workspace, workspace_bytes, options, stream) -> int:
    """All pointer arguments are integers (device addresses) or None."""
    return int(lib.kda_prefill(q, k, v, g, beta, ctypes.c_float(scale), h0, cu_seqlens,
                               ctypes.byref(shape), out, ht, ckpt_state, ckpt_offsets, workspace,
                               int(workspace_bytes), _opt(options), stream))


def kda_prefill_status(workspace: int, stream: int, clear: bool = False):
    val = ctypes.c_int32(0)
    rc = int(lib.kda_prefill_status(workspace, stream, ctypes.byref(val), int(bool(clear))))
    return rc, int(val.value)


def kda_prefill_describe(shape: kda_shape_t, has_ckpt: bool, options=None) -> str:
    buf = ctypes.create_string_buffer(512)
    lib.kda_prefill_describe(ctypes.byref(shape), int(bool(has_ckpt)), _opt(options), buf, 512)
    return buf.value.decode()


def make_decode_shape(num_seqs, tokens_per_seq, num_heads, pool_size) -> kda_decode_shape_t:
    return kda_decode_shape_t(int(num_seqs), int(tokens_per_seq), int(num_heads), int(pool_size))


def make_frontend(flags, lower_bound=0.0, l2_eps=0.0, A_log=None, dt_bias=None) -> kda_frontend_t:
    """A_log / dt_bias are device addresses (integers) or None."""
    return kda_frontend_t(int(flags), float(lower_bound), float(l2_eps), A_log, dt_bias)


def kda_decode(q, k, v, g, beta, scale, state, state_indices, shape, out, step_states,
               device_status, flags, stream, frontend=None) -> int:
    """All pointer arguments are integers (device addresses) or None; frontend is a
    kda_frontend_t or None."""
    fe = None if frontend is None else ctypes.byref(frontend)
    return int(lib.kda_decode(q, k, v, g, beta, ctypes.c_float(scale), state, state_indices,
                              ctypes.byref(shape), out, step_states, device_status,
                              int(flags), fe, stream))
