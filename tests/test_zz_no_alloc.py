"""kda_prefill_noalloc: prefill for callers that cannot allocate device memory.

Such callers (graph capture into a pool they do not own, plugins whose host owns
all device memory, real-time paths) cannot hand kda_prefill a workspace; this
entry point runs the same kernels on a scratch area built into the library.
The test calls it through the C ABI twice in a row and compares each result
with kda_prefill's on the same inputs.  It lives in its own file, collected
last, and must pass both alone in a fresh process and after the other tests.
"""
import ctypes

import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs
from tests.gpu_helpers import O_TOL, S_TOL, to_dev

pytestmark = pytest.mark.gpu


def _noalloc_fn():
    from kda_chunked_recurrent_b200 import capi
    lib = ctypes.CDLL(capi.LIB_PATH)
    f = lib.kda_prefill_noalloc
    P = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, ctypes.POINTER(capi.kda_shape_t),
                  P, P, P, P, ctypes.POINTER(capi.kda_options_t), P]
    return f


def _p(t):
    return None if t is None else t.data_ptr()


def test_noalloc_matches_kda_prefill_on_two_calls_in_a_row():
    import kda_chunked_recurrent_b200 as K
    from kda_chunked_recurrent_b200 import capi
    inp = make_inputs([300, 77, 0, 129], 2, seed=31, with_h0=True, with_ckpt=True)
    d = to_dev(inp)
    N, T, H = inp.num_seqs, inp.total_tokens, inp.num_heads
    ref_o, ref_ht, ref_ck = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale,
                                      h0=d["h0"], cu_seqlens=d["cu_seqlens"],
                                      ckpt_offsets=d["ckpt_offsets"])
    torch.cuda.synchronize()
    f = _noalloc_fn()
    shape = capi.make_shape(N, T, H, max(inp.seqlens))
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
        ht = torch.zeros(N, H, 128, 128, dtype=torch.float32, device="cuda")
        ck = torch.zeros(N, H, 128, 128, dtype=torch.float32, device="cuda")
        rc = f(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["g"]), _p(d["beta"]), inp.scale,
               _p(d["h0"]), _p(d["cu_seqlens"]), ctypes.byref(shape), _p(out), _p(ht), _p(ck),
               _p(d["ckpt_offsets"]), None, stream)
        assert rc == 0, capi.kda_status_string(rc)
        torch.cuda.synchronize()
        assert (out.float() - ref_o.float()).abs().max().item() <= O_TOL
        for a, b in ((ht, ref_ht), (ck, ref_ck)):
            num = (a - b).flatten(2).norm(dim=-1)
            den = b.flatten(2).norm(dim=-1).clamp_min(1e-30)
            assert (num / den).max().item() <= S_TOL


def test_noalloc_refuses_shapes_beyond_its_area_without_writing():
    from kda_chunked_recurrent_b200 import capi
    f = _noalloc_fn()
    N, T, H = 8, 8 * 8192, 12   # needs far more than KDA_NOALLOC_SCRATCH_BYTES
    shape = capi.make_shape(N, T, H)
    assert capi.kda_prefill_workspace_size(shape, False) > 48 << 20
    out = torch.full((16,), 3.0, device="cuda")
    x = torch.zeros(16, device="cuda")
    rc = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), 0.1, None, None,
           ctypes.byref(shape), out.data_ptr(), None, None, None, None,
           torch.cuda.current_stream().cuda_stream)
    assert rc == capi.KDA_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)


@pytest.mark.parametrize("variant", [4, 1, 2, 3])   # token, split, fused, hybrid
def test_noalloc_each_variant_back_to_back_matches_kda_prefill(variant):
    """The variants lay the shared area out differently (the fused and hybrid ones
    rely on ready flags cleared by every call): two calls in a row per variant, each
    compared with kda_prefill on its own workspace."""
    import kda_chunked_recurrent_b200 as K
    from kda_chunked_recurrent_b200 import capi
    inp = make_inputs([200, 65, 0, 131], 2, seed=40 + variant, with_h0=True, with_ckpt=True)
    d = to_dev(inp)
    N, T, H = inp.num_seqs, inp.total_tokens, inp.num_heads
    ref_o, ref_ht, ref_ck = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale,
                                      h0=d["h0"], cu_seqlens=d["cu_seqlens"],
                                      ckpt_offsets=d["ckpt_offsets"], variant=variant)
    torch.cuda.synchronize()
    f = _noalloc_fn()
    shape = capi.make_shape(N, T, H, max(inp.seqlens))
    opts = capi.kda_options_t()
    opts.variant = variant
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.zeros(T, H, 128, dtype=torch.bfloat16, device="cuda")
        ht = torch.zeros(N, H, 128, 128, dtype=torch.float32, device="cuda")
        ck = torch.zeros(N, H, 128, 128, dtype=torch.float32, device="cuda")
        rc = f(_p(d["q"]), _p(d["k"]), _p(d["v"]), _p(d["g"]), _p(d["beta"]), inp.scale,
               _p(d["h0"]), _p(d["cu_seqlens"]), ctypes.byref(shape), _p(out), _p(ht), _p(ck),
               _p(d["ckpt_offsets"]), ctypes.byref(opts), stream)
        assert rc == 0, capi.kda_status_string(rc)
        torch.cuda.synchronize()
        assert (out.float() - ref_o.float()).abs().max().item() <= O_TOL
        for a, b in ((ht, ref_ht), (ck, ref_ck)):
            num = (a - b).flatten(2).norm(dim=-1)
            den = b.flatten(2).norm(dim=-1).clamp_min(1e-30)
            assert (num / den).max().item() <= S_TOL


def test_noalloc_refuses_status_word_modes():
    from kda_chunked_recurrent_b200 import capi
    f = _noalloc_fn()
    shape = capi.make_shape(1, 64, 1)
    x = torch.zeros(64 * 128 * 2, device="cuda")
    for flag in (1, 2):   # KDA_FLAG_VALIDATE, KDA_FLAG_TEST_FORCE_TIMEOUT
        opts = capi.kda_options_t()
        opts.flags = flag
        rc = f(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), 0.1, None,
               None, ctypes.byref(shape), x.data_ptr(), None, None, None, ctypes.byref(opts),
               torch.cuda.current_stream().cuda_stream)
        assert rc == capi.KDA_ERR_BAD_OPTION
