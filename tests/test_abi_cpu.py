"""C ABI checks that need no GPU: the library loads, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call."""
import ctypes
import os
import re

import pytest

from kda_chunked_recurrent_b200 import capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda_prefill.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("kda_prefill", "kda_prefill_workspace_size", "kda_prefill_status",
              "kda_status_string", "kda_prefill_describe", "kda_workspace_init", "kda_version"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(capi.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_status_strings_cover_all_codes():
    for code in (0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 16, 17, 18, 19):
        s = capi.kda_status_string(code)
        assert s and s != "unknown status"
    assert capi.kda_status_string(12345) == "unknown status"


def test_workspace_size_grows_with_work():
    a = capi.kda_prefill_workspace_size(capi.make_shape(1, 512, 12), False)
    b = capi.kda_prefill_workspace_size(capi.make_shape(1, 8192, 12), False)
    c = capi.kda_prefill_workspace_size(capi.make_shape(1, 8192, 12), True)
    assert 0 < a < b < c
    assert capi.kda_prefill_workspace_size(capi.make_shape(0, 512, 12), False) == 0
    assert capi.kda_prefill_workspace_size(capi.make_shape(1, 512, 0), False) == 0
    assert capi.kda_prefill_workspace_size(capi.make_shape(1, -1, 1), False) == 0


def test_describe_reports_grid_and_variant():
    d = capi.kda_prefill_describe(capi.make_shape(8, 65536, 12, 8192), False, {"variant": 1})
    assert "variant=split" in d and "chunk=64" in d and "recurrence_grid=96x448" in d
    h = capi.kda_prefill_describe(capi.make_shape(8, 65536, 12, 8192), False, {"variant": 3})
    assert "variant=hybrid" in h and "prepare_chunks=" in h and "recurrence CTAs 96" in h
    st = capi.kda_prefill_describe(capi.make_shape(8, 65536, 12, 8192), False, {"variant": 5})
    assert "variant=stream" in st and "recurrences 96" in st and "one CTA per SM" in st
    # stream and split records take the same workspace bytes
    ws = [capi.kda_prefill_workspace_size(capi.make_shape(8, 65536, 12, 8192), False,
                                          {"variant": v}) for v in (1, 5)]
    assert ws[0] == ws[1]


def test_stream_variant_needs_free_slots():
    # at most one chain per SM (148 without a GPU)
    big = capi.make_shape(2, 2 * 128, 160, 128)           # 320 chains
    assert capi.kda_prefill_describe(big, False, {"variant": 5}).startswith("variant=stream")
    o = capi.kda_options_t()
    o.variant = 5
    assert call(fake_args(T=1, H=150, h0=None, ht=None, opts=o)) == capi.KDA_ERR_BAD_OPTION


# --- host-side validation with fake, never-dereferenced device addresses ----------
BASE = 0x7F0000000000
MB = 1 << 20


def fake_args(T=128, H=2, N=1, ckpt=False, **over):
    a = dict(q=BASE, k=BASE + 1 * MB, v=BASE + 2 * MB, g=BASE + 3 * MB, beta=BASE + 5 * MB,
             scale=0.088, h0=BASE + 6 * MB, cu=None, shape=capi.make_shape(N, T, H),
             out=BASE + 8 * MB, ht=BASE + 10 * MB, ck=None, cko=None,
             ws=BASE + 64 * MB, wsb=capi.kda_prefill_workspace_size(capi.make_shape(N, T, H), ckpt),
             opts=None)
    if ckpt:
        a["ck"] = BASE + 12 * MB
        a["cko"] = BASE + 14 * MB
    a.update(over)
    return a


def call(a):
    return capi.kda_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["h0"], a["cu"],
                            a["shape"], a["out"], a["ht"], a["ck"], a["cko"], a["ws"], a["wsb"],
                            a["opts"], None)


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "beta", "out", "ws"])
def test_null_pointer_rejected(field):
    assert call(fake_args(**{field: None})) == capi.KDA_ERR_NULL_ARG


def test_bad_shapes_rejected():
    assert call(fake_args(shape=capi.make_shape(0, 128, 2))) == capi.KDA_ERR_BAD_SHAPE
    assert call(fake_args(shape=capi.make_shape(1, 128, 0))) == capi.KDA_ERR_BAD_SHAPE
    assert call(fake_args(shape=capi.make_shape(1, -5, 2))) == capi.KDA_ERR_BAD_SHAPE
    # fixed layout needs T divisible by N
    assert call(fake_args(shape=capi.make_shape(3, 128, 2))) == capi.KDA_ERR_BAD_SHAPE


@pytest.mark.parametrize("field,delta", [("q", 8), ("k", 2), ("v", 4), ("g", 4), ("out", 8),
                                         ("beta", 1), ("h0", 4), ("ht", 8), ("ws", 128)])
def test_misaligned_rejected(field, delta):
    a = fake_args()
    a[field] = a[field] + delta
    assert call(a) == capi.KDA_ERR_MISALIGNED


def test_unpaired_checkpoint_rejected():
    a = fake_args(ckpt=True)
    assert call(dict(a, cko=None)) == capi.KDA_ERR_UNPAIRED_CKPT
    assert call(dict(a, ck=None)) == capi.KDA_ERR_UNPAIRED_CKPT


def test_partial_state_alias_rejected():
    a = fake_args()
    assert call(dict(a, ht=a["h0"] + 65536)) == capi.KDA_ERR_PARTIAL_ALIAS
    b = fake_args(ckpt=True)
    assert call(dict(b, ck=b["h0"])) == capi.KDA_ERR_PARTIAL_ALIAS


def test_output_alias_rejected():
    a = fake_args()
    assert call(dict(a, out=a["q"])) == capi.KDA_ERR_OUT_ALIAS
    assert call(dict(a, out=a["h0"])) == capi.KDA_ERR_OUT_ALIAS
    assert call(dict(a, ht=a["g"])) == capi.KDA_ERR_OUT_ALIAS
    assert call(dict(a, ws=a["v"])) == capi.KDA_ERR_OUT_ALIAS


def test_workspace_too_small_rejected():
    a = fake_args()
    assert call(dict(a, wsb=a["wsb"] - 1)) == capi.KDA_ERR_WORKSPACE_TOO_SMALL


def test_bad_options_rejected():
    o = capi.kda_options_t()
    o.variant = 7
    assert call(fake_args(opts=o)) == capi.KDA_ERR_BAD_OPTION
    o.variant = 0
    o.flags = 1 << 9
    assert call(fake_args(opts=o)) == capi.KDA_ERR_BAD_OPTION


def test_valid_arguments_reach_the_device_check_without_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("would launch on fake pointers")
    assert call(fake_args()) == capi.KDA_ERR_UNSUPPORTED_DEVICE
    assert call(fake_args(ht=BASE + 6 * MB)) == capi.KDA_ERR_UNSUPPORTED_DEVICE  # exact alias ok


def test_auto_variant_follows_the_table():
    # few (sequence, head) chains: the fused launch; chains filling the GPU: split
    few = capi.kda_prefill_describe(capi.make_shape(1, 8192, 12), False)
    short = capi.kda_prefill_describe(capi.make_shape(1, 512, 12), False)
    many = capi.kda_prefill_describe(capi.make_shape(8, 65536, 12), False)
    assert "variant=fused" in few and "recurrence CTAs 12" in few, few
    assert "variant=split" in short, short
    assert "variant=hybrid" in many, many
    mid = capi.kda_prefill_describe(capi.make_shape(4, 32768, 12), False)    # 48 chains
    wide = capi.kda_prefill_describe(capi.make_shape(6, 49152, 12), False)   # 72 chains
    huge = capi.kda_prefill_describe(capi.make_shape(32, 16384, 12), False)  # 384 chains
    assert "variant=fused" in mid and "variant=hybrid" in wide, (mid, wide)
    assert "variant=split" in huge, huge


def _hybrid_tail(N, T_seq, H, fe=False):
    import re
    opts = {"variant": 3}
    if fe:
        opts["frontend"] = {"flags": 7, "lower_bound": -5.0, "l2_eps": 1e-6}
    d = capi.kda_prefill_describe(capi.make_shape(N, N * T_seq, H, T_seq), False, opts)
    m = re.search(r"prepare_chunks=(\d+)/(\d+)", d)
    assert m, d
    first, jmax = int(m.group(1)), int(m.group(2))
    return jmax - first, jmax


def test_hybrid_tail_follows_the_throughput_rule():
    # the tail (chunk rows made inside the fused launch) grows with the chunks per
    # sequence and the free SMs, shrinks with the chains and with a slower prepare
    tails = {N: _hybrid_tail(N, 8192, 12) for N in (5, 6, 7, 8, 9, 10)}
    for N, (tail, jmax) in tails.items():
        assert jmax == 128 and 1 <= tail <= jmax - 1, (N, tail)
    seq = [tails[N][0] for N in sorted(tails)]
    assert all(a > b for a, b in zip(seq, seq[1:])), seq
    t_long, j_long = _hybrid_tail(8, 16384, 12)
    assert j_long == 256 and abs(t_long - 2 * tails[8][0]) <= 1, (t_long, tails[8])
    fe_tail, _ = _hybrid_tail(8, 8192, 12, fe=True)
    assert 1 <= fe_tail < tails[8][0]
    # two chunks per sequence: the tail is clamped to leave one row for the prepare launch
    assert _hybrid_tail(8, 128, 12) == (1, 2)
    # nearly every SM carries a chain: the fused prepare groups get the one-row minimum
    assert _hybrid_tail(11, 8192, 12)[0] == 4 and _hybrid_tail(12, 8192, 12)[0] == 1
    # the rule at the measured shapes: 96 chains on 148 SMs keep 20 of 128 rows in the
    # fused launch, 72 chains 40
    assert tails[8][0] == 20 and tails[6][0] == 40, tails


def test_fused_variant_needs_free_sms():
    torch = pytest.importorskip("torch")
    o = capi.kda_options_t()
    o.variant = 2
    # 140 chains leave fewer than 16 SMs of the 148 for prepare CTAs
    assert call(fake_args(T=1, H=140, h0=None, ht=None, opts=o)) == capi.KDA_ERR_BAD_OPTION
    if not torch.cuda.is_available():
        assert call(fake_args(H=4, opts=o)) == capi.KDA_ERR_UNSUPPORTED_DEVICE


def test_int64_cu_seqlens_validation():
    torch = pytest.importorskip("torch")
    o = capi.kda_options_t()
    o.flags = capi.KDA_FLAG_CU_SEQLENS_I64
    # the flag describes a cu_seqlens array: meaningless without one
    assert call(fake_args(opts=o)) == capi.KDA_ERR_BAD_OPTION
    wsb = capi.kda_prefill_workspace_size(capi.make_shape(2, 128, 2), False)
    a = fake_args(N=2, cu=BASE + 20 * MB + 4, shape=capi.make_shape(2, 128, 2), wsb=wsb, opts=o)
    assert call(a) == capi.KDA_ERR_MISALIGNED        # INT64 entries need 8-byte alignment
    if not torch.cuda.is_available():
        assert call(dict(a, cu=BASE + 20 * MB)) == capi.KDA_ERR_UNSUPPORTED_DEVICE


def test_prefill_frontend_validation():
    torch = pytest.importorskip("torch")
    G, N2, B = capi.KDA_FE_GATE, capi.KDA_FE_QK_L2NORM, capi.KDA_FE_BETA_LOGIT

    def opts(flags, lb=-5.0, eps=1e-6, A=BASE + 30 * MB, dt=BASE + 31 * MB):
        o = capi.kda_options_t()
        o._fe = capi.make_frontend(flags, lb, eps, A, dt)
        o.frontend = ctypes.pointer(o._fe)
        return o

    assert call(fake_args(opts=opts(1 << 6))) == capi.KDA_ERR_BAD_OPTION
    assert call(fake_args(opts=opts(G, lb=0.0))) == capi.KDA_ERR_BAD_OPTION
    assert call(fake_args(opts=opts(G, lb=float("nan")))) == capi.KDA_ERR_BAD_OPTION
    assert call(fake_args(opts=opts(N2, eps=-1.0))) == capi.KDA_ERR_BAD_OPTION
    assert call(fake_args(opts=opts(G, A=None))) == capi.KDA_ERR_NULL_ARG
    assert call(fake_args(opts=opts(G, dt=BASE + 31 * MB + 8))) == capi.KDA_ERR_MISALIGNED
    # the gate parameters are inputs: an output on top of them is refused
    assert call(fake_args(opts=opts(G, dt=BASE + 8 * MB))) == capi.KDA_ERR_OUT_ALIAS
    # beta from logits is accepted by every variant (the chunked ones hold T diag(beta)
    # in FP16, which keeps a squashed FP32 beta on its diagonal to 2^-11)
    chunked = opts(G | N2 | B)
    chunked.variant = capi.KDA_VARIANT_SPLIT
    tok = opts(G | N2 | B)
    tok.variant = capi.KDA_VARIANT_TOKEN
    # with the gate switch g is BF16: a buffer right after its half size does not overlap it
    a = fake_args(opts=opts(G | N2))
    half_g_end = a["g"] + 128 * 2 * 128 * 2
    if not torch.cuda.is_available():
        assert call(dict(a, out=half_g_end)) == capi.KDA_ERR_UNSUPPORTED_DEVICE
        assert call(a) == capi.KDA_ERR_UNSUPPORTED_DEVICE
        assert call(fake_args(opts=tok)) == capi.KDA_ERR_UNSUPPORTED_DEVICE
        assert call(fake_args(opts=chunked)) == capi.KDA_ERR_UNSUPPORTED_DEVICE
        assert call(fake_args(opts=opts(B))) == capi.KDA_ERR_UNSUPPORTED_DEVICE


def test_noalloc_host_checks_before_any_device_work():
    """kda_prefill_noalloc refuses the status-word modes, then bad shapes, then a
    missing B200, all on the host."""
    lib = ctypes.CDLL(capi.LIB_PATH)
    f = lib.kda_prefill_noalloc
    P = ctypes.c_void_p
    f.restype = ctypes.c_int
    f.argtypes = [P, P, P, P, P, ctypes.c_float, P, P, ctypes.POINTER(capi.kda_shape_t),
                  P, P, P, P, ctypes.POINTER(capi.kda_options_t), P]
    x = BASE
    shape = capi.make_shape(1, 64, 1)
    for flag in (capi.KDA_FLAG_VALIDATE, capi.KDA_FLAG_TEST_FORCE_TIMEOUT):
        o = capi.kda_options_t()
        o.flags = flag
        assert f(x, x, x, x, x, 0.1, None, None, ctypes.byref(shape), x + MB, None, None, None,
                 ctypes.byref(o), None) == capi.KDA_ERR_BAD_OPTION
    bad = capi.make_shape(0, 64, 1)
    assert f(x, x, x, x, x, 0.1, None, None, ctypes.byref(bad), x + MB, None, None, None,
             None, None) == capi.KDA_ERR_BAD_SHAPE
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        assert f(x, x, x, x, x, 0.1, None, None, ctypes.byref(shape), x + MB, None, None, None,
                 None, None) == capi.KDA_ERR_UNSUPPORTED_DEVICE
