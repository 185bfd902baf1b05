"""Host-side checks of kda_decode and of the token variant of kda_prefill that
need no GPU: argument validation happens before any CUDA call."""
import pytest

from kda_chunked_recurrent_b200 import capi

BASE = 0x7F0000000000
MB = 1 << 20


def dargs(N=4, T=1, H=2, P=8, **over):
    a = dict(q=BASE, k=BASE + 1 * MB, v=BASE + 2 * MB, g=BASE + 3 * MB, beta=BASE + 5 * MB,
             scale=0.088, state=BASE + 16 * MB, idx=BASE + 6 * MB,
             shape=capi.make_decode_shape(N, T, H, P), out=BASE + 8 * MB, steps=None,
             status=None, flags=0, fe=None)
    a.update(over)
    return a


def dcall(a):
    return capi.kda_decode(a["q"], a["k"], a["v"], a["g"], a["beta"], a["scale"], a["state"],
                           a["idx"], a["shape"], a["out"], a["steps"], a["status"], a["flags"],
                           None, a["fe"])


@pytest.mark.parametrize("field", ["q", "k", "v", "g", "beta", "state", "out"])
def test_decode_null_pointer_rejected(field):
    assert dcall(dargs(**{field: None})) == capi.KDA_ERR_NULL_ARG


def test_decode_bad_shapes_rejected():
    for shp in [(0, 1, 2, 8), (4, 0, 2, 8), (4, 1, 0, 8), (4, 1, 2, 0)]:
        assert dcall(dargs(shape=capi.make_decode_shape(*shp))) == capi.KDA_ERR_BAD_SHAPE
    # without state_indices sequence n uses slot n: the pool must hold N slots
    assert dcall(dargs(idx=None, shape=capi.make_decode_shape(9, 1, 2, 8))) == \
        capi.KDA_ERR_BAD_SHAPE


@pytest.mark.parametrize("field,delta", [("q", 8), ("g", 4), ("out", 2), ("state", 4),
                                         ("beta", 1), ("idx", 2)])
def test_decode_misaligned_rejected(field, delta):
    a = dargs()
    a[field] = a[field] + delta
    assert dcall(a) == capi.KDA_ERR_MISALIGNED


def test_decode_aliasing_rejected():
    a = dargs()
    assert dcall(dict(a, out=a["q"])) == capi.KDA_ERR_OUT_ALIAS
    assert dcall(dict(a, state=a["v"])) == capi.KDA_ERR_OUT_ALIAS
    assert dcall(dict(a, steps=a["state"] + 4 * 65536)) == capi.KDA_ERR_OUT_ALIAS
    assert dcall(dict(a, status=a["idx"])) == capi.KDA_ERR_OUT_ALIAS
    assert dcall(dict(a, out=a["state"])) == capi.KDA_ERR_OUT_ALIAS


def test_decode_unknown_flag_rejected():
    assert dcall(dargs(flags=1 << 5)) == capi.KDA_ERR_BAD_OPTION
    both = capi.KDA_DECODE_NARROW | capi.KDA_DECODE_WIDE
    assert dcall(dargs(flags=both)) == capi.KDA_ERR_BAD_OPTION


def test_decode_valid_arguments_reach_the_device_check_without_gpu():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("would launch on fake pointers")
    assert dcall(dargs()) == capi.KDA_ERR_UNSUPPORTED_DEVICE
    assert dcall(dargs(idx=None, flags=capi.KDA_DECODE_KEEP_STATE,
                       steps=BASE + 64 * MB, status=BASE + 7 * MB)) == \
        capi.KDA_ERR_UNSUPPORTED_DEVICE


def test_token_variant_describe_and_workspace():
    shp = capi.make_shape(32, 32 * 16, 12, 16)
    d = capi.kda_prefill_describe(shp, False, {"variant": capi.KDA_VARIANT_TOKEN})
    assert "variant=token" in d and "grid=384x256 (wide" in d, d     # 384 units: one CTA each
    few = capi.kda_prefill_describe(capi.make_shape(2, 2 * 48, 12, 48), False,
                                    {"variant": capi.KDA_VARIANT_TOKEN})
    assert "grid=96x256 (narrow" in few, few                         # 24 units: four CTAs each
    # the table: up to 16 tokens always, up to 32 for at most 16 units
    auto = capi.kda_prefill_describe(shp, False)
    assert "variant=token" in auto, auto
    one = capi.kda_prefill_describe(capi.make_shape(1, 32, 12, 32), False)
    assert "variant=token" in one, one
    mid = capi.kda_prefill_describe(capi.make_shape(8, 8 * 32, 12, 32), False)
    assert "variant=split" in mid, mid
    longer = capi.kda_prefill_describe(capi.make_shape(32, 32 * 2048, 12, 2048), False)
    assert "variant=token" not in longer, longer
    # the token variant keeps no chunk records: its workspace is far smaller
    w_tok = capi.kda_prefill_workspace_size(shp, False, {"variant": capi.KDA_VARIANT_TOKEN})
    w_auto = capi.kda_prefill_workspace_size(shp, False)
    assert 0 < w_tok < w_auto // 10


def test_decode_frontend_validation():
    fe = lambda flags, lb=-5.0, eps=1e-6, A=BASE + 30 * MB, dt=BASE + 31 * MB: \
        capi.make_frontend(flags, lb, eps, A, dt)
    G, N2, B = capi.KDA_FE_GATE, capi.KDA_FE_QK_L2NORM, capi.KDA_FE_BETA_LOGIT
    assert dcall(dargs(fe=fe(1 << 4))) == capi.KDA_ERR_BAD_OPTION           # unknown switch
    for lb in (0.0, -5.5, 1.0, float("nan"), float("-inf")):                # bound in [-5, 0)
        assert dcall(dargs(fe=fe(G, lb=lb))) == capi.KDA_ERR_BAD_OPTION
    assert dcall(dargs(fe=fe(N2, eps=-1.0))) == capi.KDA_ERR_BAD_OPTION
    assert dcall(dargs(fe=fe(N2, eps=float("nan")))) == capi.KDA_ERR_BAD_OPTION
    assert dcall(dargs(fe=fe(G, A=None))) == capi.KDA_ERR_NULL_ARG
    assert dcall(dargs(fe=fe(G, dt=None))) == capi.KDA_ERR_NULL_ARG
    assert dcall(dargs(fe=fe(G, dt=BASE + 31 * MB + 4))) == capi.KDA_ERR_MISALIGNED
    # dt_bias must not overlap an output
    assert dcall(dargs(fe=fe(G, dt=BASE + 16 * MB))) == capi.KDA_ERR_OUT_ALIAS
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        # switches that need no parameters, and the full set, reach the device check
        assert dcall(dargs(fe=fe(B | N2, A=None, dt=None))) == capi.KDA_ERR_UNSUPPORTED_DEVICE
        assert dcall(dargs(fe=fe(G | N2 | B, lb=-5.0))) == capi.KDA_ERR_UNSUPPORTED_DEVICE
