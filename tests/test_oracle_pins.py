"""The oracle against its pins, and planted mistakes against the same pins (CPU)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as P


def oracle_fn(mutation=0):
    def f(q, k, v, g, beta, scale, cu, h0=None, ck=None):
        return oracle.prefill_f64(q, k, v, g, beta, scale, cu, h0, ck, threads=1,
                                  mutation=mutation)
    return f


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    ok, detail = pin(oracle_fn())
    assert ok, f"{pin.__name__}: {detail}"


MUTATIONS = {
    1: "u uses the state before the decay",
    2: "read-out before the update",
    3: "decay applied to value columns",
    4: "sign of the correction flipped",
    5: "beta ignored in the update",
    6: "decay uses g of the next token",
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS), ids=lambda m: MUTATIONS[m])
def test_planted_mistake_is_caught(mutation):
    f = oracle_fn(mutation)
    failed = []
    for pin in P.ALL_PINS:
        try:
            ok, _ = pin(f)
        except Exception:
            ok = False
        if not ok:
            failed.append(pin.__name__)
    assert failed, f"no pin catches planted mistake {mutation}: {MUTATIONS[mutation]}"


def test_oracle_rejects_bad_offsets():
    q, k, v, g, beta, cu, S0 = P.random_case(1, [3, 4])
    with pytest.raises(ValueError):
        oracle.prefill_f64(q, k, v, g, beta, 1.0, np.array([1, 3, 7]), None, None)
    with pytest.raises(ValueError):
        oracle.prefill_f64(q, k, v, g, beta, 1.0, cu, None, np.array([4, 1]))


def test_oracle_threads_do_not_change_results():
    q, k, v, g, beta, cu, S0 = P.random_case(2, [17, 5, 9], H=3, h0=True)
    a = oracle.prefill_f64(q, k, v, g, beta, 0.3, cu, S0, None, threads=1)
    b = oracle.prefill_f64(q, k, v, g, beta, 0.3, cu, S0, None, threads=4)
    for x, y in zip(a[:2], b[:2]):
        assert np.array_equal(x, y)


def test_oracle_on_generated_inputs_matches_chunked_at_full_width():
    """K = V = 128 with the benchmark's input distribution, several chunks plus a tail."""
    from kda_chunked_recurrent_b200.inputs import make_inputs
    inp = make_inputs([150, 64, 1], 2, seed=21, with_h0=True, with_ckpt=True)
    o, ht, c = oracle.prefill_f64(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.scale,
                                  inp.cu_seqlens, inp.h0, inp.ckpt_offsets)
    o2, h2, c2 = oracle.chunked_prefill_f64(
        inp.q.double().numpy(), inp.k.double().numpy(), inp.v.double().numpy(),
        inp.g.double().numpy(), inp.beta.double().numpy(), inp.scale,
        inp.cu_seqlens.numpy(), inp.h0.double().numpy(), inp.ckpt_offsets.numpy(), chunk=64)
    assert np.abs(o - o2).max() < 1e-12
    assert np.abs(ht - h2).max() < 1e-12
    assert np.abs(c - c2).max() < 1e-12
