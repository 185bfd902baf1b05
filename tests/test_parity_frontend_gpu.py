"""Prefill from raw projections: the input front end (q/k L2 norm, gate from A_log and
dt_bias under a lower bound, beta from its logit) inside every
variant's kernels vs the FP64 front-end oracle followed by the FP64 recurrence oracle
(needs a B200)."""
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_frontend_inputs
from tests.gpu_helpers import assert_parity, compare, run_gpu

pytestmark = pytest.mark.gpu

SPLIT, FUSED, HYBRID, TOKEN = 1, 2, 3, 4


def fe_dict(A_log, dt_bias, flags=7, lower_bound=-5.0):
    return {"flags": flags, "lower_bound": lower_bound, "l2_eps": 1e-6, "A_log": A_log,
            "dt_bias": dt_bias}


def chunked_inputs(lens, H, seed, **kw):
    """Raw q, k and gate; beta given as a BF16 value (the chunked variants' contract)."""
    inp, A_log, dt = make_frontend_inputs(lens, H, seed, **kw)
    inp.beta = torch.sigmoid(inp.beta.float()).to(torch.bfloat16)
    return inp, A_log, dt


@pytest.mark.parametrize("variant", [SPLIT, FUSED, HYBRID])
def test_frontend_norm_and_gate_chunked_variants(variant):
    inp, A_log, dt = chunked_inputs([300, 0, 129, 64, 1, 77], 3, seed=800 + variant,
                                    with_h0=True, with_ckpt=True)
    fe = fe_dict(A_log, dt, flags=3)
    assert_parity(compare(inp, run_gpu(inp, variant=variant, frontend=fe), frontend=fe))


def test_frontend_all_switches_token_variant():
    inp, A_log, dt = make_frontend_inputs([13, 0, 16, 1, 9], 3, seed=804, with_h0=True,
                                          with_ckpt=True)
    fe = fe_dict(A_log, dt)
    assert_parity(compare(inp, run_gpu(inp, variant=TOKEN, frontend=fe), frontend=fe))


@pytest.mark.parametrize("variant", [SPLIT, FUSED, HYBRID])
def test_frontend_all_switches_chunked_variants(variant):
    """All three switches, beta from its logit included (FlashInfer PR #4262 "Dispatch
    contract" lists beta_is_logit with the norm and gate switches on the fast path)."""
    inp, A_log, dt = make_frontend_inputs([300, 0, 129, 64, 1, 77], 3, seed=805 + variant,
                                          with_h0=True, with_ckpt=True)
    fe = fe_dict(A_log, dt)
    assert_parity(compare(inp, run_gpu(inp, variant=variant, frontend=fe), frontend=fe))


@pytest.mark.parametrize("variant", [SPLIT, HYBRID])
def test_frontend_beta_logit_only_long(variant):
    """Beta from logits alone over a multi-chunk sequence, g and q/k as given."""
    inp, A_log, dt = make_frontend_inputs([1100, 700], 3, seed=809, with_h0=True)
    inp.g = -5.0 * torch.sigmoid(inp.g.float())
    unit = lambda x: (x.float() / x.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
    inp.q, inp.k = unit(inp.q), unit(inp.k)
    fe = fe_dict(A_log, dt, flags=4)
    assert_parity(compare(inp, run_gpu(inp, variant=variant, frontend=fe), frontend=fe))


@pytest.mark.parametrize("flags", [1, 2])
def test_frontend_single_switches_split(flags):
    inp, A_log, dt = make_frontend_inputs([200, 70], 2, seed=810 + flags, with_h0=True)
    if not flags & 2:
        inp.g = -5.0 * torch.sigmoid(inp.g.float())          # an FP32 log-decay in [-5, 0]
    if not flags & 4:
        inp.beta = torch.sigmoid(inp.beta.float()).to(torch.bfloat16)
    if not flags & 1:
        unit = lambda x: (x.float() / x.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        inp.q, inp.k = unit(inp.q), unit(inp.k)
    fe = fe_dict(A_log, dt, flags=flags, lower_bound=-3.0)
    assert_parity(compare(inp, run_gpu(inp, variant=SPLIT, frontend=fe), frontend=fe))


def test_frontend_hybrid_equals_split_bitwise():
    inp, A_log, dt = chunked_inputs([4100, 64, 2000], 3, seed=820, with_h0=True)
    fe = fe_dict(A_log, dt, flags=3)
    a = run_gpu(inp, variant=HYBRID, frontend=fe)
    b = run_gpu(inp, variant=SPLIT, frontend=fe)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["ht"], b["ht"])
    assert_parity(compare(inp, a, frontend=fe))


def test_frontend_full_length_sampled():
    inp, A_log, dt = chunked_inputs([8192], 12, seed=830, fixed_layout=True)
    fe = fe_dict(A_log, dt, flags=3)
    res = run_gpu(inp, frontend=fe)   # the table's choice (fused for 12 chains)
    assert_parity(compare(inp, res, seqs=[0], heads=[0, 6, 11], frontend=fe))
