"""CUDA path vs the FP64 oracle on the method's edge inputs, for every variant.

The seeded workloads draw g = -5 sigmoid(N(0, 1)) and beta = sigmoid(N(0, 1)), which
almost never reach the ends of their ranges.  The gate bound is [-5, 0] with both
endpoints in scope (lmdeploy PR #5050 "Motivation"; FlashInfer PR #4633's review
notes two codebases disagreeing about 0), and beta lies in [0, 1].  These cases put
whole chunks at the endpoints:

  * g = 0 over several whole chunks plus a tail (no decay: Gamma = 1 and the chunked
    form reduces to the plain delta rule);
  * g = -5 over several whole chunks (16 tokens at -5 make the sub-block factor
    2^(B_i - G_s) reach e^75 before its BF16 rounding), and chunks that alternate
    16 tokens at -5 with 16 at 0;
  * beta = 0 (the state is h0 decayed by exp(sum g), a closed form the oracle pins)
    and beta = 1;
  * h0 with standard deviation 10 and v ~ N(0, 4), inside the FP16 operand range
    the header states.

Each case runs with an initial state and a checkpoint inside a chunk, element by
element against the oracle at the path's tolerances (2e-2 max-abs on o, 1e-3
relative Frobenius on the final and checkpoint states).
"""
import numpy as np
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs
from tests.edge_inputs import CASES, CKPT, LENS, edge_inputs
from tests.gpu_helpers import assert_parity, compare, run_gpu

pytestmark = pytest.mark.gpu

VARIANTS = {"split": 1, "fused": 2, "hybrid": 3, "token": 4, "stream": 5}


@pytest.mark.parametrize("variant", list(VARIANTS))
@pytest.mark.parametrize("case", CASES)
def test_edge_inputs_match_oracle(case, variant):
    inp = edge_inputs(case)
    res = run_gpu(inp, variant=VARIANTS[variant])
    m = compare(inp, res)
    assert_parity(m)
    assert torch.isfinite(res["o"]).all() and torch.isfinite(res["ht"]).all()


@pytest.mark.parametrize("variant", list(VARIANTS))
def test_beta0_state_is_decayed_h0(variant):
    """beta = 0: no token writes the state, so ht = Diag(exp(sum_t g_t)) h0 per
    (sequence, head) and the checkpoint is the same with the prefix sum.  The gate is
    scaled to 1/50 of its draw so that exp(sum g) over a whole sequence stays far from
    underflow and the closed form is a meaningful reference."""
    inp = edge_inputs("beta0", seed=520)
    inp.g = 0.02 * inp.g
    res = run_gpu(inp, variant=VARIANTS[variant])
    g = inp.g.double().numpy()
    h0 = inp.h0.double().numpy()
    cu = inp.cu_seqlens.tolist()
    for n in range(len(LENS)):
        seg = g[cu[n]:cu[n + 1]]                       # [L, H, K]
        decay = np.exp(seg.sum(axis=0))                # [H, K]
        want = decay[:, :, None] * h0[n]
        got = res["ht"][n].double().numpy()
        rel = np.linalg.norm(got - want) / np.linalg.norm(want)
        assert rel <= 1e-3, (n, rel)
        p = CKPT[n]
        want_ck = np.exp(seg[:p].sum(axis=0))[:, :, None] * h0[n]
        got_ck = res["ckpt"][n].double().numpy()
        assert np.linalg.norm(got_ck - want_ck) / np.linalg.norm(want_ck) <= 1e-3


@pytest.mark.parametrize("variant", ["split", "fused", "hybrid", "stream"])
def test_g_minus5_long_sequence(variant):
    """g = -5 for every token of a multi-chunk sequence per head, B2 T1024 H4."""
    inp = make_inputs([1024, 1024], 4, seed=530, with_h0=True, fixed_layout=True)
    inp.g = torch.full_like(inp.g, -5.0)
    res = run_gpu(inp, variant=VARIANTS[variant])
    assert_parity(compare(inp, res))
