"""Prepare CTAs that walk more than one batch of item lookups (each 256-thread group looks
its items' chunk spans up 64 at a time into shared memory and refills the batch every 64
items) vs the FP64 oracle on sampled (sequence, head) pairs (needs a B200)."""
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs
from tests.gpu_helpers import assert_parity, compare, run_gpu

pytestmark = pytest.mark.gpu

SPLIT, FUSED, HYBRID = 1, 2, 3


@pytest.mark.parametrize("fixed", [False, True])
def test_split_prepare_with_several_lookup_batches(fixed):
    # 16 x 8192 tokens, 12 heads: 24576 records over 296 prepare CTAs, 83 items each
    inp = make_inputs([8192] * 16, 12, seed=901, with_h0=True, fixed_layout=fixed)
    res = run_gpu(inp, variant=SPLIT)
    assert_parity(compare(inp, res, seqs=[0, 7, 15], heads=[0, 11]))
    assert torch.isfinite(res["o"]).all()


def test_hybrid_prepare_launch_with_several_lookup_batches():
    # 10 x 16384 tokens, 12 heads: the prepare launch walks about 100 items per CTA
    inp = make_inputs([16384] * 10, 12, seed=902, fixed_layout=False)
    res = run_gpu(inp, variant=HYBRID)
    assert_parity(compare(inp, res, seqs=[0, 9], heads=[0, 11]))


def test_fused_prepare_groups_with_several_lookup_batches():
    # 2 x 65536 tokens, 12 heads: 24576 records over 248 prepare groups, 99 each
    inp = make_inputs([65536] * 2, 12, seed=903, fixed_layout=True)
    res = run_gpu(inp, variant=FUSED)
    assert_parity(compare(inp, res, seqs=[0, 1], heads=[0, 11]))
