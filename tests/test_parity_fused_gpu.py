"""The fused launch (recurrence CTAs fed by prepare CTAs of the same cooperative
launch through per-record ready flags) vs the FP64 oracle, and the variant
choice of the measured table (needs a B200)."""
import numpy as np
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs, workload
from tests.gpu_helpers import assert_parity, compare, run_gpu, to_dev

pytestmark = pytest.mark.gpu

FUSED = 2
SPLIT = 1


def test_fused_b1_t64_h1_full():
    inp = workload("B1_T64_H1")
    assert_parity(compare(inp, run_gpu(inp, variant=FUSED)))


@pytest.mark.parametrize("T", [1, 17, 64, 65, 200, 1000])
def test_fused_short_and_ragged_tail_lengths(T):
    inp = make_inputs([T], 3, seed=300 + T, with_h0=(T % 2 == 1), fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=FUSED)))


def test_fused_packed_ragged_with_empty_sequences():
    lens = [70, 0, 129, 5, 64, 1, 0, 300, 191]
    inp = make_inputs(lens, 3, seed=311, with_h0=True)
    res = run_gpu(inp, variant=FUSED)
    assert_parity(compare(inp, res))
    h0 = inp.h0.numpy()
    for n, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(res["ht"].numpy()[n], h0[n])


def test_fused_checkpoints_at_edges_and_inside_chunks():
    lens = [200, 64, 65, 1, 130, 128, 7]
    inp = make_inputs(lens, 2, seed=312, with_h0=True)
    inp.ckpt_offsets = torch.tensor([0, 64, 1, 1, 129, 64, 7], dtype=torch.int32)
    res = run_gpu(inp, variant=FUSED)
    assert_parity(compare(inp, res))
    assert np.array_equal(res["ckpt"].numpy()[0], inp.h0.numpy()[0])


def test_fused_equals_split_bitwise():
    # the two variants run the same arithmetic on the same records
    inp = make_inputs([700, 333, 64], 4, seed=313, with_h0=True)
    a = run_gpu(inp, variant=FUSED)
    b = run_gpu(inp, variant=SPLIT)
    assert torch.equal(a["o"], b["o"])
    assert torch.equal(a["ht"], b["ht"])


def test_fused_rerun_reuses_workspace():
    # the ready flags are cleared by every call: a second call on the same
    # workspace with other inputs must wait for its own records
    import kda_chunked_recurrent_b200 as K
    inp1 = make_inputs([500], 4, seed=314, fixed_layout=True)
    inp2 = make_inputs([500], 4, seed=315, fixed_layout=True)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 500, 4), False))
    run_gpu(inp1, variant=FUSED, workspace=ws)
    res = run_gpu(inp2, variant=FUSED, workspace=ws)
    assert ws.status() == 0
    assert_parity(compare(inp2, res))


def test_fused_forced_timeout_reports_status_and_context_survives():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([300], 2, seed=316, fixed_layout=True)
    d = to_dev(inp)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 300, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, workspace=ws,
              variant=FUSED, flags=K.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert ws.status() == K.capi.KDA_ERR_TIMEOUT
    assert_parity(compare(inp, run_gpu(inp, variant=FUSED)))


@pytest.mark.parametrize("name", ["B1_T512_H12", "B1_T8192_H12"])
def test_fused_full_size_sampled(name):
    inp = workload(name)
    res = run_gpu(inp, variant=FUSED)
    m = compare(inp, res, seqs=[0], heads=[0, inp.num_heads // 2, inp.num_heads - 1])
    assert_parity(m)


HYBRID = 3


@pytest.mark.parametrize("lens,H", [([700, 333, 64], 4), ([4100, 64, 2000, 1], 3)])
def test_hybrid_equals_split_bitwise(lens, H):
    inp = make_inputs(lens, H, seed=320 + H, with_h0=True)
    a = run_gpu(inp, variant=HYBRID)
    b = run_gpu(inp, variant=SPLIT)
    assert torch.equal(a["o"], b["o"])
    assert torch.equal(a["ht"], b["ht"])
    assert_parity(compare(inp, a))


def test_hybrid_checkpoints_and_fixed_layout():
    inp = make_inputs([2500] * 3, 4, seed=330, with_h0=True, with_ckpt=True, fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=HYBRID)))


def test_hybrid_forced_timeout_reports_status_and_context_survives():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([3000], 2, seed=331, fixed_layout=True)
    d = to_dev(inp)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 3000, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, workspace=ws,
              variant=HYBRID, flags=K.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert ws.status() == K.capi.KDA_ERR_TIMEOUT
    assert_parity(compare(inp, run_gpu(inp, variant=HYBRID)))
