"""The stream launch (one CTA per SM; on up to one SM per chain, half the CTA carries a
recurrence with the state's key channel on the tensor-memory lanes, beside a prepare
group in the other half) vs the FP64 oracle (needs a B200)."""
import numpy as np
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_frontend_inputs, make_inputs, workload
from tests.gpu_helpers import assert_parity, compare, run_gpu, to_dev

pytestmark = pytest.mark.gpu

STREAM = 5
SPLIT = 1


def test_stream_b1_t64_h1_full():
    inp = workload("B1_T64_H1")
    assert_parity(compare(inp, run_gpu(inp, variant=STREAM)))


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 127, 129, 200, 1000])
def test_stream_short_and_ragged_tail_lengths(T):
    inp = make_inputs([T], 3, seed=600 + T, with_h0=(T % 2 == 1), fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=STREAM)))


def test_stream_several_chunks_fixed_layout_batch():
    inp = make_inputs([333] * 3, 3, seed=607, fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=STREAM)))


def test_stream_packed_ragged_with_empty_sequences():
    lens = [70, 0, 129, 5, 64, 1, 0, 300, 191]
    inp = make_inputs(lens, 3, seed=611, with_h0=True)
    res = run_gpu(inp, variant=STREAM)
    assert_parity(compare(inp, res))
    h0 = inp.h0.numpy()
    for n, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(res["ht"].numpy()[n], h0[n])


def test_stream_checkpoints_at_edges_and_inside_chunks():
    lens = [200, 64, 65, 1, 130, 128, 7]
    inp = make_inputs(lens, 2, seed=612, with_h0=True)
    inp.ckpt_offsets = torch.tensor([0, 64, 1, 1, 129, 64, 7], dtype=torch.int32)
    res = run_gpu(inp, variant=STREAM)
    assert_parity(compare(inp, res))
    assert np.array_equal(res["ckpt"].numpy()[0], inp.h0.numpy()[0])


def test_stream_random_checkpoints_fixed_layout():
    inp = make_inputs([777] * 2, 2, seed=613, with_h0=True, with_ckpt=True, fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=STREAM)))


def test_stream_inplace_state_matches_separate_buffers():
    inp = make_inputs([150, 90], 2, seed=614, with_h0=True)
    a = run_gpu(inp, variant=STREAM)
    b = run_gpu(inp, variant=STREAM, inplace=True)
    assert torch.equal(a["ht"], b["ht"])
    assert torch.equal(a["o"], b["o"])
    assert_parity(compare(inp, b))


def test_stream_rerun_is_bitwise_deterministic_and_reuses_workspace():
    # the ready flags are cleared by every call: a second call on the same workspace
    # with other inputs waits for its own records
    import kda_chunked_recurrent_b200 as K
    inp1 = make_inputs([513, 77], 3, seed=615, with_h0=True, with_ckpt=True)
    inp2 = make_inputs([513, 77], 3, seed=616, with_h0=True, with_ckpt=True)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(2, 590, 3, 513), True))
    a = run_gpu(inp1, variant=STREAM, workspace=ws)
    b = run_gpu(inp2, variant=STREAM, workspace=ws)
    c = run_gpu(inp1, variant=STREAM, workspace=ws)
    assert ws.status() == 0
    assert torch.equal(a["o"], c["o"]) and torch.equal(a["ht"], c["ht"])
    assert torch.equal(a["ckpt"], c["ckpt"])
    assert_parity(compare(inp2, b))


def test_stream_outputs_outside_their_rows_are_untouched():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([100, 37], 2, seed=617, with_h0=True)
    d = to_dev(inp)
    T, H = inp.total_tokens, inp.num_heads
    big = torch.full((T + 64, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[32:32 + T]
    sbig = torch.full((2 + 2, H, 128, 128), 3.0, dtype=torch.float32, device="cuda")
    ht = sbig[1:3]
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
              cu_seqlens=d["cu_seqlens"], out=out, ht=ht, variant=STREAM)
    torch.cuda.synchronize()
    assert torch.all(big[:32] == 7.0) and torch.all(big[32 + T:] == 7.0)
    assert torch.all(sbig[0] == 3.0) and torch.all(sbig[3] == 3.0)


def test_stream_forced_timeout_reports_status_and_context_survives():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([300], 2, seed=618, fixed_layout=True)
    d = to_dev(inp)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 300, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, workspace=ws,
              variant=STREAM, flags=K.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert ws.status() == K.capi.KDA_ERR_TIMEOUT
    assert_parity(compare(inp, run_gpu(inp, variant=STREAM)))


def test_stream_validate_mode_rejects_bad_cu_seqlens_without_writing():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([100, 50], 2, seed=619)
    d = to_dev(inp)
    bad = torch.tensor([0, 120, 149], dtype=torch.int32, device="cuda")
    out = torch.full((150, 2, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(2, 150, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu_seqlens=bad, out=out,
              workspace=ws, flags=K.KDA_FLAG_VALIDATE, variant=STREAM)
    assert ws.status() == K.capi.KDA_ERR_BAD_CU_SEQLENS
    assert torch.all(out == 5.0)


def test_stream_frontend_all_switches():
    fe_inp, A_log, dt = make_frontend_inputs([300, 0, 129, 64, 1, 77], 3, seed=620,
                                             with_h0=True, with_ckpt=True)
    fe = {"flags": 7, "lower_bound": -5.0, "l2_eps": 1e-6, "A_log": A_log, "dt_bias": dt}
    assert_parity(compare(fe_inp, run_gpu(fe_inp, variant=STREAM, frontend=fe), frontend=fe))


def test_stream_many_chains_one_per_sm():
    # 144 chains: nearly every SM carries a recurrence beside one prepare group
    inp = make_inputs([130, 70] * 9, 8, seed=621, with_h0=True)
    res = run_gpu(inp, variant=STREAM)
    assert_parity(compare(inp, res, seqs=[0, 9, 17]))


def test_stream_more_chains_than_sms_is_refused():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([64] * 20, 8, seed=622)                  # 160 chains
    with pytest.raises(K.KDAError) as e:
        run_gpu(inp, variant=STREAM)
    assert e.value.code == K.capi.KDA_ERR_BAD_OPTION


@pytest.mark.parametrize("name", ["B1_T8192_H12", "B8_T8192_H12", "B4_T8192_H12_h0_ckpt",
                                  "B6_T8192_H12", "packed_1024x8_H12_h0"])
def test_stream_full_size_workloads_sampled(name):
    inp = workload(name)
    res = run_gpu(inp, variant=STREAM)
    N, H = inp.num_seqs, inp.num_heads
    seqs = sorted({0, N - 1, N // 2})
    heads = sorted({0, H - 1})
    assert_parity(compare(inp, res, seqs=seqs, heads=heads))
    assert torch.isfinite(res["o"]).all()
