"""CUDA path vs the FP64 oracle, element by element, through the C ABI (needs a B200)."""
import numpy as np
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs, workload, WORKLOADS
from tests.gpu_helpers import assert_parity, compare, run_gpu, to_dev

pytestmark = pytest.mark.gpu


def test_b1_t64_h1_full():
    inp = workload("B1_T64_H1")
    res = run_gpu(inp)
    m = compare(inp, res)
    assert_parity(m)


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 127, 129, 200])
def test_short_and_ragged_tail_lengths(T):
    inp = make_inputs([T], 2, seed=100 + T, with_h0=(T % 2 == 1), fixed_layout=True)
    res = run_gpu(inp)
    assert_parity(compare(inp, res))


def test_several_chunks_fixed_layout_batch():
    inp = make_inputs([333] * 3, 3, seed=7, fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp)))


def test_packed_ragged_with_empty_sequences():
    lens = [70, 0, 129, 5, 64, 1, 0, 300, 191]
    inp = make_inputs(lens, 3, seed=11, with_h0=True)
    res = run_gpu(inp)
    m = compare(inp, res)
    assert_parity(m)
    # zero-length sequences keep h0 exactly
    h0 = inp.h0.numpy()
    for n, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(res["ht"].numpy()[n], h0[n])


def test_checkpoints_at_edges_and_inside_chunks():
    lens = [200, 64, 65, 1, 130, 128, 7]
    inp = make_inputs(lens, 2, seed=12, with_h0=True)
    inp.ckpt_offsets = torch.tensor([0, 64, 1, 1, 129, 64, 7], dtype=torch.int32)
    res = run_gpu(inp)
    m = compare(inp, res)
    assert_parity(m)
    # offset 0 exports h0 exactly
    assert np.array_equal(res["ckpt"].numpy()[0], inp.h0.numpy()[0])


def test_random_checkpoints_fixed_layout():
    inp = make_inputs([777] * 2, 2, seed=13, with_h0=True, with_ckpt=True, fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp)))


def test_inplace_state_matches_separate_buffers():
    inp = make_inputs([150, 90], 2, seed=14, with_h0=True)
    a = run_gpu(inp)
    b = run_gpu(inp, inplace=True)
    assert torch.equal(a["ht"], b["ht"])
    assert torch.equal(a["o"], b["o"])
    assert_parity(compare(inp, b))


def test_prefix_then_suffix_equals_one_call():
    import kda_chunked_recurrent_b200 as K
    L, p = 300, 131
    inp = make_inputs([L], 2, seed=15, with_h0=True, fixed_layout=True)
    d = to_dev(inp)
    full_o, full_ht, ck = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale,
                                    h0=d["h0"], ckpt_offsets=torch.tensor([p], dtype=torch.int32,
                                                                          device="cuda"))
    sl = slice(p, L)
    suf_o, suf_ht, _ = K.prefill(d["q"][sl].contiguous(), d["k"][sl].contiguous(),
                                 d["v"][sl].contiguous(), d["g"][sl].contiguous(),
                                 d["beta"][sl].contiguous(), inp.scale, h0=ck)
    torch.cuda.synchronize()
    assert (suf_o.float() - full_o[sl].float()).abs().max().item() <= 2e-2
    rel = ((suf_ht - full_ht).norm() / full_ht.norm()).item()
    assert rel <= 1e-3


def test_rerun_is_bitwise_deterministic():
    inp = make_inputs([513, 77], 3, seed=16, with_h0=True, with_ckpt=True)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["ht"], b["ht"])
    assert torch.equal(a["ckpt"], b["ckpt"])


def test_zero_tokens_returns_h0():
    import kda_chunked_recurrent_b200 as K
    H = 2
    h0 = torch.randn(3, H, 128, 128, device="cuda")
    e16 = torch.empty(0, H, 128, dtype=torch.bfloat16, device="cuda")
    g = torch.empty(0, H, 128, dtype=torch.float32, device="cuda")
    beta = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    out, ht, _ = K.prefill(e16, e16.clone(), e16.clone(), g, beta, 0.1, h0=h0, cu_seqlens=cu)
    torch.cuda.synchronize()
    assert torch.equal(ht, h0)


def test_outputs_outside_their_rows_are_untouched():
    """Canary: output rows and states of the call are written, nothing beyond them."""
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([100, 37], 2, seed=17, with_h0=True)
    d = to_dev(inp)
    T, H = inp.total_tokens, inp.num_heads
    big = torch.full((T + 64, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    out = big[32:32 + T]
    sbig = torch.full((2 + 2, H, 128, 128), 3.0, dtype=torch.float32, device="cuda")
    ht = sbig[1:3]
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
              cu_seqlens=d["cu_seqlens"], out=out, ht=ht)
    torch.cuda.synchronize()
    assert torch.all(big[:32] == 7.0) and torch.all(big[32 + T:] == 7.0)
    assert torch.all(sbig[0] == 3.0) and torch.all(sbig[3] == 3.0)


def test_forced_timeout_reports_status_and_context_survives():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([200], 2, seed=18, fixed_layout=True)
    d = to_dev(inp)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 200, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, workspace=ws,
              flags=K.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert ws.status() == K.capi.KDA_ERR_TIMEOUT
    assert ws.status() == 0  # cleared by the previous read
    res = run_gpu(inp)
    assert_parity(compare(inp, res))


def test_validate_mode_rejects_bad_cu_seqlens_without_writing():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([100, 50], 2, seed=19)
    d = to_dev(inp)
    bad = torch.tensor([0, 120, 149], dtype=torch.int32, device="cuda")  # last != T
    out = torch.full((150, 2, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(2, 150, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu_seqlens=bad, out=out,
              workspace=ws, flags=K.KDA_FLAG_VALIDATE)
    assert ws.status() == K.capi.KDA_ERR_BAD_CU_SEQLENS
    assert torch.all(out == 5.0)
    # valid metadata in validate mode computes normally
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu_seqlens=d["cu_seqlens"],
              workspace=ws, flags=K.KDA_FLAG_VALIDATE)
    assert ws.status() == 0


# ---- the benchmark shapes at full size; oracle on sampled (sequence, head) pairs ----
FULL = [n for n in WORKLOADS if n != "B1_T64_H1"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads_sampled(name):
    inp = workload(name)
    res = run_gpu(inp)
    N, H = inp.num_seqs, inp.num_heads
    seqs = sorted({0, N - 1, N // 2})
    heads = sorted({0, H - 1})
    m = compare(inp, res, seqs=seqs, heads=heads)
    assert_parity(m)
    assert torch.isfinite(res["o"]).all()
