"""The per-token kernel vs the FP64 oracle (needs a B200): the token variant of
kda_prefill on short and ragged sequences, and kda_decode over a state pool
(single-token decode, draft verification with per-token states, padding rows,
read-only pool, CUDA-graph capture)."""
import numpy as np
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import (make_decode_frontend_inputs, make_decode_inputs,
                                               make_inputs, workload)
from tests.gpu_helpers import (O_TOL, S_TOL, assert_parity, compare, decode_oracle, rel_fro,
                               run_gpu, to_dev)

pytestmark = pytest.mark.gpu

TOKEN = 4
SPLIT = 1


def test_token_b1_t64_h1():
    inp = workload("B1_T64_H1")
    assert_parity(compare(inp, run_gpu(inp, variant=TOKEN)))


@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 31, 33, 64, 100])
def test_token_lengths_around_the_staging_block(T):
    inp = make_inputs([T], 3, seed=500 + T, with_h0=(T % 2 == 0), fixed_layout=True)
    assert_parity(compare(inp, run_gpu(inp, variant=TOKEN)))


def test_token_packed_ragged_with_empty_sequences_and_checkpoints():
    lens = [7, 0, 33, 1, 16, 0, 64, 50]
    inp = make_inputs(lens, 3, seed=511, with_h0=True)
    inp.ckpt_offsets = torch.tensor([0, 0, 33, 1, 5, 0, 64, 17], dtype=torch.int32)
    res = run_gpu(inp, variant=TOKEN)
    assert_parity(compare(inp, res))
    h0 = inp.h0.numpy()
    for n, L in enumerate(lens):
        if L == 0:
            assert np.array_equal(res["ht"].numpy()[n], h0[n])
    assert np.array_equal(res["ckpt"].numpy()[0], h0[0])   # offset 0 exports h0


def test_token_in_place_state_update():
    inp = make_inputs([40, 9, 70], 2, seed=512, with_h0=True)
    a = run_gpu(inp, variant=TOKEN)
    b = run_gpu(inp, variant=TOKEN, inplace=True)
    assert torch.equal(a["o"], b["o"]) and torch.equal(a["ht"], b["ht"])


def test_token_int64_cu_seqlens_and_validate():
    import kda_chunked_recurrent_b200 as K
    lens = [30, 0, 64, 5]
    inp = make_inputs(lens, 2, seed=513, with_h0=True)
    d = to_dev(inp)
    o32, h32, _ = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
                            cu_seqlens=d["cu_seqlens"], variant=TOKEN)
    o64, h64, _ = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
                            cu_seqlens=d["cu_seqlens"].to(torch.int64), variant=TOKEN,
                            flags=K.KDA_FLAG_VALIDATE)
    torch.cuda.synchronize()
    assert torch.equal(o32, o64) and torch.equal(h32, h64)
    bad = torch.tensor([0, 40, 30, 99, 99], dtype=torch.int32, device="cuda")   # decreasing
    out = torch.full_like(o32, 3.0)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(4, 99, 2), False,
                                                       {"variant": TOKEN}))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu_seqlens=bad, out=out,
              workspace=ws, variant=TOKEN, flags=K.KDA_FLAG_VALIDATE)
    assert ws.status() == K.capi.KDA_ERR_BAD_CU_SEQLENS
    assert torch.all(out == 3.0)


def test_token_forced_timeout_reports_status_and_context_survives():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([50], 2, seed=514, fixed_layout=True)
    d = to_dev(inp)
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(1, 50, 2), False,
                                                       {"variant": TOKEN}))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, workspace=ws,
              variant=TOKEN, flags=K.KDA_FLAG_TEST_FORCE_TIMEOUT)
    assert ws.status() == K.capi.KDA_ERR_TIMEOUT
    assert_parity(compare(inp, run_gpu(inp, variant=TOKEN)))


def test_token_matches_chunked_within_tolerance_and_auto_picks_it():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([16] * 6, 4, seed=515, with_h0=True, fixed_layout=True)
    a = run_gpu(inp, variant=TOKEN)
    b = run_gpu(inp, variant=SPLIT)
    assert float((a["o"] - b["o"]).abs().max()) <= O_TOL
    assert float(rel_fro(a["ht"].numpy(), b["ht"].numpy()).max()) <= S_TOL
    auto = run_gpu(inp)   # every sequence within the table's token bound
    assert torch.equal(auto["o"], a["o"]) and torch.equal(auto["ht"], a["ht"])
    d = K.capi.kda_prefill_describe(K.capi.make_shape(6, 96, 4, 16), False)
    assert "variant=token" in d, d


def test_token_sampled_at_b32_t512():
    inp = workload("B32_T512_H12")
    res = run_gpu(inp, variant=TOKEN)
    assert_parity(compare(inp, res, seqs=[0, 31], heads=[0, 11]))


# ---------------------------------------------------------------- kda_decode

def _decode(K, d, **kw):
    dev = lambda t: None if t is None else t.cuda()
    pool = d.pool.cuda()
    out, steps = K.decode(dev(d.q), dev(d.k), dev(d.v), dev(d.g), dev(d.beta), d.scale, pool,
                          state_indices=dev(d.state_indices), **kw)
    torch.cuda.synchronize()
    return out.float().cpu(), pool.cpu(), None if steps is None else steps.cpu()


def _check_decode(d, out, pool, steps=None, keep=False, frontend=None):
    ref = decode_oracle(d, steps=steps is not None, frontend=frontend)
    N = d.q.shape[0]
    idx = list(range(N)) if d.state_indices is None else d.state_indices.tolist()
    live = ref["live"]
    if live:
        assert float(np.abs(out.double().numpy()[live] - ref["o"]).max()) <= O_TOL
        slots = [idx[n] for n in live]
        if keep:
            assert torch.equal(pool, d.pool)
        else:
            assert float(rel_fro(pool.numpy()[slots], ref["ht"]).max()) <= S_TOL
        if steps is not None:
            st = steps.double().numpy()[live]
            for t in range(st.shape[1]):
                assert float(rel_fro(st[:, t], ref["steps"][:, t]).max()) <= S_TOL
    dead = [n for n in range(N) if n not in live]
    for n in dead:
        assert torch.all(out[n] == 0)
    untouched = sorted(set(range(d.pool.shape[0])) - {idx[n] for n in live})
    assert torch.equal(pool[untouched], d.pool[untouched])


@pytest.mark.parametrize("N,H,P", [(1, 1, 1), (7, 3, 20), (64, 12, 64)])
def test_decode_single_token(N, H, P):
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(N, 1, H, P, seed=520 + N, indices=(P > N))
    out, pool, _ = _decode(K, d)
    _check_decode(d, out, pool)


@pytest.mark.parametrize("shape_flag", [2, 4])   # KDA_DECODE_NARROW, KDA_DECODE_WIDE
@pytest.mark.parametrize("N,T,H,P", [(5, 1, 3, 11), (3, 5, 2, 3), (40, 2, 4, 64)])
def test_decode_both_kernel_shapes(shape_flag, N, T, H, P):
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(N, T, H, P, seed=600 + N + T + shape_flag, pad_every=4)
    out, pool, steps = _decode(K, d, return_step_states=True, flags=shape_flag)
    _check_decode(d, out, pool, steps=steps)


def test_decode_shapes_agree_closely():
    # both shapes run the same FP32 recurrence; only the order of the row sums
    # differs (the narrow shape splits them over two accumulators)
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(9, 3, 4, 9, seed=610)
    a = _decode(K, d, flags=K.KDA_DECODE_NARROW)
    b = _decode(K, d, flags=K.KDA_DECODE_WIDE)
    assert float((a[0] - b[0]).abs().max()) <= 2e-3          # a BF16 rounding step at most
    assert float(rel_fro(a[1].numpy(), b[1].numpy()).max()) <= 1e-5


def test_decode_padding_rows_and_permuted_slots():
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(10, 1, 4, 16, seed=531, pad_every=3)
    out, pool, _ = _decode(K, d)
    _check_decode(d, out, pool)


@pytest.mark.parametrize("T", [2, 4, 17])
def test_verify_exports_every_step_and_keeps_the_pool(T):
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(6, T, 3, 9, seed=540 + T, pad_every=4)
    out, pool, steps = _decode(K, d, return_step_states=True, keep_state=True)
    _check_decode(d, out, pool, steps=steps, keep=True)


def test_decode_bad_slot_recorded_and_skipped():
    import kda_chunked_recurrent_b200 as K
    d = make_decode_inputs(4, 1, 2, 6, seed=550)
    d.state_indices[2] = 6   # == pool size
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dev = lambda t: t.cuda()
    pool = d.pool.cuda()
    out, _ = K.decode(dev(d.q), dev(d.k), dev(d.v), dev(d.g), dev(d.beta), d.scale, pool,
                      state_indices=dev(d.state_indices), device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == K.capi.KDA_ERR_BAD_STATE_INDEX
    _check_decode(d, out.float().cpu(), pool.cpu())


def test_decode_steps_chain_equals_one_prefill_bitwise():
    """T single-token decode calls on one slot give exactly the token variant's
    prefill of the same T tokens (same kernel arithmetic, state kept in FP32)."""
    import kda_chunked_recurrent_b200 as K
    T, H = 9, 2
    inp = make_inputs([T], H, seed=560, with_h0=True, fixed_layout=True)
    d = to_dev(inp)
    o_ref, h_ref, _ = K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
                                variant=TOKEN)
    pool = d["h0"].clone()
    outs = []
    for t in range(T):
        sl = lambda x: x[t:t + 1].unsqueeze(0).contiguous()
        o, _ = K.decode(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]),
                        inp.scale, pool)
        outs.append(o[0])
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(outs, 0), o_ref)
    assert torch.equal(pool, h_ref)


def test_decode_cuda_graph_replays():
    import kda_chunked_recurrent_b200 as K
    a = make_decode_inputs(8, 1, 4, 12, seed=570)
    b = make_decode_inputs(8, 1, 4, 12, seed=571)
    st = {n: getattr(a, n).cuda() for n in ("q", "k", "v", "g", "beta", "state_indices")}
    pool = a.pool.cuda()
    out = torch.empty(8, 1, 4, 128, dtype=torch.bfloat16, device="cuda")
    run = lambda: K.decode(st["q"], st["k"], st["v"], st["g"], st["beta"], a.scale, pool,
                           state_indices=st["state_indices"], out=out)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for n in ("q", "k", "v", "g", "beta", "state_indices"):
        st[n].copy_(getattr(b, n))
    pool.copy_(b.pool)
    g.replay()
    torch.cuda.synchronize()
    _check_decode(b, out.float().cpu(), pool.cpu())


# ------------------------------------------------------ kda_decode input front end
# The oracle's switch values equal the library's KDA_FE_* values (1, 2, 4).

@pytest.mark.parametrize("shape_flag", [2, 4])   # KDA_DECODE_NARROW, KDA_DECODE_WIDE
@pytest.mark.parametrize("fe_flags", [7, 1, 2, 4])
def test_decode_frontend_matches_oracle(shape_flag, fe_flags):
    import kda_chunked_recurrent_b200 as K
    d, A_log, dt_bias = make_decode_frontend_inputs(6, 3, 3, 9, seed=700 + fe_flags, pad_every=5)
    if not fe_flags & 2:
        # without the gate switch g is an FP32 log-decay in [-5, 0]
        d.g = -5.0 * torch.sigmoid(d.g.float())
    if not fe_flags & 4:
        d.beta = torch.sigmoid(d.beta.float()).to(torch.bfloat16)
    if not fe_flags & 1:
        # without the norm switch q and k are given unit rows (the delta rule needs them)
        unit = lambda x: (x.float() / x.float().norm(dim=-1, keepdim=True)).to(torch.bfloat16)
        d.q, d.k = unit(d.q), unit(d.k)
    fe = {"flags": fe_flags, "lower_bound": -4.0, "l2_eps": 1e-6, "A_log": A_log,
          "dt_bias": dt_bias}
    dev_fe = dict(fe, A_log=A_log.cuda(), dt_bias=dt_bias.cuda())
    out, pool, steps = _decode(K, d, return_step_states=True, flags=shape_flag, frontend=dev_fe)
    _check_decode(d, out, pool, steps=steps, frontend=fe)


def test_decode_frontend_zero_rows_and_bounds():
    # a zero q row stays finite (eps), lower_bound -5 and a steep gate rate
    import kda_chunked_recurrent_b200 as K
    d, A_log, dt_bias = make_decode_frontend_inputs(4, 2, 2, 4, seed=720)
    d.q[1, 0, 1] = 0
    A_log[0] = 3.0
    fe = {"flags": 7, "lower_bound": -5.0, "l2_eps": 1e-6, "A_log": A_log, "dt_bias": dt_bias}
    out, pool, _ = _decode(K, d, frontend=dict(fe, A_log=A_log.cuda(), dt_bias=dt_bias.cuda()))
    assert torch.isfinite(out).all() and torch.isfinite(pool).all()
    _check_decode(d, out, pool, frontend=fe)
