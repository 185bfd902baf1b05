"""INT64 cu_seqlens (narrowed on the device) and CUDA-graph capture of a warmed call
(needs a B200)."""
import pytest
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs
from tests.gpu_helpers import assert_parity, compare, to_dev

pytestmark = pytest.mark.gpu


def _call(K, d, inp, cu, variant, **kw):
    return K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, h0=d["h0"],
                     cu_seqlens=cu, max_seqlen=max(inp.seqlens), ckpt_offsets=d["ckpt_offsets"],
                     variant=variant, **kw)


@pytest.mark.parametrize("variant", [1, 2])
def test_int64_cu_seqlens_matches_int32_bitwise(variant):
    import kda_chunked_recurrent_b200 as K
    lens = [300, 0, 129, 64, 1, 700]
    inp = make_inputs(lens, 2, seed=401, with_h0=True, with_ckpt=True)
    d = to_dev(inp)
    o32, h32, c32 = _call(K, d, inp, d["cu_seqlens"], variant)
    o64, h64, c64 = _call(K, d, inp, d["cu_seqlens"].to(torch.int64), variant)
    torch.cuda.synchronize()
    assert torch.equal(o32, o64) and torch.equal(h32, h64) and torch.equal(c32, c64)
    res = {"o": o64.float().cpu(), "ht": h64.cpu(), "ckpt": c64.cpu()}
    assert_parity(compare(inp, res))


def test_int64_validate_rejects_out_of_range_offsets():
    import kda_chunked_recurrent_b200 as K
    inp = make_inputs([100, 50], 2, seed=402)
    d = to_dev(inp)
    bad = torch.tensor([0, 1 << 33, 150], dtype=torch.int64, device="cuda")
    out = torch.full((150, 2, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(K.capi.make_shape(2, 150, 2), False))
    K.prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], inp.scale, cu_seqlens=bad, out=out,
              workspace=ws, flags=K.KDA_FLAG_VALIDATE)
    assert ws.status() == K.capi.KDA_ERR_BAD_CU_SEQLENS
    assert torch.all(out == 5.0)


@pytest.mark.parametrize("variant", [1, 2, 3, 5])   # split, fused, hybrid, stream
def test_cuda_graph_capture_replays_bitwise(variant):
    """A warmed call captured into a CUDA graph replays with new inputs in the same
    buffers and gives exactly the eager results (no host reads, no allocation)."""
    import kda_chunked_recurrent_b200 as K
    lens = [640, 200, 1000]
    a = make_inputs(lens, 3, seed=403, with_h0=True)
    b = make_inputs(lens, 3, seed=404, with_h0=True)
    da, db = to_dev(a), to_dev(b)
    N, T, H = a.num_seqs, a.total_tokens, a.num_heads
    shape = K.capi.make_shape(N, T, H, max(lens))
    ws = K.Workspace(K.capi.kda_prefill_workspace_size(shape, False, {"variant": variant}))
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device="cuda")
    ht = torch.empty(N, H, 128, 128, dtype=torch.float32, device="cuda")
    # eager reference for inputs b
    ob, hb, _ = _call(K, db, b, db["cu_seqlens"], variant)
    # static buffers hold inputs a; warm up, capture, then swap in inputs b and replay
    st = {k: (v.clone() if v is not None else None) for k, v in da.items()}
    run = lambda: K.prefill(st["q"], st["k"], st["v"], st["g"], st["beta"], a.scale, h0=st["h0"],
                            cu_seqlens=st["cu_seqlens"], max_seqlen=max(lens), out=out, ht=ht,
                            workspace=ws, variant=variant)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    for k in ("q", "k", "v", "g", "beta", "h0"):
        st[k].copy_(db[k])
    g.replay()
    g.replay()   # replaying twice is idempotent (h0 and ht are distinct buffers)
    torch.cuda.synchronize()
    assert ws.status() == 0
    assert torch.equal(out, ob) and torch.equal(ht, hb)
