"""Edge inputs of the method for the parity and precision tests: whole chunks at the
ends of the gate range [-5, 0] (lmdeploy PR #5050 "Motivation"), beta at 0 or 1, and a
large initial state.  Built from the seeded generator's inputs by overwriting tensors;
no arithmetic of the method is here."""
import torch

from kda_chunked_recurrent_b200.inputs import make_inputs

# 3 whole chunks + a 37-token tail, and 2 whole chunks + 22; two heads
LENS = [64 * 3 + 37, 150]
CKPT = [101, 64]   # inside a chunk; on a chunk boundary
CASES = ["g0", "g_minus5", "g_alternating", "beta0", "beta1", "beta1_g0", "large_state"]


def edge_inputs(case: str, seed: int = None):
    """The named edge case over LENS with h0 ~ N(0, 0.1) and checkpoints at CKPT."""
    if seed is None:
        seed = 500 + CASES.index(case)
    inp = make_inputs(LENS, 2, seed=seed, with_h0=True)
    inp.ckpt_offsets = torch.tensor(CKPT, dtype=torch.int32)
    T = inp.total_tokens
    if case == "g0":
        inp.g = torch.zeros_like(inp.g)
    elif case == "g_minus5":
        inp.g = torch.full_like(inp.g, -5.0)
    elif case == "g_alternating":
        # per sequence, 16-token blocks alternate -5 / 0, starting with -5
        g = torch.zeros_like(inp.g)
        start = 0
        for L in LENS:
            t = torch.arange(L)
            g[start:start + L][((t // 16) % 2) == 0] = -5.0
            start += L
        inp.g = g
    elif case == "beta0":
        inp.beta = torch.zeros_like(inp.beta)
    elif case == "beta1":
        inp.beta = torch.ones_like(inp.beta)
    elif case == "beta1_g0":
        inp.beta = torch.ones_like(inp.beta)
        inp.g = torch.zeros_like(inp.g)
    elif case == "large_state":
        gen = torch.Generator().manual_seed(seed + 99)
        inp.h0 = 10.0 * torch.randn(inp.h0.shape, generator=gen)
        inp.v = (2.0 * torch.randn(T, inp.num_heads, 128, generator=gen)).to(torch.bfloat16)
    else:
        raise ValueError(case)
    return inp
