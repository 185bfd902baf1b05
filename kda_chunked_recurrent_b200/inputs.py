"""Seeded synthetic inputs for KDA prefill.

This module only draws random tensors; it holds none of the method's
arithmetic.  Both the CUDA path's tests/benchmark and the CPU oracle are fed
from here, so the two always see bit-identical inputs.

Distributions follow the workload statements of the benchmark shapes (the
pages measure synthetic shapes only: FlashInfer PR #4633 "Performance",
FlashInfer PR #4262 "Fresh B200 CUPTI benchmark"):

* q, k ~ N(0, 1), L2-normalised per (token, head) row of 128 in FP32, then BF16
* v ~ N(0, 1), BF16
* g = -5 * sigmoid(N(0, 1)), FP32, so every log-decay lies in [-5, 0]
* beta = sigmoid(N(0, 1)), BF16, in (0, 1)
* scale = 1 / sqrt(128)
* h0 ~ N(0, 0.1) (0.1 read as the standard deviation), FP32, when requested
* ragged lengths uniform on [1, 4096] (seed 7); checkpoint offsets uniform on
  [1, len] per sequence
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import torch

DK = 128
DV = 128


@dataclass
class KDAInputs:
    q: torch.Tensor            # [T_total, H, 128] bf16
    k: torch.Tensor            # [T_total, H, 128] bf16
    v: torch.Tensor            # [T_total, H, 128] bf16
    g: torch.Tensor            # [T_total, H, 128] fp32
    beta: torch.Tensor         # [T_total, H] bf16
    scale: float
    cu_seqlens: torch.Tensor   # [N+1] int32
    h0: Optional[torch.Tensor] = None            # [N, H, 128, 128] fp32 (S[k][v])
    ckpt_offsets: Optional[torch.Tensor] = None  # [N] int32
    fixed_layout: bool = False                   # True: B x T with no cu_seqlens needed
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens.numel() - 1)

    @property
    def total_tokens(self) -> int:
        return int(self.q.shape[0])

    @property
    def num_heads(self) -> int:
        return int(self.q.shape[1])

    @property
    def seqlens(self) -> List[int]:
        c = self.cu_seqlens.tolist()
        return [c[i + 1] - c[i] for i in range(len(c) - 1)]


def make_inputs(seqlens: List[int], num_heads: int, seed: int, *, with_h0: bool = False,
                h0_std: float = 0.1, with_ckpt: bool = False, ckpt_seed: Optional[int] = None,
                fixed_layout: bool = False, dk: int = DK, dv: int = DV) -> KDAInputs:
    """Draw one packed batch on the CPU with a dedicated torch.Generator."""
    gen = torch.Generator().manual_seed(int(seed))
    T = int(sum(seqlens))
    H = int(num_heads)
    q = torch.randn(T, H, dk, generator=gen, dtype=torch.float32)
    k = torch.randn(T, H, dk, generator=gen, dtype=torch.float32)
    q = q / q.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    k = k / k.norm(dim=-1, keepdim=True).clamp_min(1e-30)
    v = torch.randn(T, H, dv, generator=gen, dtype=torch.float32)
    g = -5.0 * torch.sigmoid(torch.randn(T, H, dk, generator=gen, dtype=torch.float32))
    beta = torch.sigmoid(torch.randn(T, H, generator=gen, dtype=torch.float32))
    cu = torch.zeros(len(seqlens) + 1, dtype=torch.int32)
    if len(seqlens):
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0).to(torch.int32)
    h0 = None
    if with_h0:
        h0 = h0_std * torch.randn(len(seqlens), H, dk, dv, generator=gen, dtype=torch.float32)
    ck = None
    if with_ckpt:
        cg = torch.Generator().manual_seed(int(seed if ckpt_seed is None else ckpt_seed) + 1)
        offs = []
        for L in seqlens:
            offs.append(int(torch.randint(1, L + 1, (1,), generator=cg).item()) if L > 0 else 0)
        ck = torch.tensor(offs, dtype=torch.int32)
    return KDAInputs(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16),
                     g=g.contiguous(), beta=beta.to(torch.bfloat16), scale=1.0 / math.sqrt(dk),
                     cu_seqlens=cu, h0=h0, ckpt_offsets=ck, fixed_layout=fixed_layout,
                     meta={"seed": int(seed), "seqlens": list(map(int, seqlens))})


def ragged_lengths(n: int, lo: int = 1, hi: int = 4096, seed: int = 7) -> List[int]:
    """Sequence lengths drawn uniformly on [lo, hi] with their own generator."""
    gen = torch.Generator().manual_seed(int(seed))
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=gen).tolist()]


# The benchmark shapes (H = 12 unless stated).  Index i is seeded 1000 + i.
WORKLOADS = {
    "B1_T64_H1": dict(seqlens=[64], H=1, seed=1000, fixed=True),
    "B1_T512_H12": dict(seqlens=[512], H=12, seed=1001, fixed=True),
    "B1_T8192_H12": dict(seqlens=[8192], H=12, seed=1001, fixed=True),
    "B8_T1024_H12": dict(seqlens=[1024] * 8, H=12, seed=1002, fixed=True),
    "B32_T512_H12": dict(seqlens=[512] * 32, H=12, seed=1002, fixed=True),
    "B6_T8192_H12": dict(seqlens=[8192] * 6, H=12, seed=1002, fixed=True),
    "B8_T8192_H12": dict(seqlens=[8192] * 8, H=12, seed=1002, fixed=True),
    "packed_1024x8_H12_h0": dict(seqlens=[1024] * 8, H=12, seed=1003, h0=True),
    "ragged16_H12_h0": dict(seqlens=None, H=12, seed=1003, h0=True, ragged=16),
    "B4_T8192_H12_h0_ckpt": dict(seqlens=[8192] * 4, H=12, seed=1004, h0=True, ckpt=True,
                                 fixed=True),
}


def workload(name: str) -> KDAInputs:
    w = WORKLOADS[name]
    lens = w["seqlens"] if w.get("seqlens") is not None else ragged_lengths(w["ragged"])
    return make_inputs(lens, w["H"], w["seed"], with_h0=w.get("h0", False),
                       with_ckpt=w.get("ckpt", False), fixed_layout=w.get("fixed", False))


@dataclass
class DecodeInputs:
    """N sequences of T new tokens each over a pool of P states."""
    q: torch.Tensor              # [N, T, H, 128] bf16
    k: torch.Tensor              # [N, T, H, 128] bf16
    v: torch.Tensor              # [N, T, H, 128] bf16
    g: torch.Tensor              # [N, T, H, 128] fp32
    beta: torch.Tensor           # [N, T, H] bf16
    scale: float
    pool: torch.Tensor           # [P, H, 128, 128] fp32
    state_indices: Optional[torch.Tensor]   # [N] int32 (negative = padding) or None


def make_decode_inputs(num_seqs: int, tokens: int, num_heads: int, pool_size: int, seed: int, *,
                       indices: bool = True, pad_every: int = 0, pool_std: float = 0.1
                       ) -> DecodeInputs:
    """Token rows as in make_inputs; a pool of N(0, pool_std) states; the slots of the
    sequences a random injective map into the pool (every ``pad_every``-th entry -1)."""
    base = make_inputs([tokens] * num_seqs, num_heads, seed, fixed_layout=True)
    N, T, H = int(num_seqs), int(tokens), int(num_heads)
    gen = torch.Generator().manual_seed(int(seed) + 7)
    pool = pool_std * torch.randn(int(pool_size), H, DK, DV, generator=gen, dtype=torch.float32)
    idx = None
    if indices:
        assert pool_size >= N
        idx = torch.randperm(int(pool_size), generator=gen)[:N].to(torch.int32)
        if pad_every > 0:
            idx[::pad_every] = -1
    shp = (N, T, H)
    return DecodeInputs(q=base.q.view(*shp, DK), k=base.k.view(*shp, DK), v=base.v.view(*shp, DV),
                        g=base.g.view(*shp, DK), beta=base.beta.view(*shp), scale=base.scale,
                        pool=pool, state_indices=idx)


def make_decode_frontend_inputs(num_seqs: int, tokens: int, num_heads: int, pool_size: int,
                                seed: int, *, pad_every: int = 0):
    """Raw projections for the decode front end: q, k ~ N(0, 1) BF16 (not normalised),
    the raw gate a ~ N(0, 1) BF16 in the ``g`` field, beta logits ~ N(0, 1) BF16 in the
    ``beta`` field, A_log ~ N(0, 0.5) FP32 [H], dt_bias ~ N(0, 0.5) FP32 [H, 128].
    Returns (DecodeInputs, A_log, dt_bias)."""
    d = make_decode_inputs(num_seqs, tokens, num_heads, pool_size, seed, pad_every=pad_every)
    gen = torch.Generator().manual_seed(int(seed) + 11)
    shp = tuple(d.q.shape)
    d.q = torch.randn(*shp, generator=gen).to(torch.bfloat16)
    d.k = torch.randn(*shp, generator=gen).to(torch.bfloat16)
    d.g = torch.randn(*shp, generator=gen).to(torch.bfloat16)
    d.beta = torch.randn(*shp[:3], generator=gen).to(torch.bfloat16)
    A_log = 0.5 * torch.randn(num_heads, generator=gen)
    dt_bias = 0.5 * torch.randn(num_heads, DK, generator=gen)
    return d, A_log, dt_bias


def make_frontend_inputs(seqlens: List[int], num_heads: int, seed: int, *, with_h0: bool = False,
                         with_ckpt: bool = False, fixed_layout: bool = False):
    """Raw projections for a prefill through the input front end: the KDAInputs of
    make_inputs with q, k replaced by N(0, 1) BF16 rows (not normalised), the ``g``
    field by the raw gate ~ N(0, 1) BF16 and ``beta`` by logits ~ N(0, 1) BF16; plus
    A_log ~ N(0, 0.5) FP32 [H] and dt_bias ~ N(0, 0.5) FP32 [H, 128].
    Returns (KDAInputs, A_log, dt_bias)."""
    inp = make_inputs(seqlens, num_heads, seed, with_h0=with_h0, with_ckpt=with_ckpt,
                      fixed_layout=fixed_layout)
    gen = torch.Generator().manual_seed(int(seed) + 13)
    T, H = inp.total_tokens, inp.num_heads
    inp.q = torch.randn(T, H, DK, generator=gen).to(torch.bfloat16)
    inp.k = torch.randn(T, H, DK, generator=gen).to(torch.bfloat16)
    inp.g = torch.randn(T, H, DK, generator=gen).to(torch.bfloat16)
    inp.beta = torch.randn(T, H, generator=gen).to(torch.bfloat16)
    A_log = 0.5 * torch.randn(H, generator=gen)
    dt_bias = 0.5 * torch.randn(H, DK, generator=gen)
    return inp, A_log, dt_bias
