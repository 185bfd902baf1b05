#!/usr/bin/env python
"""Benchmark of KDA multi-token recurrent prefill on B200 (one JSON line on rank 0).

A step is one full prefill (every kernel of the path) over one batch of
synthetic inputs already resident in HBM.  Default workload: B8 T8192 H12
(K = V = 128, BF16 q/k/v/beta, FP32 g in [-5, 0], no initial state), the
shape the throughput target is stated on.  Its inputs (1.0 GB) exceed the 126 MB
L2, so no flush is needed between steps; a workload whose inputs are smaller than
twice L2 gets a 256 MB write before every step and is timed from the first to the
last kernel of each step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   # the FP64 CPU oracle on the host cores
  python bench.py --op decode [--decode N,T,H]  # kda_decode over a state pool

Multi-GPU (torchrun, one rank per GPU): every rank runs the same per-GPU
workload on its own seeded data (weak scaling, no collective on the data path);
the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KDA prefill ms and Mtokens·heads/s at 1 B200; % tensor-core roofline"
UNIT = "Mtokens·heads/s"
# bytes every prefill must move per token and head: q, k, v (3 x 256) + g (512) + beta (2) + o (256)
PATH_BYTES_PER_TOKHEAD = 1538
STATE_BYTES = 128 * 128 * 4
# per-kernel bytes per token and head, as designed (split variant)
PREP_BYTES_PER_TOKHEAD = 768 + 512 + 2 + 1160     # reads q,k,v,g,beta; writes W,QG,U,Kd,Aqk,Gamma
REC_BYTES_PER_TOKHEAD = 1160 + 256                 # reads the prepared tiles; writes o
OUT_BYTES_PER_TOKHEAD = 256                        # the o row every prefill writes
# tensor-core FLOPs per token and head at a fixed C = 64 count: 6 K V + 10 C d
FLOPS_PER_TOKHEAD_C64 = 6 * 128 * 128 + 10 * 64 * 128
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_sha(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, "kda_chunked_recurrent_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel, variant, units):
    """DRAM bytes per launch from the committed ncu summary (kernel@variant), if the
    kernel sources are unchanged since it was taken."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(p))[f"{kernel}@{variant}"]
    except Exception:
        return None
    if d.get("source_sha") != kernel_source_sha(d.get("sources", [])):
        return None
    return float(d["dram_bytes_per_tokhead"]) * units


class ClockSampler:
    """nvidia-smi clock / throttle-reason sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.thread = None
        self.t_on = self.t_off = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), [x.strip() for x in line.split(",")]))

    def mark_on(self):
        self.t_on = time.time()

    def mark_off(self):
        self.t_off = time.time()

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        inside = [s for t, s in self.samples if self.t_on and self.t_off and
                  self.t_on - 0.15 <= t <= self.t_off + 0.15]
        use = inside if inside else [s for _, s in self.samples]
        sm = [float(s[1]) for s in use if s[1].replace(".", "").isdigit()]
        mx = [float(s[2]) for s in use if s[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in use for i in range(4)
                          if len(s) > 5 + i and s[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(use), "in_window": bool(inside)}


def dist_setup(backend="nccl"):
    """Join the process group when launched with WORLD_SIZE > 1 (one rank per GPU).

    Returns (rank, world, local_rank).  The group carries only the timing barrier
    and the max-over-ranks reduction; the data path has no collective."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(base_seed, rank):
    """Every rank draws its own inputs of the same per-GPU workload (weak scaling)."""
    return base_seed + 7919 * rank


L2_BYTES = 126 * 2**20


_WL_CACHE = {}


def _oracle_sample(inp, nseq):
    """The first nseq sequences of a workload (each cut to 8192 tokens), packed."""
    import torch
    from kda_chunked_recurrent_b200.inputs import KDAInputs
    cu = inp.cu_seqlens.tolist()
    rows, lens = [], []
    for n in range(nseq):
        L = min(cu[n + 1] - cu[n], 8192)
        rows.append(torch.arange(cu[n], cu[n] + L))
        lens.append(L)
    r = torch.cat(rows)
    sub_cu = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()), dtype=torch.int32)
    return KDAInputs(q=inp.q[r], k=inp.k[r], v=inp.v[r], g=inp.g[r], beta=inp.beta[r],
                     scale=inp.scale, cu_seqlens=sub_cu,
                     h0=None if inp.h0 is None else inp.h0[:nseq]), sum(lens)


def cpu_baseline(inp_name, threads=0, max_tokens=8192, min_seconds=0.0, one_thread=False):
    """The oracle as it stands, on the host cores, on a bounded sample of the workload:
    its first sequences up to max_tokens tokens (each cut to 8192), every head, rerun
    until min_seconds have passed.  With one_thread, also one (sequence, head) unit
    on a single thread."""
    import oracle
    from kda_chunked_recurrent_b200.inputs import workload
    if inp_name not in _WL_CACHE:
        _WL_CACHE[inp_name] = workload(inp_name)
    inp = _WL_CACHE[inp_name]
    cu = inp.cu_seqlens.tolist()
    nseq, tok = 0, 0
    while nseq < inp.num_seqs and (nseq == 0 or tok + min(cu[nseq + 1] - cu[nseq], 8192) <= max_tokens):
        tok += min(cu[nseq + 1] - cu[nseq], 8192)
        nseq += 1
    sub, L = _oracle_sample(inp, nseq)
    oracle.build_oracle()
    # OpenMP runs over the (sequence, head) units of the sample, so at most that
    # many threads can be busy
    cores = min(threads if threads > 0 else (os.cpu_count() or 1), nseq * inp.num_heads)
    units = L * inp.num_heads
    reps, dt = 0, 0.0
    while reps == 0 or (dt < min_seconds and reps < 8):
        t = time.perf_counter()
        oracle.prefill(sub, threads=cores)
        dt += time.perf_counter() - t
        reps += 1
    res = {"value": units * reps / dt / 1e6, "unit": UNIT, "cores": cores, "kind": "oracle",
           "sample": f"first {nseq} sequence(s) of {inp_name}: {L} tokens x {inp.num_heads} "
                     f"heads ({units} token-heads) x {reps} run(s), FP64 per-token recurrence, "
                     f"OpenMP over (sequence, head)",
           "seconds": dt / reps}
    if one_thread:
        one, L1 = _oracle_sample(inp, 1)
        t = time.perf_counter()
        oracle.prefill(one, threads=1, heads=[0])
        res["value_1_thread"] = L1 / (time.perf_counter() - t) / 1e6
        res["sample_1_thread"] = f"sequence 0, head 0 of {inp_name}: {L1} tokens, 1 thread"
    return res


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    steps, warm = args.steps, args.warmup
    for _ in range(warm):
        cpu_baseline(args.workload)
    vals, secs = [], []
    for _ in range(steps):
        r = cpu_baseline(args.workload)
        vals.append(r["value"])
        secs.append(r["seconds"])
    value = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": steps, "warmup": warm,
            "ms_per_step": 1e3 * statistics.median(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample": r["sample"]},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": r["cores"], "kind": "oracle",
                             "sample": r["sample"]},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


TOKEN_SOURCES = ["kda_token.cu", "kda_token.cuh", "kda_common.cuh", "sm100_primitives.cuh"]


def token_kernel_name(capi, N, H):
    """Which per-token kernel the library launches for N x H units (its describe line)."""
    d = capi.kda_prefill_describe(capi.make_shape(N, N, H, 1), False, {"variant": 4})
    return "kda_token_wide_kernel" if "(wide" in d else "kda_token_narrow_kernel"


DECODE_METRIC = "KDA decode Mtokens·heads/s at 1 B200 (state pool, one launch per step)"


def run_decode(args):
    """kda_decode over a pool of N states: N sequences of T new tokens, H heads, each
    sequence on a random slot of the pool.  A step is one kda_decode call; the pool is
    updated in place (the recurrence continues from step to step)."""
    import torch
    rank, world, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    import kda_chunked_recurrent_b200 as K
    from kda_chunked_recurrent_b200 import capi
    from kda_chunked_recurrent_b200.inputs import make_decode_frontend_inputs, make_decode_inputs
    N, T, H = (int(x) for x in args.decode.split(","))
    fe_on = args.decode_frontend
    if fe_on:
        dinp, A_log, dt_bias = make_decode_frontend_inputs(N, T, H, N, rank_seed(1010, rank))
    else:
        dinp = make_decode_inputs(N, T, H, N, rank_seed(1010, rank), indices=True)
    dev = torch.device("cuda", local)
    fe = None
    if fe_on:
        A_log, dt_bias = A_log.to(dev), dt_bias.to(dev)
        fe = capi.make_frontend(7, -5.0, 1e-6, A_log.data_ptr(), dt_bias.data_ptr())
    q, k, v, g, beta, idx = (x.to(dev) for x in (dinp.q, dinp.k, dinp.v, dinp.g, dinp.beta,
                                                  dinp.state_indices))
    pool = dinp.pool.to(dev)
    out = torch.empty(N, T, H, 128, dtype=torch.bfloat16, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    shape = capi.make_decode_shape(N, T, H, N)
    stream = torch.cuda.current_stream(dev)
    Pt = lambda t: t.data_ptr()

    def step():
        rc = capi.kda_decode(Pt(q), Pt(k), Pt(v), Pt(g), Pt(beta), dinp.scale, Pt(pool), Pt(idx),
                             shape, Pt(out), None, Pt(status), 0, stream.cuda_stream, fe)
        if rc != 0:
            raise K.KDAError(rc, "kda_decode")

    units = N * T * H
    # bytes a decode step must move: the state slice read and written once, the token rows
    # (with the front end the raw gate is BF16: 256 B instead of the 512 B FP32 g)
    row_bytes = PATH_BYTES_PER_TOKHEAD - (256 if fe_on else 0)
    algo_bytes = N * H * 2 * STATE_BYTES + units * row_bytes
    flush = None
    if algo_bytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev_a = [mk() for _ in range(args.steps)]
    ev_b = [mk() for _ in range(args.steps)]
    clk = ClockSampler(local if world > 1 else int(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or 0))
    clk.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    clk.mark_on()
    t0, t1 = mk(), mk()
    t0.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        ev_a[i].record(stream)
        step()
        ev_b[i].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    clk.mark_off()
    barrier(world)
    clk.stop()
    kern_ms = statistics.mean(ev_a[i].elapsed_time(ev_b[i]) for i in range(args.steps))
    ms_local = kern_ms if flush is not None else t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms_local, world)
    if int(status.item()) != 0:
        raise K.KDAError(int(status.item()), "decode device status")
    value = units * world / (ms / 1e3) / 1e6
    peaks, peak_src = load_peaks()
    achieved = algo_bytes / (kern_ms / 1e3) / 1e9
    kname = token_kernel_name(capi, N, H).replace("_kernel", "_fe_kernel" if fe_on else "_kernel")
    roof = {"kernel": kname, "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": ncu_traffic(kname, f"decode_N{N}_T{T}_H{H}", units),
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
            else "fallback 6650 GB/s", "kernel_ms": round(kern_ms, 4),
            "algorithmic_bytes": int(algo_bytes)}

    # end to end: the step's token rows and slots from pinned host memory, o back;
    # the pool stays resident on the device as in a serving engine
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv, hg, hb, hi = (x.pin_memory() for x in (dinp.q, dinp.k, dinp.v, dinp.g,
                                                           dinp.beta, dinp.state_indices))
        ho = torch.empty(N, T, H, 128, dtype=torch.bfloat16).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg, hb, hi))

        def e2e_step():
            for dst, src in ((q, hq), (k, hk), (v, hv), (g, hg), (beta, hb), (idx, hi)):
                dst.copy_(src, non_blocking=True)
            step()
            ho.copy_(out, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize()
        barrier(world)
        a, b = mk(), mk()
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world)
        e2e = {"value": units * world / (e_ms / 1e3) / 1e6, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(ho.numel() * 2),
               "ms_per_step": round(e_ms, 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import numpy as np
        import oracle
        oracle.build_oracle()
        ns = min(N, 64)
        sel = lambda x: np.ascontiguousarray(x[:ns].double().numpy().reshape(ns * T, H, -1))
        qs, ks, vs, gs = sel(dinp.q), sel(dinp.k), sel(dinp.v), sel(dinp.g)
        bs = np.ascontiguousarray(dinp.beta[:ns].double().numpy().reshape(ns * T, H))
        h0 = np.ascontiguousarray(dinp.pool.double().numpy()[dinp.state_indices[:ns].long().numpy()])
        cu = np.arange(ns + 1, dtype=np.int64) * T
        cores = min(os.cpu_count() or 1, ns * H)
        reps, dt = 0, 0.0
        while reps == 0 or (dt < 2.0 and reps < 200):
            t = time.perf_counter()
            if fe_on:
                fq, fk, fg, fb = oracle.frontend_f64(qs, ks, gs, bs, A_log.cpu().double().numpy(),
                                                     dt_bias.cpu().double().numpy(), -5.0, 1e-6, 7)
                oracle.prefill_f64(fq, fk, vs, fg, fb, dinp.scale, cu, h0, threads=cores)
            else:
                oracle.prefill_f64(qs, ks, vs, gs, bs, dinp.scale, cu, h0, threads=cores)
            dt += time.perf_counter() - t
            reps += 1
        cpu = {"value": ns * T * H * reps / dt / 1e6, "unit": UNIT, "cores": cores,
               "kind": "oracle",
               "sample": f"first {ns} of {N} sequences x {T} token(s) x {H} heads from their pool "
                         f"slots, x {reps} run(s), FP64 " + ("front end and " if fe_on else "") +
                         "per-token recurrence"}

    if rank == 0:
        line = {"metric": DECODE_METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
                "data": "synthetic",
                "config": {"workload": f"decode_N{N}_T{T}_H{H}" + ("_frontend" if fe_on else ""),
                           "num_seqs": N, "tokens_per_seq": T, "frontend": fe_on,
                           "heads": H, "pool_slots": N, "head_dim": 128,
                           "parallelism": f"dp{world}" if world > 1 else "single",
                           "l2": "state and rows (%.3f GB) larger than 2x L2, no flush" %
                           (algo_bytes / 1e9) if flush is None else
                           "state and rows (%.3f GB) smaller than 2x L2: 256 MB written before "
                           "every step, each step timed alone" % (algo_bytes / 1e9)},
                "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": args.steps, "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="B8_T8192_H12")
    ap.add_argument("--variant", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=6)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--op", default="prefill", choices=["prefill", "decode"])
    ap.add_argument("--frontend", action="store_true",
                    help="prefill from raw projections through the input front end")
    ap.add_argument("--decode", default="256,1,12",
                    help="N,T,H of the decode workload: N sequences of T new tokens, H heads")
    ap.add_argument("--decode-frontend", action="store_true",
                    help="decode from raw projections through the input front end")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.op == "decode":
        return run_decode(args)

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        world = int(os.environ.get("WORLD_SIZE", "1"))
        return run_reference(args, rank, world)

    import torch
    rank, world, local = dist_setup("nccl")
    torch.cuda.set_device(local)
    import kda_chunked_recurrent_b200 as K
    from kda_chunked_recurrent_b200 import capi
    from kda_chunked_recurrent_b200.inputs import (WORKLOADS, make_frontend_inputs, make_inputs,
                                                   ragged_lengths)

    w = WORKLOADS[args.workload]
    lens = w["seqlens"] if w.get("seqlens") is not None else ragged_lengths(w["ragged"])
    kw = dict(with_h0=w.get("h0", False), with_ckpt=w.get("ckpt", False),
              fixed_layout=w.get("fixed", False))
    fe_opt = None
    if args.frontend:
        inp, A_log, dt_bias = make_frontend_inputs(lens, w["H"], rank_seed(w["seed"], rank), **kw)
    else:
        inp = make_inputs(lens, w["H"], rank_seed(w["seed"], rank), **kw)
    N, T, H = inp.num_seqs, inp.total_tokens, inp.num_heads
    fixed = inp.fixed_layout
    dev = torch.device("cuda", local)
    q, k, v, g, beta = (x.to(dev) for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
    cu = None if fixed else inp.cu_seqlens.to(dev)
    h0 = None if inp.h0 is None else inp.h0.to(dev)
    cko = None if inp.ckpt_offsets is None else inp.ckpt_offsets.to(dev)
    out = torch.empty(T, H, 128, dtype=torch.bfloat16, device=dev)
    ht = torch.empty(N, H, 128, 128, dtype=torch.float32, device=dev)
    ck = None if cko is None else torch.empty(N, H, 128, 128, dtype=torch.float32, device=dev)
    shape = capi.make_shape(N, T, H, max(lens))
    opts = {"variant": args.variant}
    if args.frontend:
        A_log, dt_bias = A_log.to(dev), dt_bias.to(dev)
        # every variant forms q/k norms, the gate and beta from the raw projections
        fe_flags = 7
        opts["frontend"] = capi.make_frontend(fe_flags, -5.0, 1e-6, A_log.data_ptr(),
                                              dt_bias.data_ptr())
    ws = K.Workspace(capi.kda_prefill_workspace_size(shape, cko is not None, opts), dev)
    desc = capi.kda_prefill_describe(shape, cko is not None, opts)
    variant = desc.split()[0].split("=")[1] if desc.startswith("variant=") else "split"
    hybrid_frac = 0.0   # share of the chunks the hybrid's separate prepare launch makes
    if variant == "hybrid":
        a, b = desc.split("prepare_chunks=")[1].split()[0].split("/")
        hybrid_frac = int(a) / int(b)
    stream = torch.cuda.current_stream(dev)
    P = lambda t: None if t is None else t.data_ptr()

    def step(events=None):
        o = dict(opts)
        if events is not None:
            o["events"] = events
        rc = capi.kda_prefill(P(q), P(k), P(v), P(g), P(beta), inp.scale, P(h0), P(cu), shape,
                              P(out), P(ht), P(ck), P(cko), ws.ptr, ws.nbytes, o,
                              stream.cuda_stream)
        if rc != 0:
            raise K.KDAError(rc)

    # schedule (packed layout or checkpoints), then prepare + recurrence (split) or
    # the single cooperative launch (fused)
    if variant == "token":
        launches_per_step = 1   # no metadata kernel for INT32 offsets without validation
    else:
        launches_per_step = (0 if fixed and cko is None else 1) + \
            {"fused": 1, "hybrid": 2}.get(variant, (1 if T > 0 else 0) + 1)
    in_bytes = sum(x.numel() * x.element_size() for x in (q, k, v, g, beta))
    flush = None
    if in_bytes < 2 * L2_BYTES:
        flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = ws.status()
    if st != 0:
        raise K.KDAError(st, "device status after warm-up")

    # per-step events: start, after prepare, after recurrence
    mk = lambda: torch.cuda.Event(enable_timing=True)
    ev_s = [mk() for _ in range(args.steps)]
    ev_p = [mk() for _ in range(args.steps)]
    ev_r = [mk() for _ in range(args.steps)]
    for e in ev_p + ev_r:
        e.record(stream)  # materialise the CUDA events before handing them to the library
    torch.cuda.synchronize()
    clk = ClockSampler(local if world > 1 else int(os.environ.get("CUDA_VISIBLE_DEVICES", "0").split(",")[0] or 0))
    clk.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    clk.mark_on()
    t_start, t_end = mk(), mk()
    t_start.record(stream)
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()   # evict the previous step's data from L2
        ev_s[i].record(stream)
        step([None, ev_p[i].cuda_event, ev_r[i].cuda_event])
    t_end.record(stream)
    torch.cuda.synchronize()
    clk.mark_off()
    barrier(world)
    clk.stop()
    if flush is None:
        ms_local = t_start.elapsed_time(t_end) / args.steps
    else:
        ms_local = statistics.mean(ev_s[i].elapsed_time(ev_r[i]) for i in range(args.steps))
    ms = max_over_ranks(ms_local, world)
    st = ws.status()
    if st != 0:
        raise K.KDAError(st, "device status after timed steps")
    prep_ms = statistics.mean(ev_s[i].elapsed_time(ev_p[i]) for i in range(args.steps))
    rec_ms = statistics.mean(ev_p[i].elapsed_time(ev_r[i]) for i in range(args.steps))

    units = T * H
    value = units * world / (ms / 1e3) / 1e6

    # ---- roofline of the dominant kernel
    peaks, peak_src = load_peaks()
    # from raw projections the gate is read as BF16: 256 B less per token and head
    gate_saving = 256 if args.frontend else 0
    prep_b, path_b = PREP_BYTES_PER_TOKHEAD - gate_saving, PATH_BYTES_PER_TOKHEAD - gate_saving
    in_b = path_b - OUT_BYTES_PER_TOKHEAD     # the inputs every prefill must read
    state_io = N * H * STATE_BYTES * ((1 if h0 is not None else 0) + 1 + (1 if ck is not None else 0))
    # Per launch: (ms, algorithmic bytes, designed bytes, sources).  The algorithmic
    # bytes of a launch are its share of the path's bytes: the inputs of the token-heads
    # whose chunk records it makes, the o rows it writes and the state I/O it does; over
    # the launches of one step they add up to path_b per token-head plus the state I/O.
    # The designed bytes add the chunk records each launch writes or reads.
    F = hybrid_frac
    fused_src = ["kda_fused.cu", "kda_prepare.cuh", "kda_recurrence.cuh", "kda_common.cuh",
                 "sm100_primitives.cuh"]
    prep_src = ["kda_prepare.cu", "kda_prepare.cuh", "kda_common.cuh", "sm100_primitives.cuh"]
    if variant == "hybrid":
        kernels = {
            "kda_prepare_kernel": (prep_ms, F * in_b * units, F * prep_b * units, prep_src),
            "kda_fused_kernel": (rec_ms, ((1 - F) * in_b + OUT_BYTES_PER_TOKHEAD) * units + state_io,
                                 ((1 - F) * prep_b + REC_BYTES_PER_TOKHEAD) * units + state_io,
                                 fused_src),
        }
    elif variant == "token":
        kernels = {
            token_kernel_name(capi, N, H): (prep_ms + rec_ms, path_b * units + state_io,
                                            path_b * units + state_io, TOKEN_SOURCES),
        }
    elif variant == "stream":
        # one launch: prepare CTAs and recurrence CTAs side by side, records through L2
        kernels = {
            "kda_stream_kernel": (prep_ms + rec_ms, path_b * units + state_io,
                                  (prep_b + REC_BYTES_PER_TOKHEAD) * units + state_io,
                                  ["kda_stream.cu", "kda_chain.cuh", "kda_prepare.cuh",
                                   "kda_common.cuh", "sm100_primitives.cuh"]),
        }
    elif variant == "fused":
        # one launch moves both halves' bytes (the records still go through HBM/L2)
        kernels = {
            "kda_fused_kernel": (prep_ms + rec_ms, path_b * units + state_io,
                                 (prep_b + REC_BYTES_PER_TOKHEAD) * units + state_io, fused_src),
        }
    else:
        kernels = {
            "kda_prepare_kernel": (prep_ms, in_b * units, prep_b * units, prep_src),
            "kda_recurrence_kernel": (rec_ms, OUT_BYTES_PER_TOKHEAD * units + state_io,
                                      REC_BYTES_PER_TOKHEAD * units + state_io,
                                      ["kda_recurrence.cu", "kda_recurrence.cuh", "kda_common.cuh",
                                       "sm100_primitives.cuh"]),
        }
    if args.frontend:   # the front-end instances of the prepare-side kernels
        kernels = {(n if n == "kda_recurrence_kernel" else n.replace("_kernel", "_fe_kernel")): v
                   for n, v in kernels.items()}
    dom = max(kernels, key=lambda n: kernels[n][0])
    dms, dbytes, dsgn, _ = kernels[dom]
    achieved = dbytes / (dms / 1e3) / 1e9
    traffic = ncu_traffic(dom, variant, units)
    roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
            if peak_src == "measured" else "fallback 6650 GB/s",
            "kernel_ms": round(dms, 4),
            "algorithmic_bytes": int(dbytes),
            "designed_bytes": int(dsgn),
            "traffic_ratio": None if traffic is None else round(traffic / dbytes, 3),
            "per_kernel_ms": {n: round(kernels[n][0], 4) for n in kernels}}
    path_bytes = path_b * units + state_io
    flops = FLOPS_PER_TOKHEAD_C64 * units
    s = ms / 1e3
    # the serial part: time of the launch that runs the recurrence chains per step of
    # the longest chain (a 64-token chunk, or a token for the token variant)
    max_len = max(lens) if lens else 0
    if variant == "token":
        chain_steps, chain_ms = max_len, prep_ms + rec_ms
    else:
        chain_steps = (max_len + 63) // 64 + (1 if ck is not None else 0)
        chain_ms = rec_ms if variant in ("split", "hybrid") else prep_ms + rec_ms
    chain = {"steps_per_chain": int(chain_steps),
             "step": "token" if variant == "token" else "chunk of 64 tokens",
             "us_per_step": round(1e3 * chain_ms / chain_steps, 3) if chain_steps else None,
             "launch_ms": round(chain_ms, 4)}
    path = {"bytes": int(path_bytes), "hbm_frac": round(path_bytes / s / 1e9 / peaks["hbm_gbs"], 4),
            "tc_frac_c64_burst": round(flops / s / 1e12 / peaks["bf16_tflops"], 4),
            "tc_frac_c64_sustained": round(flops / s / 1e12 / peaks["bf16_tflops_sustained"], 4),
            "binding_frac": round(max(flops / (peaks["bf16_tflops_sustained"] * 1e12),
                                      path_bytes / (peaks["hbm_gbs"] * 1e9)) / s, 4),
            "executed_chunk": 64}

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the timing.
    # Every step copies its inputs in and its outputs (o and the final state) out.  The
    # steps are pipelined the way a serving loop would run them: two sets of device
    # buffers, the host-to-device copies on a copy stream, the call and the device-to-host
    # copies on the compute stream, so step i + 1's inputs cross PCIe while step i's
    # outputs come back (the link is full duplex).
    e2e = None
    if args.e2e_steps > 0:
        hq, hk, hv, hg, hb = (x.pin_memory() for x in (inp.q, inp.k, inp.v, inp.g, inp.beta))
        hh0 = None if inp.h0 is None else inp.h0.pin_memory()
        ho = torch.empty(T, H, 128, dtype=torch.bfloat16).pin_memory()
        hht = torch.empty(N, H, 128, 128, dtype=torch.float32).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hg, hb)) + \
            (0 if hh0 is None else hh0.numel() * 4)
        d2h = ho.numel() * 2 + hht.numel() * 4
        # buffer set 0 is the timed run's own; set 1 is a second copy
        sets = [(q, k, v, g, beta, h0, out, ht),
                tuple(None if x is None else torch.empty_like(x) for x in (q, k, v, g, beta, h0, out, ht))]
        s_copy = torch.cuda.Stream(dev)
        in_ready = [torch.cuda.Event(), torch.cuda.Event()]
        in_free = [torch.cuda.Event(), torch.cuda.Event()]
        for e in in_free:
            e.record(stream)

        def e2e_step(i):
            bq, bk, bv, bg, bbeta, bh0, bout, bht = sets[i % 2]
            with torch.cuda.stream(s_copy):
                s_copy.wait_event(in_free[i % 2])   # the call two steps back is done with them
                for dst, src in ((bq, hq), (bk, hk), (bv, hv), (bg, hg), (bbeta, hb)):
                    dst.copy_(src, non_blocking=True)
                if hh0 is not None:
                    bh0.copy_(hh0, non_blocking=True)
                in_ready[i % 2].record(s_copy)
            stream.wait_event(in_ready[i % 2])
            rc = capi.kda_prefill(P(bq), P(bk), P(bv), P(bg), P(bbeta), inp.scale, P(bh0), P(cu),
                                  shape, P(bout), P(bht), P(ck), P(cko), ws.ptr, ws.nbytes, opts,
                                  stream.cuda_stream)
            if rc != 0:
                raise K.KDAError(rc)
            in_free[i % 2].record(stream)
            ho.copy_(bout, non_blocking=True)
            hht.copy_(bht, non_blocking=True)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        barrier(world)
        a, b = mk(), mk()
        a.record(stream)
        s_copy.wait_stream(stream)
        for i in range(args.e2e_steps):
            e2e_step(i)
        b.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b) / args.e2e_steps, world)
        # the pipelined calls read the same inputs as the timed ones: same outputs, bit for bit
        if not (torch.equal(ho, out.cpu()) and torch.equal(hht, ht.cpu())):
            raise RuntimeError("end-to-end outputs differ from the timed run's")
        e2e = {"value": units * world / (e_ms / 1e3) / 1e6, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": round(e_ms, 3),
               "pipeline": "double-buffered: H2D of step i+1 overlaps D2H of step i"}

    cpu = None   # (the oracle baseline is timed on the plain inputs only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.frontend:
        cpu = cpu_baseline(args.workload, max_tokens=65536, min_seconds=10.0, one_thread=True)
        cpu.pop("seconds", None)

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": {"workload": args.workload, "num_seqs": N, "seq_lens": "x".join(
                    map(str, sorted(set(lens)))) if len(set(lens)) < 4 else "ragged",
                    "total_tokens": T, "heads": H, "head_dim": 128, "h0": h0 is not None,
                    "checkpoint": ck is not None, "variant": variant,
                    "frontend": bool(args.frontend),
                    "chunk": None if variant == "token" else 64,
                    "parallelism": f"dp{world}" if world > 1 else "single",
                    "l2": ("inputs (%.2f GB) larger than L2, no flush" % (in_bytes / 1e9))
                    if flush is None else
                    ("inputs (%.3f GB) smaller than 2x L2: 256 MB written before every step, "
                     "each step timed from its first to its last kernel" % (in_bytes / 1e9))},
                "roofline": roof, "path_roofline": path, "chain": chain,
                "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_step * args.steps,
                "clocks": clk.summary()}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
