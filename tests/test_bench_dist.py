"""Multi-rank host logic of bench.py, as world_size-2 gloo process groups on the CPU.

The data path has no collective: every rank runs the same per-GPU workload on
its own seeded inputs (weak scaling), the timing barrier and the max-over-ranks
reduction are the only group operations, and under the reference arm only
rank 0 works and prints.
"""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _child(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import argparse
    import contextlib
    import io

    import torch.distributed as dist

    import bench
    from kda_chunked_recurrent_b200.inputs import make_inputs

    r, w, local = bench.dist_setup("gloo")
    res = {"rank": r, "world": w, "local": local}
    bench.barrier(w)
    res["max"] = bench.max_over_ranks(1.5 + r, w)
    seed = bench.rank_seed(1002, r)
    res["seed"] = seed
    inp = make_inputs([64], 1, seed)
    res["q0"] = float(inp.q.float()[0, 0, :4].sum())
    buf = io.StringIO()
    args = argparse.Namespace(steps=1, warmup=0, workload="B1_T64_H1", gpus=w)
    with contextlib.redirect_stdout(buf):
        res["ref_rc"] = bench.run_reference(args, r, w)
    res["ref_out"] = buf.getvalue()
    bench.barrier(w)
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump(res, f)


def test_two_rank_timing_and_reference_arm(tmp_path):
    world = 2
    mp.start_processes(_child, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["world"] == world and d["local"] == r
        # max over ranks reaches every rank
        assert d["max"] == pytest.approx(1.5 + world - 1)
        assert d["ref_rc"] == 0
    # each rank draws its own inputs
    assert res[0]["seed"] != res[1]["seed"]
    assert res[0]["q0"] != res[1]["q0"]
    # the reference arm: rank 0 alone runs the oracle and prints one JSON line
    assert res[1]["ref_out"] == ""
    lines = [l for l in res[0]["ref_out"].splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0
