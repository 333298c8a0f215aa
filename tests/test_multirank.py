"""Multi-rank host logic of the benchmark on CPU (gloo, world size 2).

The path shards into independent problems, so `bench.py --gpus N` runs one
replica per rank with no data-path collective.  The process group is used only
for the timing barrier and the maximum of the per-rank times.  What is checked:

* `dist_env` reads RANK / WORLD_SIZE / LOCAL_RANK as torchrun sets them;
* `max_over_ranks` gives every rank the slowest rank's time (gloo: host tensor);
* the barrier returns on every rank;
* each rank's replica has the same shape and its own seeds, so its inputs differ;
* the whole-job value is the work of all ranks over the slowest time;
* the reference arm runs on rank 0 alone: other ranks print nothing and return.
"""
import contextlib
import datetime
import io
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
from bit_quantized_attention_sage_b200 import synth  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        env = bench.dist_env()
        ms = 10.0 + 5.0 * rank  # this rank's step time
        ms_max = bench.max_over_ranks(ms, world)
        bench.barrier(world)
        w = bench.rank_workload(synth.TINY, rank)
        q = synth.head_q(w, 0, 0)
        value = bench.aggregate_value(synth.TINY.ops(), world, ms_max)
        # the reference arm: rank 0 alone runs it (stubbed here to a fixed sample)
        args = type("A", (), {"workload": synth.TINY.name, "steps": 1, "warmup": 0})()
        saved = bench.cpu_baseline
        bench.cpu_baseline = lambda w_, t_: {"value": 1.0, "cores": 1, "sample": "stub"}
        buf = io.StringIO()
        try:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(args)
        finally:
            bench.cpu_baseline = saved
        bench.barrier(world)
        res = {"env": list(env), "ms_max": ms_max, "seed": w.seed, "q_sum": int(q.astype(np.int64).sum()),
               "value": value, "ref_out": buf.getvalue()}
        with open(os.path.join(out_dir, "rank%d.json" % rank), "w") as f:
            json.dump(res, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / ("rank%d.json" % i))) for i in range(world)]
    for i in range(world):
        assert r[i]["env"] == [i, world, i]
        assert r[i]["ms_max"] == 15.0  # the slowest rank's time on every rank
        assert r[i]["value"] == pytest.approx(synth.TINY.ops() * world / 15e-3 / 1e12)
    assert r[0]["seed"] != r[1]["seed"] and r[0]["q_sum"] != r[1]["q_sum"]
    line = json.loads(r[0]["ref_out"].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == world
    # the reference arm reports the GPU arm's metric, unit and direction on
    # the same workload, its own CPU baseline and an e2e with no copies
    assert (line["metric"], line["unit"], line["higher_is_better"]) == (bench.METRIC, bench.UNIT, True)
    assert line["config"]["workload"] == synth.TINY.name
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert r[1]["ref_out"] == ""  # other ranks exit without work


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)
    assert bench.rank_workload(synth.TINY, 0) == synth.TINY
    assert bench.aggregate_value(2e12, 1, 1000.0) == pytest.approx(2.0)
