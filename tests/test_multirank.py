"""The multi-rank host logic of bench.py on CPU: two gloo ranks.

bench.py --gpus N runs one process per GPU (torchrun), each on its own seeded
batch, with no data-path collective; the only exchange is the max over ranks
of the measured times.  These tests run that host logic as two gloo processes
on CPU: the max reduction, the whole-job throughput, the per-rank seeding and
the reference arm's rank-0-only output.
"""

import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _load_bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench = _load_bench()
        local_ms = [3.0, 5.0][rank]
        ms = bench.max_over_ranks(local_ms, torch.device("cpu"), world)
        # the reference arm: rank 0 alone prints, the others return without work
        buf = io.StringIO()

        class A:
            workload, steps, warmup = "tiny_n256", 1, 0

        with redirect_stdout(buf):
            bench.run_reference(A, rank, world)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "ref_out": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_reference_arm(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    assert r[0]["ms"] == r[1]["ms"] == 5.0                 # both ranks see the slowest rank
    assert r[1]["ref_out"] == ""                            # rank 1 of the reference arm: no work, no line
    line = json.loads(r[0]["ref_out"].strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] == 0


def test_job_throughput_is_weak_scaling_sum():
    bench = _load_bench()
    # every rank does the same FLOPs; the job takes the slowest rank's time
    assert bench.job_tflops(10 ** 12, 1, 1000.0) == pytest.approx(1.0)
    assert bench.job_tflops(10 ** 12, 8, 1000.0) == pytest.approx(8.0)
    assert bench.max_over_ranks(2.5, None, 1) == 2.5


def test_each_rank_draws_its_own_batch():
    sys.path.insert(0, ROOT)
    import fqa_synth as synth
    bench = _load_bench()
    w = synth.workload("tiny_n256")
    g0, w0 = bench.host_inputs(w, 0)
    g1, w1 = bench.host_inputs(w, 1)
    g0b, _ = bench.host_inputs(w, 0)
    assert w0.seed == w.seed and w1.seed == w.seed + 7919
    assert np.array_equal(g0["q"], g0b["q"])                 # seeded: rank 0 reproduces
    assert not np.array_equal(g0["q"], g1["q"])              # rank 1 has its own batch
