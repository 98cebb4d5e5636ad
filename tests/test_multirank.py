"""Host-side plumbing of the N-GPU benchmark, run as two gloo ranks on the CPU.

The decode path shards by sequence with no data-path collective (each rank is an
independent replica), so what N > 1 adds is timing plumbing: the elapsed time is the
slowest rank's, the value counts the units of all ranks, and the reference arm runs on
rank 0 alone.
"""
import io
import json
import os
import socket
import sys
import types
from contextlib import redirect_stdout

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, torch.device("cpu"))
        value = bench.whole_job_value(world, 24576, 3, ms)
        # the reference arm: rank 0 times a tiny oracle sample and prints; others return
        args = types.SimpleNamespace(workload="opt-125m", layers=None, steps=1, warmup=1)
        buf = io.StringIO()
        with redirect_stdout(buf):
            bench.run_reference(args)
        dist.barrier()
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": value, "printed": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    # every rank sees the slowest rank's time
    assert r[0]["ms"] == r[1]["ms"] == 15.0
    # whole-job throughput: 2 replicas x 24,576 layer-tokens x 3 steps in 15 ms
    assert r[0]["value"] == pytest.approx(2 * 24576 * 3 / 0.015)
    # the reference arm prints one JSON line on rank 0 and nothing elsewhere
    assert r[1]["printed"] == ""
    lines = r[0]["printed"].strip().splitlines()
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world and line["value"] > 0
    assert line["config"]["parallelism"] == f"replicas x{world}"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
