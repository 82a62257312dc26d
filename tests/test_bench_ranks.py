"""The replicas' rank logic of bench.py, as two gloo ranks on the CPU.

bench.py runs one replica of the layer per GPU with no data-path collective:
the ranks only meet at the barriers around the timed region and in the
maximum of the timed duration, rank 0 alone prints the line, and the whole-job
value counts every rank's tokens. The same Comm code runs here over gloo.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        comm = bench.Comm(world, dist, "cpu")
        comm.barrier()
        # each rank times its own replica; the job time is the slowest rank's
        own_ms = 10.0 + 5.0 * rank
        ms_max = comm.max(own_ms)
        comm.barrier()
        value = bench.replica_value(16384, world, 100, ms_max)
        # the reference arm: rank 0 alone runs and prints (the others return at once)
        buf = io.StringIO()
        if rank != 0:
            with redirect_stdout(buf):
                bench.run_reference(None, rank)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms_max": ms_max, "value": value, "ref_stdout": buf.getvalue(),
                       "variants": [bench.replica_variant(v, rank) for v in range(3)]}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    world = 2
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    # both ranks see the slowest rank's time, and the value counts both replicas
    assert res[0]["ms_max"] == res[1]["ms_max"] == 15.0
    assert res[0]["value"] == res[1]["value"] == pytest.approx(16384 * 2 * 100 / 0.015)
    # ranks other than 0 run no reference work and print nothing
    assert res[1]["ref_stdout"] == ""
    # every replica draws its own input batches
    assert not set(res[0]["variants"]) & set(res[1]["variants"])


def test_single_rank_comm_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    comm = bench.Comm(1)
    comm.barrier()
    assert comm.max(3.5) == 3.5
    assert bench.replica_value(16384, 1, 10, 2.0) == pytest.approx(16384 * 10 / 0.002)
