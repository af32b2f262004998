"""The multi-process plumbing of bench.py on CPU: two gloo ranks.

The attention path has no exchange step (every (batch, head) or (sequence,
head) unit is independent), so N GPUs run N replicas; what is shared is the
host logic: a barrier, the max of the step times over ranks and the sum of the
work.  Those run here with world size 2 over gloo on 127.0.0.1."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    bench.barrier(world)
    t = bench.max_over_ranks(10.0 + rank, world)   # rank 1 is the slow one
    w = bench.sum_over_ranks(100.0 * (rank + 1), world)
    bench.barrier(world)
    out[rank] = (t, w)
    dist.destroy_process_group()


def test_two_rank_max_time_and_total_work():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == out[1] == (11.0, 300.0)


def _ref_worker(rank, world, port, out):
    import contextlib
    import io
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world))
    import bench
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        rc = bench.main(["--impl", "reference", "--workload", "tiny_causal", "--steps", "1",
                         "--warmup", "3"])
    # the reference arm runs the oracle alone: the product library stays unloaded
    with open("/proc/self/maps") as f:
        loaded = "libattn.so" in f.read()
    out[rank] = (rc, buf.getvalue(), loaded)


def test_reference_arm_prints_on_rank_zero_only():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_ref_worker, args=(2, 0, out), nprocs=2, join=True, start_method="spawn")
    import json
    assert out[0][0] == 0 and out[1][0] == 0
    line = json.loads(out[0][1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert out[1][1] == ""
    assert not out[0][2] and not out[1][2], "the reference arm loaded libattn.so"
