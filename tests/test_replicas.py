"""Multi-process replicas (bench.py --gpus N): world size 2 over gloo on the CPU.

The path does not shard (one bank per GPU, no exchange), so N GPUs run N
independent replicas.  What crosses ranks is only the timing: every rank must
take the max over ranks, and only rank 0 prints.  These tests run that logic
in two spawned processes on 127.0.0.1."""
import json
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    r, w, loc = bench.replica_env()
    import datetime
    dist.init_process_group("gloo", rank=r, world_size=w, timeout=datetime.timedelta(seconds=60))
    try:
        # rank r timed 10 + r ms: every rank must see the slowest, 11 ms
        got = bench.max_over_ranks(10.0 + r, w, torch.device("cpu"))
        dist.barrier()
        # the reference arm runs on rank 0 only; the others return at once
        class A:
            workload, steps, warmup, gpus, cpu_seconds = "tiny-fp32-64x512", 1, 0, w, 0.2
        import contextlib
        import io
        buf = io.StringIO()
        if r != 0:
            with contextlib.redirect_stdout(buf):
                bench.run_reference(A, r)
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump({"rank": r, "world": w, "local": loc, "max": got, "printed": buf.getvalue()}, f)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rank_zero_only_two_processes(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    assert [x["rank"] for x in res] == [0, 1] and all(x["world"] == 2 for x in res)
    assert [x["local"] for x in res] == [0, 1]
    assert all(x["max"] == 11.0 for x in res)
    assert res[1]["printed"] == ""


def test_single_process_is_its_own_max(monkeypatch):
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.replica_env() == (0, 1, 0)
    assert bench.max_over_ranks(3.5, 1, torch.device("cpu")) == 3.5
