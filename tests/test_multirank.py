"""The multi-GPU path of bench.py is replicas only: each rank runs its own batch
(seed = rank), no collective touches the data path, and the job's time is the
maximum over ranks. This checks the rank-level aggregation with two gloo
processes on the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, times, out):
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.reduce_max(times[rank], world, "cpu")
        value = bench.job_throughput(4096, 10, world, ms)
        out.put((rank, ms, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    times = [120.0, 150.0]
    procs = [ctx.Process(target=_worker, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, value in res:
        assert ms == 150.0
        assert value == pytest.approx(2 * 4096 * 10 / 0.150)


def test_single_rank_needs_no_process_group():
    import bench

    assert bench.reduce_max(3.5, 1) == 3.5
    assert bench.job_throughput(64, 2, 1, 1000.0) == 128.0


def test_launcher_starts_ranks_that_split_an_expert_parallel_group(tmp_path):
    """bench.launch_ranks (what `bench.py --gpus N` runs as a plain command) starts N ranks under
    torch.distributed.run on 127.0.0.1; each rank's group plan (token slice, owned experts, receive
    rows) is exchanged through the process group: the token slices partition the batch, the owned
    experts partition the experts, and every rank sizes the same receive buffers. The slowest rank's
    time is the job's."""
    import json
    import sys

    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench

    out = tmp_path / "ranks.json"
    probe = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rank_probe.py")
    rc = bench.launch_ranks(2, 180, script=probe, argv=[str(out), "16387", "256", "8"])
    assert rc == 0
    res = json.loads(out.read_text())
    assert res["world"] == 2 and res["master"] == "127.0.0.1" and res["ms"] == 11.0
    plans = res["plans"]
    assert [tuple(p["tokens"]) for p in plans] == [(0, 8194), (8194, 16387)]
    assert [tuple(p["experts"]) for p in plans] == [(0, 128), (128, 256)]
    assert plans[0]["recv_rows"] == plans[1]["recv_rows"] == 16387 * 8
