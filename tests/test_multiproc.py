"""World-size-2 checks (gloo, CPU) of the bench's multi-rank host logic: every
rank runs its own replica, the elapsed time is the max over ranks, and the
reported value is all ranks' steps over that time."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    r, w, local = bench.dist_env()
    elapsed = 1.0 + rank  # rank 1 is the slow one
    t_max = bench.reduce_max(elapsed, w, torch.device("cpu"))
    value = bench.aggregate_value(100, w, t_max)
    dist.barrier()
    dist.destroy_process_group()
    q.put((r, w, local, t_max, value))


def test_two_rank_timing_aggregation():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and all(r[1] == 2 for r in res)
    for _, _, _, t_max, value in res:
        assert t_max == 2.0                      # max over ranks, not the local time
        assert value == pytest.approx(100.0)     # 2 ranks x 100 steps / 2 s


def test_stage_bytes_match_survey_decode32k():
    import bench
    from sparse_attention_04_b200 import inputs
    wl = inputs.WORKLOADS["decode32k"]
    assert bench.stage_bytes(wl, [32768])["step"] == 11_043_072
    fp8 = inputs.WORKLOADS["fp8"]
    assert bench.stage_bytes(fp8, [131072] * 4)["step"] == 4 * (131072 * 132 + 8192 + 256 + 2_359_296 + 147_456 + 131_072)
