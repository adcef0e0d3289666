"""The N>1 host path of bench.py on CPU: two gloo ranks, each timing its own
replica, agree on the slowest rank's time and on the whole-job throughput."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = 100.0 + 50.0 * rank                     # rank 1 is the slower replica
    mx = bench.max_over_ranks(local_ms, world, "cpu")
    q.put((rank, mx, bench.job_throughput(world, 4, 10, mx)))
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_replicas_take_the_slowest_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [150.0, 150.0]
    # 2 ranks x 4 queries x 10 steps in 150 ms
    assert abs(out[0][2] - 2 * 4 * 10 / 0.150) < 1e-6 and out[0][2] == out[1][2]


def test_single_rank_helpers():
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert abs(bench.job_throughput(1, 4, 1000, 300.0) - 4 * 1000 / 0.3) < 1e-9
    ab = bench.algorithmic_bytes(__import__("synth").workload(3))
    # 4 requests: 131072 summaries x 128 B, 16384 pool keys x 128 B + ids, reindex, 8 attends
    assert ab["block_summaries"] == 4 * 131072 * 128
    assert ab["step"] == ab["index"] + ab["attend"] + ab["append"]
