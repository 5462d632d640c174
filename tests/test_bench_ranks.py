"""bench.py's multi-rank host logic on CPU, as torchrun runs it for --gpus 2: two gloo ranks on
127.0.0.1. The path does not shard (each rank runs a full replica), so the only exchange is the
element-wise maximum of the timings over the ranks, and the reference arm runs on rank 0 alone."""
import datetime
import multiprocessing as mp
import os
import socket


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench

        # rank r reports [r + 1, 10 - r, -r]: the slowest (largest) value of each entry must win
        got = bench.max_over_ranks([rank + 1.0, 10.0 - rank, -float(rank)], dist, "cpu")
        # the reference arm: every rank but 0 leaves at once, without work and without output
        rc = bench.run_reference(None, rank) if rank != 0 else None
        dist.barrier()
        q.put((rank, got, rc))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_reference_arm_with_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in procs:
            rank, got, rc = q.get(timeout=120)
            results[rank] = (got, rc)
    finally:
        for p in procs:
            p.join(timeout=30)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    assert results[0][0] == [2.0, 10.0, 0.0]
    assert results[1][0] == [2.0, 10.0, 0.0]
    assert results[1][1] == 0


def test_max_over_ranks_without_a_process_group():
    import bench

    assert bench.max_over_ranks([1, 2.5], None, "cpu") == [1.0, 2.5]
