"""The data-parallel exchange on two CPU ranks (gloo): the gradient bucket sums
dA/dB views across ranks and timings reduce to their maximum."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from bit_quantized_lora_02_b200.dp import GradBucket, max_over_ranks
        shapes = [(8, 64), (64, 8), (5, 33), (33, 5)]      # dA, dB of two projections (one ragged)
        b = GradBucket(shapes, "cpu")
        for i, v in enumerate(b.views):
            v.copy_(torch.arange(v.numel(), dtype=torch.float32).view(v.shape) * (rank + 1) + i)
        b.allreduce()
        ok = True
        for i, v in enumerate(b.views):
            base = torch.arange(v.numel(), dtype=torch.float32).view(v.shape)
            want = base * sum(r + 1 for r in range(world)) + i * world
            ok &= torch.equal(v, want)
            ok &= v.data_ptr() % 16 == 0
        mx = max_over_ranks(10.0 + rank, "cpu")
        result_q.put((rank, bool(ok), mx))
    finally:
        dist.destroy_process_group()


def test_gradient_bucket_allreduce_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, mx in results:
        assert ok, rank
        assert mx == 11.0


def test_single_process_bucket_is_identity():
    from bit_quantized_lora_02_b200.dp import GradBucket, max_over_ranks
    b = GradBucket([(3, 4)], "cpu")
    b.views[0].fill_(2.0)
    b.allreduce()
    assert torch.all(b.views[0] == 2.0)
    assert max_over_ranks(3.5, "cpu") == 3.5
