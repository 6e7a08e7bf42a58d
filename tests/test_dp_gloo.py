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


def _grouped_worker(rank, world, port, result_q):
    """Data parallel over tokens with grouped projections: each rank holds the
    stacked dA (n r x k) and dB (sum d x r) of its own token batch in one
    bucket; after the all-reduce they equal the gradients of all ranks' tokens
    together (the oracle's backward, projection by projection)."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    import numpy as np
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from bit_quantized_lora_02_b200 import synth
        from bit_quantized_lora_02_b200.dp import GradBucket
        from oracle import qlora_oracle as O
        ds, k, r, M, alpha = (24, 16, 8), 32, 4, 6, 16.0
        Whs = [O.dequantize_tensor(O.quantize_tensor(synth.weight(d, k, seed=i).reshape(-1), True)).reshape(d, k)
               for i, d in enumerate(ds)]
        As = [synth.lora_a(r, k, seed=i) for i in range(len(ds))]
        Bs = [synth.lora_b(d, r, seed=i) for i, d in enumerate(ds)]

        def grads(X, dY):
            dA, dB, row = [], [], 0
            for i, d in enumerate(ds):
                _, a, b = O.qlora_backward(dY[:, row:row + d], X, Whs[i], As[i], Bs[i], alpha, r)
                dA.append(a)
                dB.append(b)
                row += d
            return np.concatenate(dA), np.concatenate(dB)
        batches = [(synth.activations(M, k, seed=100 + q), synth.grad_output(M, sum(ds), seed=100 + q))
                   for q in range(world)]
        bucket = GradBucket([(len(ds) * r, k), (sum(ds), r)], "cpu")
        dA, dB = grads(*batches[rank])
        bucket.views[0].copy_(torch.from_numpy(dA.astype(np.float32)))
        bucket.views[1].copy_(torch.from_numpy(dB.astype(np.float32)))
        bucket.allreduce()
        X_all = np.concatenate([b[0] for b in batches])
        dY_all = np.concatenate([b[1] for b in batches])
        dA_all, dB_all = grads(X_all, dY_all)
        ok = np.allclose(bucket.views[0].numpy(), dA_all, rtol=1e-5, atol=1e-5)
        ok &= np.allclose(bucket.views[1].numpy(), dB_all, rtol=1e-5, atol=1e-5)
        result_q.put((rank, bool(ok), 0.0))
    finally:
        dist.destroy_process_group()


def test_grouped_gradient_bucket_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_grouped_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, _ in results:
        assert ok, rank
