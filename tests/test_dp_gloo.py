"""The data-parallel path on CPU: two gloo ranks, each with its token shard.

Each rank computes the adapter gradients of its shard with the oracle (the GPU kernels are
not needed for the host-side logic); after allreduce_adapter_grads every rank must hold the
gradients of the whole batch, and max_over_ranks must agree on every rank."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_quantized_lora_03_b200 import dp, inputs
from oracle import nf4_oracle as O


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        li = inputs.random_linear(37, 128, 192, 16, 0.5, seed=3)
        Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
        sl = dp.token_shard(li.t, rank, world)
        f = lambda t: t.float().numpy()  # noqa: E731
        _, dL1, dL2, _ = O.qlora_linear_bwd(f(li.dY)[sl], f(li.X)[sl], Wdq, f(li.L1), f(li.L2), li.s)
        g1 = torch.from_numpy(dL1.astype(np.float32))
        g2 = torch.from_numpy(dL2.astype(np.float32))
        dp.allreduce_adapter_grads([g1, g2])
        mx = dp.max_over_ranks(float(rank + 1))
        out[rank] = (g1.numpy().copy(), g2.numpy().copy(), mx)
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_allreduce_equals_full_batch():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    li = inputs.random_linear(37, 128, 192, 16, 0.5, seed=3)
    Wdq = O.nf4_dequantize(O.nf4_quantize(li.Wt.numpy()))
    f = lambda t: t.float().numpy()  # noqa: E731
    _, dL1, dL2, _ = O.qlora_linear_bwd(f(li.dY), f(li.X), Wdq, f(li.L1), f(li.L2), li.s)
    for rank in range(world):
        g1, g2, mx = out[rank]
        assert np.allclose(g1, dL1, rtol=1e-5, atol=1e-6)
        assert np.allclose(g2, dL2, rtol=1e-5, atol=1e-6)
        assert mx == float(world)


def test_token_shards_cover_the_batch():
    for t in [1, 7, 4096, 4097]:
        for world in [1, 2, 3, 8]:
            parts = [dp.token_shard(t, r, world) for r in range(world)]
            assert parts[0].start == 0 and parts[-1].stop == t
            for a, b in zip(parts, parts[1:]):
                assert a.stop == b.start
            sizes = [p.stop - p.start for p in parts]
            assert max(sizes) - min(sizes) <= 1
