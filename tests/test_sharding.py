"""Host logic of a packed batch split across ranks (CPU, gloo, 2 ranks).

Each rank takes some images (balanced on S^2), computes the q/k/v amax of its
share with the oracle, and the ranks all-reduce(max) them: the result must be
the amax of the whole batch, and the ring rule applied to it must give the
descales a single process gets."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from fp8_quantized_vit_b200.sharding import allreduce_amax3, local_batch, shard_images


def test_shard_images_cover_and_balance():
    lens = [14400, 14400, 14400, 3000, 1, 0, 512]
    for world in (1, 2, 3, 4):
        parts = [shard_images(lens, world, r) for r in range(world)]
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(lens)))
        loads = [sum(lens[i] ** 2 for i in p) for p in parts]
        # greedy bound: no rank exceeds the average by more than one image
        assert max(loads) <= sum(x ** 2 for x in lens) / world + max(lens) ** 2
    with pytest.raises(ValueError):
        shard_images(lens, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, lens, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import synth
        H, D = 16, 72
        T = sum(lens)
        full = [synth.bf16_tensor(synth.stream_key(41, 0, t), T, H * D) for t in range(3)]
        _, _, ranges = local_batch(lens, world, rank)
        local = [np.concatenate([x[a:b] for a, b in ranges]) if ranges else x[:0] for x in full]
        amax = torch.tensor([oracle.amax_bf16(x) for x in local], dtype=torch.float32)
        allreduce_amax3(amax)
        want = [oracle.amax_bf16(x) for x in full]
        ring = oracle.Ring()
        desc = ring.update(amax.numpy())
        ring1 = oracle.Ring()
        desc1 = ring1.update(np.asarray(want, np.float32))
        result_q.put((rank, amax.tolist() == [float(np.float32(w)) for w in want],
                      bool((desc.view(np.uint32) == desc1.view(np.uint32)).all())))
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_batch_amax():
    lens = [700, 300, 520, 64]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, lens, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert sorted(r[0] for r in results) == [0, 1]
    assert all(r[1] and r[2] for r in results), results
