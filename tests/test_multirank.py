"""The multi-process logic of the benchmark on CPU, world size 2 over gloo.

Heads are independent, so each rank runs its own batch and no data-path
collective exists: the only cross-rank step is the max of the step time
(outside the timed region).  These tests run that step and the sharding
argument on the host."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

WORLD = 2


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _max_worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        ms = 1.0 + 0.5 * rank                   # rank 1 is the slow one
        got = bench.max_over_ranks(ms, world, "cpu")
        out.put((rank, got, bench.job_throughput(1000, world, got)))
    finally:
        dist.destroy_process_group()


def _shard_worker(rank, world, port, out):
    import datetime
    import torch
    import torch.distributed as dist
    from oracle import nystrom as orc
    from nystr_self_attention_segment_b200.inputs import make_custom
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        x = make_custom((1, 4, 32, 16), "f32", seed=77, conv_k=5)
        mine = [h for h in range(4) if h % world == rank]
        part = np.stack([orc.nystrom_head(x["Q"][0, h], x["K"][0, h], x["V"][0, h], 8, 6,
                                          x["conv_w"][h])["out"] for h in mine])
        buf = [torch.zeros(part.shape, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(buf, torch.from_numpy(part))
        out.put((rank, [b.numpy() for b in buf]))
    finally:
        dist.destroy_process_group()


def run(fn):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=fn, args=(r, WORLD, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res, key=lambda r: r[0])


def test_step_time_is_the_max_over_ranks():
    res = run(_max_worker)
    for rank, got, thr in res:
        assert got == pytest.approx(1.5)
        assert thr == pytest.approx(1000 * WORLD / 1.5e-3)


def test_head_sharding_reproduces_the_whole_batch():
    from oracle import nystrom as orc
    from nystr_self_attention_segment_b200.inputs import make_custom
    x = make_custom((1, 4, 32, 16), "f32", seed=77, conv_k=5)
    whole = orc.nystrom_forward(x["Q"], x["K"], x["V"], 8, 6, x["conv_w"])[0]
    for rank, parts in run(_shard_worker):
        for r, p in enumerate(parts):
            heads = [h for h in range(4) if h % WORLD == r]
            np.testing.assert_array_equal(p, whole[heads])
