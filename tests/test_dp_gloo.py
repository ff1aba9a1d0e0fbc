"""World-size-2 checks of the data-parallel host logic on CPU (gloo)."""
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


def _worker(r, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=r, world_size=world)
    try:
        from spatiotemporal_neural_field_b200 import dp
        frames = [None] * world
        dist.all_gather_object(frames, dp.rank_frame(75, dp.rank(), 150))
        t_max = dp.max_over_ranks(1.5 + r)          # rank 1 is the slow one
        g = torch.full((4, 3), float(r + 1))
        w = torch.arange(5, dtype=torch.float32) * (r + 1)
        dp.allreduce_gradients([g, w])
        q.put((r, frames, t_max, g.tolist(), w.tolist()))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_time_and_sum_gradients():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, frames, t_max, g, w in res:
        assert frames == [75, 76]                      # distinct consecutive frames, no overlap
        assert t_max == 2.5                            # max over ranks
        assert g == [[3.0] * 3] * 4                    # 1 + 2 on every element
        assert w == [0.0, 3.0, 6.0, 9.0, 12.0]


def test_single_process_is_a_no_op():
    from spatiotemporal_neural_field_b200 import dp
    t = torch.ones(3)
    dp.allreduce_gradients([t])
    assert t.tolist() == [1.0, 1.0, 1.0]
    assert dp.max_over_ranks(2.0) == 2.0 and dp.world() == 1 and dp.rank() == 0
