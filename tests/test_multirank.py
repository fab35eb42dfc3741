"""Multi-rank host logic of the bench on CPU (gloo, world size 2): the
max-over-ranks timing reduction, the sum of the ranks' work, and per-rank
input shards (rank k draws the heads [k*H, (k+1)*H) of one larger seeded
problem, so ranks hold different inputs of the same shape)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    from entropy_adaptive_radius_b200 import inputs
    t = bench.max_over_ranks(10.0 + 5.0 * rank)
    w = bench.sum_over_ranks(1.5 + rank)
    Q, K, V = inputs.make_qkv(2, 3, 4, 2, 8, seed=7, dtype="f32", head_offset=rank * 2)
    out[rank] = (t, Q.clone(), V.clone(), w)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_input_shards():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][3] == out[1][3] == 4.0
    from entropy_adaptive_radius_b200 import inputs
    Q, K, V = inputs.make_qkv(2, 3, 4, 4, 8, seed=7, dtype="f32")
    assert torch.equal(out[0][1], Q[:2]) and torch.equal(out[1][1], Q[2:])
    assert torch.equal(out[1][2], V[2:])
    assert not torch.equal(out[0][1], out[1][1])


def test_max_over_ranks_without_process_group():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.sum_over_ranks(3.5) == 3.5
