"""The multi-rank host logic of bench.py on CPU: two gloo ranks on
127.0.0.1, each with its own problem (weak scaling); the job time is the
max over ranks and the value is all ranks' work over that time."""
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


def _rank_main(rank, world, port, out):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    my_ms = 1.5 + rank  # rank 1 is the slow one
    slowest = bench.max_over_ranks(world, my_ms)
    out[rank] = slowest
    out[world + rank] = bench.whole_job(world, 10.0, slowest)
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_max_and_whole_job():
    world = 2
    out = torch.zeros(2 * world, dtype=torch.float64).share_memory_()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[:world].tolist() == [2.5, 2.5]
    assert out[world:].tolist() == pytest.approx([8.0, 8.0])


def test_each_rank_draws_its_own_instance():
    """bench.py builds every row with seed_offset = rank: rank 0 gets the
    workload itself, other ranks another draw of the same shapes and
    distributions (weak scaling: no two ranks solve the same problem)."""
    from mxfp8_block_scaled_nvfp4_b200 import workloads
    for name in ["tiny", "gemv", "prefill", "moe", "quant1g", "prefill_bwd"]:
        sd = 1 if name in ("tiny", "gemv") else 32
        r0 = workloads.make(name, scale_down=sd)
        r0b = workloads.make(name, scale_down=sd, seed_offset=0)
        r1 = workloads.make(name, scale_down=sd, seed_offset=1)
        for k in r0:
            assert torch.equal(r0[k], r0b[k])
            assert r1[k].shape == r0[k].shape and r1[k].dtype == r0[k].dtype
            assert not torch.equal(r0[k], r1[k]), (name, k)
