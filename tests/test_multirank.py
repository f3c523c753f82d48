"""Multi-rank host logic of bench.py on CPU: two gloo ranks.

Each rank must draw its own independent matrices (weak scaling: one set of
layers per GPU, no collective on the data path) and the job time must be the
maximum over ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from sparse_gemm_wanda_b200 import inputs
        wl = inputs.workloads()["tiny"]
        mats, calib = bench.make_tensors(wl, rank)
        w = mats[0]["W"].float()
        digest = torch.tensor([w.sum().item(), w.abs().sum().item(),
                               calib["in256"].float().sum().item()], dtype=torch.float64)
        gathered = [torch.zeros(3, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        mx = bench.max_over_ranks(1.5 + rank, "cpu")
        out[rank] = (tuple(tuple(g.tolist()) for g in gathered), mx)
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_ranks_independent_data_and_max_time():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, join=True,
                       start_method="spawn")
    assert set(out.keys()) == {0, 1}
    g0, mx0 = out[0]
    g1, mx1 = out[1]
    assert g0 == g1                    # both ranks saw the same gathered digests
    assert g0[0] != g0[1]              # and the two ranks' matrices differ
    assert mx0 == mx1 == 2.5           # max over ranks


def test_single_process_max_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
