"""Host-side multi-rank logic of bench.py on CPU ranks (gloo, world size 2):
the step time reported is the maximum over ranks, and throughput counts the
clips of every rank."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms = 100.0 + 25.0 * rank  # rank 1 is the slow one
    out[rank] = bench.reduce_max(ms, world, torch.device("cpu"))
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    world = 2
    out = mp.get_context("spawn").Manager().dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    assert dict(out) == {0: 125.0, 1: 125.0}


def test_single_rank_is_identity_and_config_names_replicas():
    import bench
    from video_diffusion_transformer_h3attn_b200 import inputs
    assert bench.reduce_max(3.5, 1) == 3.5
    w = inputs.make_workload("cfg", [256], 2, 64, seed=1, norm=False)
    assert bench.workload_config(w, 1)["parallelism"] == "replicas"
    assert bench.workload_config(w, 4)["parallelism"] == "dp4"
    assert bench.workload_config(w, 4)["global_batch"] == 4
