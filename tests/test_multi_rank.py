"""The multi-GPU path of bench.py on the host: N independent replicas (no collective on the data path), a
barrier around the timed region, the job's time = the slowest rank's (all-reduce MAX), value = N x units per
rank / time.  Run as two gloo ranks on the CPU; the GPU work itself is per rank and covered elsewhere."""
import importlib.util
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    b = _bench()
    dist.barrier()
    t = b.max_over_ranks(10.0 + 5.0 * rank, world)                 # rank 1 is the slow one
    e = b.max_over_ranks(3.0 - rank, world)
    from kv_cache_vector_norm_b200 import synth
    # replicas draw their caches from their own seed (seed = rank): different data, same shapes
    x = synth.kv_tensor(rank, synth.STREAM_K, 1, 2, 16, 64)
    results[rank] = (t, e, b.job_value(world, 1000, t), float(x.float().sum()))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_rank, args=(world, port, results), nprocs=world, join=True, start_method="spawn")
    assert results[0][:3] == results[1][:3] == (15.0, 3.0, 2 * 1000 / 0.015 / 1e6)
    assert results[0][3] != results[1][3]


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(7.5, 1) == 7.5
    assert b.job_value(1, 2_000_000, 1000.0) == 2.0
