"""The N>1 host path of bench.py on CPU: two gloo ranks.

The wave-round path has no exchange step, so N GPUs run N independent
replicas; the only collectives are the barrier and the max over ranks of the
device time.  These run here on the gloo backend with world size 2, including
a replica that leaves between steps: the surviving rank's reduction ends with
an error within the process group's timeout instead of waiting for good.
"""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _load_bench()
        # each replica reports its own device time; every rank must see the slowest
        got = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        dist.barrier()
        seeds = [None] * world
        dist.all_gather_object(seeds, bench.replica_seed(rank))

        class Args:
            steps, warmup, gpus, config = 1, 0, world, "wan13b_round"
        ref = bench.run_reference(Args, rank, world) if rank == 1 else "skipped"
        out[rank] = (got, seeds, ref)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_max_and_split_seeds():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == 15.0 and res[1][0] == 15.0
    assert res[0][1] == [42, 43] and res[1][1] == [42, 43]
    # the reference arm runs on rank 0 only; other ranks return nothing
    assert res[1][2] is None


def test_single_rank_needs_no_process_group():
    bench = _load_bench()
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.replica_seed(0) == 42


def _worker_rank_dies(rank, world, port, out):
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    if rank == 1:
        # a replica that fails between steps: it leaves without joining the timing reduction
        dist.destroy_process_group()
        out[rank] = "left"
        return
    bench = _load_bench()
    t0 = time.time()
    try:
        bench.max_over_ranks(10.0, world)
        out[rank] = ("no error", time.time() - t0)
    except Exception as e:  # the surviving rank learns of the failure instead of waiting for good
        out[rank] = (type(e).__name__, time.time() - t0)
    finally:
        try:
            dist.destroy_process_group()
        except Exception:
            pass


def test_a_replica_that_leaves_ends_the_others_reduction_with_an_error():
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker_rank_dies, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[1] == "left"
    kind, waited = res[0]
    assert kind != "no error" and waited < 60, res
