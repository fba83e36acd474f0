"""N > 1 replicas on CPU (gloo, world size 2).

The decode path has no data-path collective: each rank decodes its own replica.  What
spans ranks is the bench's timing: the job's time is the slowest rank's (a MAX all-reduce)
and its rate counts every rank's bytes.  Two processes with different local times must
both report the slower time and the whole-job rate."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_module", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _load_bench()
        local_ms = [3.0, 5.0][rank]
        ms, gbs = bench.job_rate(local_ms, 1_000_000, 10, world, "cpu")
        dist.barrier()
        out[rank] = (ms, gbs)
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_replicas_report_the_slowest_rank_and_all_bytes():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for ms, gbs in res.values():
        assert ms == 5.0
        assert gbs == pytest.approx(world * 1_000_000 * 10 / 5e-3 / 1e9)


def test_single_rank_needs_no_process_group():
    bench = _load_bench()
    ms, gbs = bench.job_rate(4.0, 2_000_000, 5, 1, "cpu")
    assert ms == 4.0 and gbs == pytest.approx(2_000_000 * 5 / 4e-3 / 1e9)
