"""Multi-rank plumbing of bench.py on CPU: two gloo ranks as independent replicas.

The decode path has no exchange step, so N GPUs run N independent replicas; the only
cross-rank work is the barrier and the max/sum reductions that turn per-rank bytes and
times into the whole-job number, and the reference arm running on rank 0 only.  These
run here as world_size-2 gloo process groups on 127.0.0.1.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, local = bench.dist_setup(ws)
    assert (r, w, local) == (rank, ws, rank)
    assert dist.get_backend() == "gloo"
    bench.barrier(w)
    # rank r processed (r+1) GB in (r+1) ms: 3 GB over the slowest rank's 2 ms
    gbs, ms_max = bench.job_gbs((rank + 1) * 1e9, float(rank + 1), w)
    out[rank] = (bench.max_over_ranks(rank + 0.5, w), bench.sum_over_ranks(rank + 1.0, w),
                 gbs, ms_max)
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_replicas_aggregate():
    ws = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_rank_main, args=(ws, _free_port(), out), nprocs=ws,
                           start_method="spawn", join=True)
        got = dict(out)
    for rank in range(ws):
        mx, sm, gbs, ms_max = got[rank]
        assert mx == 1.5 and sm == 3.0
        assert ms_max == 2.0
        assert gbs == pytest.approx(3e9 / 2e-3 / 1e9)


def _reference_rank(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        warmup, steps, gpus = 0, 0, ws

    # ranks other than 0 return at once without work; rank 0 would time the oracle
    if rank != 0:
        bench.run_reference(Args, rank, ws)
        out[rank] = "returned"
    else:
        out[rank] = "skipped"


def test_reference_arm_runs_on_rank_zero_only():
    ws = 2
    with mp.Manager() as m:
        out = m.dict()
        mp.start_processes(_reference_rank, args=(ws, _free_port(), out), nprocs=ws,
                           start_method="spawn", join=True)
        assert dict(out) == {0: "skipped", 1: "returned"}
