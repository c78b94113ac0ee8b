"""Host logic of the multi-GPU benchmark with two gloo ranks on the CPU.

Every rank decodes its own batch (weak scaling; no collective on the data
path). The only exchanges are the barrier and the max of the per-rank times;
the whole-job throughput counts all ranks' sequences over the slowest rank's
time. Rank 0 alone runs the CPU oracle leg of ``--impl reference``.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w, r, lr = bench.rank_env()
        mine = [10.0 + rank, 5.0 - rank, 7.0 * (rank + 1)]
        dist.barrier()
        got = bench.max_over_ranks(mine, dist)
        tput = bench.job_throughput(w, 1024, 100, got[0])

        class A:
            steps, warmup, gpus, seed = 2, 1, world, 0
            config = "tiny"

        class AP(A):
            config = "prefill_tiny"

        class AN(A):
            config = "norm_tiny"

        # the oracle legs (decode, prefill, add + RMSNorm) run on rank 0 alone:
        # every other rank returns at once
        ref_rc = None
        if rank != 0:
            ref_rc = (bench.run_reference(A), bench.run_prefill_reference(AP), bench.run_norm_reference(AN))
        q.put((rank, w, r, lr, got, tput, ref_rc))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_take_the_max_and_count_all_sequences():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, w, r, lr, got, tput, ref_rc in res:
        assert (w, r, lr) == (2, rank, rank)
        assert got == [11.0, 5.0, 14.0]  # element-wise max over the two ranks
        assert tput == pytest.approx(2 * 1024 * 100 / 11.0e-3)
    assert res[1][6] == (0, 0, 0)  # rank 1 skips every oracle leg


def test_single_process_is_the_identity():
    import sys

    sys.path.insert(0, ROOT)
    import bench

    assert bench.max_over_ranks([1.5, 2.5]) == [1.5, 2.5]
    assert bench.job_throughput(1, 1024, 10, 10.0) == pytest.approx(1024 * 10 / 0.01)
