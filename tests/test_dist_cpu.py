"""The benchmark's multi-process plumbing on the CPU: two ranks over gloo
(127.0.0.1), as `torchrun --nproc-per-node 2 bench.py` would start them.

Decode shards by sequence, so each rank runs its own replica of the layer
group and the only collective is the max-over-ranks of the step time; these
tests check that reduction, the barrier, the environment parsing and the
reference arm's rank-0-only rule."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_env()
    bench.dist_init(w, "gloo")
    bench.barrier(w)
    got = bench.reduce_max(10.0 * (rank + 1), w)
    # the reference arm: only rank 0 produces a line; the others do no work
    import argparse
    args = argparse.Namespace(seed=0, steps=1, warmup=3)
    from kv_cache_csa2_b200.configs import C1
    res = bench.run_reference(args, C1.replace(L=1024, compress_new_tokens=1024, k=64), w, r)
    bench.barrier(w)
    import torch.distributed as dist
    dist.destroy_process_group()
    out.put((r, local, got, None if res is None else (res["impl"], res["n_gpus"], res["unit"])))


@pytest.mark.timeout(300)
def test_two_ranks_over_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [r[0] for r in res] == [0, 1] and [r[1] for r in res] == [0, 1]
    assert all(r[2] == 20.0 for r in res)                   # max over ranks
    assert res[0][3] == ("reference", 2, bench.UNIT)        # rank 0 reports
    assert res[1][3] is None                                # rank 1 does no work


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(3.5, 1) == 3.5
    bench.barrier(1)
    os.environ.pop("WORLD_SIZE", None)
    assert bench.dist_env()[0] == 1
