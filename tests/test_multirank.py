"""bench.py's multi-process plumbing on CPU: two gloo ranks (127.0.0.1), one process per rank.

Sequences are independent, so ranks share no data: the only collectives are the barrier
around the timed region and the max-over-ranks of the step time.  Each rank draws its own
sequences (workload seed = rank), so the job's units are world x B x layers.
"""
import multiprocessing as mp
import os
import socket

import pytest


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    from workloads import configs as W
    w, r, _ = bench.dist_setup(None)
    bench.barrier(w)
    step_ms = bench.max_over_ranks(1.5 * (r + 1), w)
    spec = W.scaled(W.CONFIGS["hier1m"](seed=r), 64, B=1)
    _, ix = W.token_latents(spec, 0)
    out.put((r, w, step_ms, float(ix.float().sum())))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_time_max_and_draw_their_own_sequences():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [x[0] for x in res] == [0, 1] and all(x[1] == 2 for x in res)
    assert all(x[2] == pytest.approx(3.0) for x in res)          # max over ranks, seen by every rank
    assert res[0][3] != res[1][3]                                 # rank-seeded sequences differ
