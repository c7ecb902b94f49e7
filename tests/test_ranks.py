"""Two gloo ranks on CPU: the multi-rank plumbing that bench.py uses for N GPUs.

Each rank draws its own problem (distinct seeds), the ranks meet at barriers,
the timing is the element-wise max over ranks, and the job's throughput counts
every rank's units over the slowest rank's time.  Nothing here needs a GPU.
"""
import os
import socket
import traceback

import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        from block_sparse_long_09_b200 import inputs, ranks
        env = ranks.env_ranks()
        assert (env["rank"], env["world"]) == (rank, world)
        assert ranks.init("gloo", env["world"], timeout_s=60)
        seeds = ranks.rank_seeds(rank)
        x = inputs.make_prefill([64], seed=seeds["prefill"])
        d = inputs.make_decode(2, 40, 60, seed=seeds["decode"])
        own_ms = [5.0 + 2.0 * rank, 3.0 - rank]  # rank 1 is slower on the first, faster on the second
        ranks.barrier(world)
        mx = ranks.max_over_ranks(own_ms, world)
        thr = ranks.job_throughput(world, 64, mx[0])
        q.put((rank, float(x.q.float().sum()), float(d.q.float().sum()), mx, thr))
        ranks.finish(world)
    except Exception:  # report instead of leaving the other rank waiting
        q.put(("error", rank, traceback.format_exc()))


def test_two_gloo_ranks_max_timing_and_distinct_problems():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=180) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    errors = [r for r in results if r[0] == "error"]
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs)
    results.sort()
    (_, xq0, dq0, mx0, thr0), (_, xq1, dq1, mx1, thr1) = results
    assert mx0 == mx1 == [7.0, 3.0]
    assert thr0 == thr1 == 2 * 64 / 7e-3
    assert xq0 != xq1 and dq0 != dq1  # every rank runs its own problem


def test_single_process_needs_no_group():
    from block_sparse_long_09_b200 import ranks
    assert not ranks.init("gloo", 1)
    assert ranks.max_over_ranks([1.5, 2.5], 1) == [1.5, 2.5]
    assert ranks.job_throughput(1, 1000, 500.0) == 2000.0
