"""Query-row sharding of one prefill (block_sparse_long_09_b200.sharded) on two
gloo ranks on the CPU.

Each rank holds a contiguous shard of the rows; it compresses the blocks of its
own rows, the ranks all-gather the compressed keys and K/V, and each rank
computes its rows as L_q = shard queries against L_k = the prefix up to the
shard's end.  The arithmetic here is the fp64 oracle's, so the test checks the
partition, the gathers and the position offsets: the shards' results must equal
the unsharded computation exactly.  The same steps run the library's kernels on
GPUs (tests/test_gpu_sharded.py emulates the ranks on one GPU).
"""
import os
import socket
import traceback

import numpy as np
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, n, k, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        import oracle
        from block_sparse_long_09_b200 import inputs, ranks
        from block_sparse_long_09_b200.sharded import gather_rows, row_partition
        assert ranks.init("gloo", world, timeout_s=60)
        x = inputs.make_prefill([n], seed=52)
        parts = row_partition(n, world)
        a, b = parts[rank]
        # 1. this rank's compressed keys (its shard starts at a multiple of r)
        assert a % 4 == 0
        kc_loc = torch.from_numpy(oracle.compress(x.k_idx[a:b], 4))
        # 2. the all-gathers
        kc = gather_rows(kc_loc, [(bb - aa) // 4 for aa, bb in parts], world).numpy()
        sizes = [bb - aa for aa, bb in parts]
        k_all = gather_rows(x.k[a:b], sizes, world)
        v_all = gather_rows(x.v[a:b], sizes, world)
        assert torch.equal(k_all.view(torch.int16), x.k.view(torch.int16))
        # 3. this rank's rows: L_q = b - a queries against L_k = b keys
        Lq, Lk = b - a, b
        out = {}
        if Lq > 0:
            sc = oracle.index_scores(x.q_idx[a:b], x.w[a:b], kc[: Lk // 4], Lq, Lk, 4, ld=max(1, (Lk - 1) // 4))
            sel = oracle.select(sc, oracle.own_blocks(Lq, Lk, 4, None), k)
            o, lse = oracle.attend(x.q[a:b], k_all[:Lk], v_all[:Lk], sel, Lq, Lk, 4, 1.0 / 16.0)
            out = {"o": o, "sel": sel, "kc": kc}
        q.put((rank, a, b, out))
        ranks.finish(world)
    except Exception:  # report instead of leaving the other rank waiting
        q.put(("error", rank, traceback.format_exc(), None))


def test_two_rank_sharded_prefill_equals_unsharded():
    import oracle
    from block_sparse_long_09_b200 import inputs
    n, k, world = 600, 16, 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, n, k, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    errors = [r for r in results if r[0] == "error"]
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs)
    results.sort(key=lambda t: t[0])
    x = inputs.make_prefill([n], seed=52)
    ref = oracle.qsa_layer(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, 4, k)
    covered = np.zeros(n, dtype=int)
    for rank, a, b, out in results:
        covered[a:b] += 1
        if b > a:
            np.testing.assert_array_equal(out["kc"], ref["kc"])
            np.testing.assert_array_equal(out["sel"], ref["sel"][a:b])
            np.testing.assert_array_equal(out["o"], ref["o"][a:b])
    assert np.all(covered == 1)


def test_row_partition_balances_and_aligns():
    from block_sparse_long_09_b200.sharded import ATTN_ROW_COST, INDEX_PAIR_COST, row_partition

    def cost(a, b):
        t = np.arange(a, b)
        return float((ATTN_ROW_COST + INDEX_PAIR_COST * (t // 4)).sum())

    for n, world in [(262144, 8), (262144, 2), (20000, 3), (4097, 4), (10, 4), (0, 2), (7, 1)]:
        parts = row_partition(n, world)
        assert len(parts) == world and parts[0][0] == 0 and parts[-1][1] == n
        for (a, b), (c, d) in zip(parts, parts[1:]):
            assert b == c
        assert all(a % 4 == 0 and a <= b for a, b in parts)
        if n >= 4096 * world:
            costs = [cost(a, b) for a, b in parts]
            assert max(costs) <= 1.01 * min(costs), costs  # balanced to within a block of rows
    # later rows cost more: with the indexer's share, the last rank gets the fewest rows
    parts = row_partition(262144, 8)
    sizes = [b - a for a, b in parts]
    assert sizes == sorted(sizes, reverse=True)
