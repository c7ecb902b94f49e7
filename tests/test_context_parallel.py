"""Context-parallel decode (block_sparse_long_09_b200.context_parallel) on gloo ranks on
the CPU.

Each rank holds a block range of every sequence's caches.  It scores its own candidate
blocks into its columns of zero rows, the ranks sum the rows (all-reduce), every rank
selects on the full rows, attends its own selected blocks, and the partial softmax
states are all-gathered and merged.  The arithmetic here is the fp64 oracle's, so the
test checks the partition, the score placement, the collectives and the merge: the
selection must equal the unsharded one exactly and the output to within rounding.  The
same steps run the library's kernels on GPUs (tests/test_gpu_context_parallel.py
emulates the ranks on one GPU).
"""
import os
import socket
import traceback

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

K, CHUNK, SCALE = 16, 24, 1.0 / 16.0


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def merge(o_parts, lse_parts):
    """The merge of partial softmax states: lse = log sum exp lse_p, o = sum exp(lse_p - lse) o_p."""
    lse = np.logaddexp.reduce(lse_parts, axis=0)
    w = np.where(np.isneginf(lse_parts), 0.0, np.exp(lse_parts - np.where(np.isneginf(lse), 0.0, lse)[None]))
    return (w[..., None] * o_parts).sum(axis=0), lse


def _worker(rank, world, port, q):
    try:
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                          WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
        import torch.distributed as dist

        import oracle
        from block_sparse_long_09_b200 import inputs, ranks
        from block_sparse_long_09_b200.context_parallel import index_lengths, score_columns, shard_of
        assert ranks.init("gloo", world, timeout_s=60)
        d = inputs.make_decode(5, 40, 700, seed=81)
        lengths = d.seqlens
        sh = shard_of(lengths, rank, world, CHUNK)
        ld = score_columns(lengths)
        mine = torch.zeros((len(lengths), ld), dtype=torch.float64)
        lk = index_lengths(sh)
        t0 = 0
        for s, L in enumerate(lengths):
            lo, hi, n = sh.tok_lo[s], sh.tok_hi[s], sh.n_cand[s]
            if n > 0:  # this rank's candidate blocks, scored from its own compressed keys
                kc = oracle.compress(d.k_idx[t0 + lo:t0 + hi], 4)
                assert kc.shape[0] == sh.n_kc[s] == lk[s] // 4 and (lk[s] - 1) // 4 == n
                sc = oracle.index_scores(d.q_idx[s:s + 1], d.w[s:s + 1], kc, 1, lk[s], 4, ld=n)
                mine[s, sh.blk_lo[s]:sh.blk_lo[s] + n] = torch.from_numpy(sc[0])
            t0 += L
        dist.all_reduce(mine)
        full = mine.numpy()
        bt = np.array([(L - 1) // 4 for L in lengths])
        sel = oracle.select(full, bt, K)
        # partial attention over this rank's own selected blocks
        o_p = np.zeros((len(lengths), 24, 256))
        l_p = np.full((len(lengths), 24), -np.inf)
        t0 = 0
        for s, L in enumerate(lengths):
            lo, hi = sh.tok_lo[s], sh.tok_hi[s]
            ids = sel[s][(sel[s] >= sh.blk_lo[s]) & (sel[s] < sh.blk_hi[s])] - sh.blk_lo[s]
            if ids.size:
                row = np.full((1, K), -1, dtype=np.int32)
                row[0, :ids.size] = ids
                o, lse = oracle.attend(d.q[s:s + 1], d.k_cache[t0 + lo:t0 + hi], d.v_cache[t0 + lo:t0 + hi], row, 1,
                                       hi - lo, 4, SCALE)
                o_p[s], l_p[s] = o[0], lse[0]
            t0 += L
        o_all = [torch.zeros_like(torch.from_numpy(o_p)) for _ in range(world)]
        l_all = [torch.zeros_like(torch.from_numpy(l_p)) for _ in range(world)]
        dist.all_gather(o_all, torch.from_numpy(o_p))
        dist.all_gather(l_all, torch.from_numpy(l_p))
        o, lse = merge(np.stack([x.numpy() for x in o_all]), np.stack([x.numpy() for x in l_all]))
        q.put((rank, sel, o, lse, full))
        ranks.finish(world)
    except Exception:  # report instead of leaving the other ranks waiting
        q.put(("error", rank, traceback.format_exc(), None, None))


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_decode_equals_unsharded(world):
    import oracle
    from block_sparse_long_09_b200 import inputs
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    errors = [r for r in results if r[0] == "error"]
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs)
    d = inputs.make_decode(5, 40, 700, seed=81)
    t0 = 0
    for s, L in enumerate(d.seqlens):
        ref = oracle.qsa_layer(d.q[s:s + 1], d.k_cache[t0:t0 + L], d.v_cache[t0:t0 + L], d.q_idx[s:s + 1],
                               d.k_idx[t0:t0 + L], d.w[s:s + 1], 1, L, 4, K)
        bt = (L - 1) // 4
        for rank, sel, o, lse, full in results:
            np.testing.assert_array_equal(full[s, :bt], ref["scores"][0, :bt])   # the summed rows
            np.testing.assert_array_equal(sel[s], ref["sel"][0])                # the one-rank selection
            np.testing.assert_allclose(o[s], ref["o"][0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[s], ref["lse"][0], rtol=0, atol=1e-12)
        t0 += L


def test_shards_partition_tokens_blocks_and_candidates():
    from block_sparse_long_09_b200.context_parallel import index_lengths, shard_of
    rng = np.random.default_rng(82)
    for world, chunk in [(1, 8), (2, 8), (3, 24), (4, 4), (8, 64)]:
        lengths = [int(x) for x in rng.integers(1, 3000, 7)] + [1, 4, 5, 8 * chunk * 4, 8 * chunk * 4 + 1]
        shards = [shard_of(lengths, j, world, chunk) for j in range(world)]
        for sh in shards:  # the indexer's lengths: own block n, complete blocks = the shard's
            for Lv, n, nkc in zip(index_lengths(sh), sh.n_cand, sh.n_kc):
                assert (Lv - 1) // 4 == n and Lv // 4 == nkc
        for s, L in enumerate(lengths):
            bt = (L - 1) // 4
            toks, blocks, cands, kcs = [], [], [], []
            for sh in shards:
                toks += list(range(sh.tok_lo[s], sh.tok_hi[s]))
                blocks += list(range(sh.blk_lo[s], sh.blk_hi[s]))
                cands += list(range(sh.blk_lo[s], sh.blk_lo[s] + sh.n_cand[s]))
                kcs += list(range(sh.blk_lo[s], sh.blk_lo[s] + sh.n_kc[s]))
                assert sh.tok_lo[s] % 4 == 0 or sh.tok_lo[s] == L
                # a rank attends only blocks whose tokens it holds
                if sh.blk_hi[s] > sh.blk_lo[s]:
                    assert sh.blk_lo[s] * 4 >= sh.tok_lo[s] and (sh.blk_hi[s] - 1) * 4 < sh.tok_hi[s]
            assert toks == list(range(L))                  # every token exactly once, in order
            assert blocks == list(range(bt + 1))           # every attendable block exactly once
            assert cands == list(range(bt))                # every candidate block exactly once
            assert kcs == list(range(L // 4))              # every complete block compressed once
