"""Query-row sharding of one prefill through the library's kernels, with the ranks
emulated one after another in this process on one GPU (no rank waits for
another: the gathers are concatenations done between the ranks' steps).

Every row's scores, selection and attention depend only on the row and on the
prefix it sees, so the shards' outputs must equal the one-process prefill bit
for bit.
"""
import pytest
import torch

from block_sparse_long_09_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_long_09_b200 import build
    build.build()
    from block_sparse_long_09_b200 import qsa as q
    assert torch.cuda.is_available()
    q.device_status(clear=True)
    return q


@pytest.mark.parametrize("n,world,k", [(20000, 3, 512), (9001, 2, 64), (70000, 4, 512)])
def test_sharded_prefill_equals_one_process(qsa, n, world, k):
    from block_sparse_long_09_b200.sharded import ShardedPrefill, row_partition
    x = inputs.make_prefill([n], seed=51, device="cuda")
    cfg = qsa.default_config(budget_blocks=k)
    o_ref = qsa.Prefill([n], cfg=cfg, device="cuda")(x.q, x.k, x.v, x.q_idx, x.w, x.k_idx)
    parts = row_partition(n, world)
    shards = [ShardedPrefill(n, j, world, chunk_rows=8192, cfg=cfg, parts=parts) for j in range(world)]
    # step 1 on every rank; step 2 (the all-gathers) as concatenations
    kc_all = torch.cat([sh.local_blocks(x.k_idx[a:b].contiguous()) for sh, (a, b) in zip(shards, parts)])
    o = torch.empty_like(x.q)
    for sh, (a, b) in zip(shards, parts):  # step 3, rank by rank
        o[a:b] = sh.attend(x.q[a:b].contiguous(), x.q_idx[a:b].contiguous(), x.w[a:b].contiguous(), kc_all,
                           x.k, x.v)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    assert torch.equal(o, o_ref)
