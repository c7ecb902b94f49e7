"""Context-parallel decode on one GPU with the ranks emulated one after another
(block_sparse_long_09_b200.context_parallel): each emulated rank holds a block range of
every sequence's caches, scores its own candidates into its columns, the rows are summed
(the all-reduce), each rank attends its own selected blocks (qsa_sparse_attn_decode_window)
and qsa_merge_attn_states merges the partial states.  The selection must equal the
one-GPU selection bit for bit, the merged output the oracle on it (attention bar) and
the one-GPU decode output to within bf16 rounding of the partial outputs.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import SCALE, check_attn

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def qsa():
    from block_sparse_long_09_b200 import build
    build.build()
    from block_sparse_long_09_b200 import qsa as q
    assert torch.cuda.is_available()
    q.device_status(clear=True)
    return q


def cu(lengths, r=4):
    a, b = [0], [0]
    for L in lengths:
        a.append(a[-1] + L)
        b.append(b[-1] + L // r)
    return (torch.tensor(a, dtype=torch.int32, device="cuda"), torch.tensor(b, dtype=torch.int32, device="cuda"))


@pytest.mark.parametrize("batch,lo,hi,k,world,chunk", [(8, 300, 9000, 512, 2, 512), (6, 20000, 40000, 512, 4, 2048),
                                                       (5, 4, 900, 64, 3, 40), (3, 70000, 70000, 512, 8, 2048)])
def test_context_parallel_decode(qsa, batch, lo, hi, k, world, chunk):
    from block_sparse_long_09_b200.context_parallel import ContextParallelDecode, shard_of
    d = inputs.make_decode(batch, lo, hi, seed=83, device="cuda")
    cfg = qsa.default_config(budget_blocks=k)
    lengths = d.seqlens
    cu_k, cu_b = cu(lengths)
    # one GPU: exact scores, selection, attention
    kc = qsa.compress_keys(d.k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    ld = max(4, ((max(lengths) - 1) // 4 + 3) // 4 * 4)
    sc = qsa.index_scores(d.q_idx, d.w, kc, cu_q, cu_k, cu_b, 1, ld, cfg=cfg)
    sel1 = qsa.select_blocks(sc, cu_q, cu_k, batch, cfg=cfg)
    o1, lse1 = qsa.sparse_attn_decode(d.q, d.k_cache, d.v_cache, cu_k, sel1, want_lse=True, cfg=cfg)
    # the emulated ranks
    ranks = []
    for j in range(world):
        sh = shard_of(lengths, j, world, chunk)
        take = []
        t0 = 0
        for s, L in enumerate(lengths):
            take.append(torch.arange(t0 + sh.tok_lo[s], t0 + sh.tok_hi[s], device="cuda"))
            t0 += L
        idx = torch.cat(take)
        ranks.append(ContextParallelDecode(lengths, j, world, chunk, d.k_cache[idx].contiguous(),
                                           d.v_cache[idx].contiguous(), d.k_idx[idx].contiguous(), cfg=cfg))
    full = sum(rk.local_scores(d.q_idx, d.w).clone() for rk in ranks)  # the all-reduce
    parts = []
    for rk in ranks:
        sel = rk.select(full)
        assert torch.equal(sel, sel1)
        o, lse = rk.attend(d.q)
        parts.append((o.clone(), lse.clone()))
    o_m, lse_m = qsa.merge_attn_states(torch.stack([p[0] for p in parts]), torch.stack([p[1] for p in parts]),
                                       cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    # the scores each rank wrote are the one-GPU scores
    for s, L in enumerate(lengths):
        bt = (L - 1) // 4
        assert torch.equal(full[s, :bt], sc[s, :bt])
    og, lg = o_m.float().cpu().numpy(), lse_m.cpu().numpy()
    # against the one-GPU decode: bf16 partial outputs, then the merge
    assert np.abs(og - o1.float().cpu().numpy()).max() <= 2e-2
    np.testing.assert_allclose(lg, lse1.cpu().numpy(), rtol=0, atol=2e-3)
    # against the oracle on the (shared) selection
    t0 = 0
    sel_h = sel1.cpu().numpy()
    for s, L in enumerate(lengths):
        ref_o, ref_lse = oracle.attend(d.q[s:s + 1].cpu(), d.k_cache[t0:t0 + L].cpu(), d.v_cache[t0:t0 + L].cpu(),
                                       sel_h[s:s + 1], 1, L, 4, SCALE)
        check_attn(og[s:s + 1], ref_o)
        np.testing.assert_allclose(lg[s:s + 1], ref_lse, rtol=0, atol=2e-3)
        t0 += L


def test_merge_of_one_part_is_identity_and_empty_parts_count_for_nothing(qsa):
    g = torch.Generator(device="cuda").manual_seed(84)
    o = torch.randn((3, 24, 256), generator=g, device="cuda").to(torch.bfloat16)
    lse = torch.randn((3, 24), generator=g, device="cuda")
    m, l = qsa.merge_attn_states(o[None], lse[None])
    assert torch.equal(m, o) and torch.allclose(l, lse, atol=1e-6, rtol=0)
    empty_o = torch.zeros_like(o)
    empty_l = torch.full_like(lse, float("-inf"))
    m2, l2 = qsa.merge_attn_states(torch.stack([empty_o, o, empty_o]), torch.stack([empty_l, lse, empty_l]))
    assert torch.equal(m2, o) and torch.allclose(l2, lse, atol=1e-6, rtol=0)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
