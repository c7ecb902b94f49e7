"""The fused index -> select path (qsa_index_select) against the materialised one
(qsa_index_scores, then qsa_select_blocks), through the C ABI.

Both paths compute the indexer scores with the same tensor-core kernel and the
same epilogue arithmetic, and both take the exact top-k, so their selections
must agree bit for bit on every row (the fused path keeps only the candidates
above a sampled lower bound of the k-th score, and proves per row that nothing
above the true threshold was dropped).  A row whose candidate list cannot prove
it (too few entries, or an overflow) is recomputed on CUDA cores: that path is
forced here with keys whose scores are exact in fp32 on both sides, so the
selections must again agree bit for bit, and match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import check_selection_invariants

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


def both_paths(qsa, q_idx, w, kc, lengths, k, chunk):
    cfg = qsa.default_config(budget_blocks=k)
    cu_k, cu_b = cu(lengths)
    total = sum(lengths)
    max_len = max(lengths)
    ld = max(4, ((max_len - 1) // 4 + 3) // 4 * 4)
    sel_m = torch.full((total, k), -7, dtype=torch.int32, device="cuda")
    sel_f = torch.full((total, k), -7, dtype=torch.int32, device="cuda")
    scores = torch.empty((min(chunk, total), ld), dtype=torch.float32, device="cuda")
    for r0 in range(0, total, chunk):
        r1 = min(total, r0 + chunk)
        qsa.index_scores(q_idx, w, kc, cu_k, cu_k, cu_b, max_len, ld, r0, r1, scores=scores, cfg=cfg)
        qsa.select_blocks(scores, cu_k, cu_k, total, r0, r1, sel=sel_m, cfg=cfg)
        qsa.index_select(q_idx, w, kc, cu_k, cu_k, cu_b, max_len, max_len, r0, r1, sel=sel_f, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    return sel_m.cpu().numpy(), sel_f.cpu().numpy()


@pytest.mark.parametrize("lengths,k,chunk", [([8192], 512, 16384), ([8192], 512, 3000), ([65536], 512, 16384),
                                             ([5000, 70, 3000], 64, 1000), ([1000, 3000], 16, 777),
                                             ([1, 3, 4, 5, 37, 130, 701, 2], 16, 16384), ([20000], 2048, 8192),
                                             ([40000, 9000], 512, 16384)])
def test_index_select_equals_materialised(qsa, lengths, k, chunk):
    x = inputs.make_prefill(lengths, seed=41, device="cuda")
    cu_k, cu_b = cu(lengths)
    kc = qsa.compress_keys(x.k_idx, cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1))
    sel_m, sel_f = both_paths(qsa, x.q_idx, x.w, kc, lengths, k, chunk)
    np.testing.assert_array_equal(sel_f, sel_m)
    bt = np.concatenate([np.arange(L) // 4 for L in lengths])
    check_selection_invariants(sel_f, bt, k)


def test_index_select_peaked(qsa):
    """Peaked indexer keys (one N(0, 0.5^2) offset per block): many rows share their
    best blocks."""
    lengths = [32768, 32768]
    x = inputs.make_prefill(lengths, seed=42, peaked=True, device="cuda")
    cu_k, cu_b = cu(lengths)
    kc = qsa.compress_keys(x.k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]))
    sel_m, sel_f = both_paths(qsa, x.q_idx, x.w, kc, lengths, 512, 16384)
    np.testing.assert_array_equal(sel_f, sel_m)


def test_index_select_fallback_rows(qsa):
    """Keys chosen so that the sampled bound is too high: only blocks of the sampled
    tiles 0 and 16 (blocks 0..127 and 2048..2175) score high, so a row with many
    candidates finds fewer than k - 1 blocks above its bound and is recomputed on
    CUDA cores.  Every key is a multiple of 1/16 in [-1/8, 1/8] (or exactly 1) and the
    query is all ones on one head, so every score is exact in fp32 on both paths."""
    L, k = 24000, 512
    g = torch.Generator().manual_seed(43)
    nb = L // 4
    kc = (torch.randint(-2, 3, (nb, 128), generator=g).float() / 16.0)
    hot = torch.zeros(nb, dtype=torch.bool)
    hot[0:128] = True
    hot[2048:2176] = True
    kc[hot] = 1.0
    kc = torch.stack([kc, torch.zeros_like(kc)], dim=1).to(torch.bfloat16).cuda()  # hi = the value, lo = 0
    q_idx = torch.zeros((L, 4, 128), dtype=torch.bfloat16)
    q_idx[:, 0, :] = 1.0
    w = torch.zeros((L, 4), dtype=torch.float32)
    w[:, 0] = 1.0
    q_idx, w = q_idx.cuda(), w.cuda()
    sel_m, sel_f = both_paths(qsa, q_idx, w, kc, [L], k, 16384)
    np.testing.assert_array_equal(sel_f, sel_m)
    # against the oracle on sampled rows (its scores are the same exact numbers)
    rows = np.r_[np.arange(0, L, 997), L - 1]
    sc = oracle.index_scores(q_idx.cpu(), w.cpu(), kc.double().sum(dim=1).cpu().numpy(), L, L, 4, rows, ld=nb)
    sel_o = oracle.select(sc, rows // 4, k)
    np.testing.assert_array_equal(sel_f[rows], sel_o)


def test_index_select_decode_rows(qsa):
    """One query per sequence (max_len_q = 1): the one-row scores go to the workspace."""
    d = inputs.make_decode(16, 300, 40000, seed=44, device="cuda")
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(17, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]))
    max_len = max(d.seqlens)
    ld = max(4, ((max_len - 1) // 4 + 3) // 4 * 4)
    sc = qsa.index_scores(d.q_idx, d.w, kc, cu_q, cu_k, cu_b, 1, ld)
    sel_m = qsa.select_blocks(sc, cu_q, cu_k, 16)
    sel_f = qsa.index_select(d.q_idx, d.w, kc, cu_q, cu_k, cu_b, 1, max_len)
    torch.cuda.synchronize()
    assert torch.equal(sel_f, sel_m)
    assert qsa.device_status(clear=True) == 0
