"""The indexer's partial RoPE (QSA_INDEX_ROPE) on the GPU against the oracle.

Section 6 of the reading notes pools the keys first and applies a partial RoPE
afterwards; the pages give no dims, base or position, so the readings are the
oracle's (first rope_dims dims in pairs (i, i + rope_dims/2), angle pos *
base^(-2i / rope_dims), a pooled key at its block's first position b r, a query
at t).  Bars:
  compressor   |hi + lo - o| <= 2e-5 |o| + 1e-6 (the compensated pair, as without RoPE)
  queries      bf16 round-to-nearest of the fp32 rotation: |g - o| <= 2^-8 |o| + 1e-6
  scores       the indexer on the GPU-rotated queries and keys, against the oracle's
               scores of the same bf16 queries and its own rotated keys: the usual
               1e-2 max(|o|, s*_t) bar, and the fused selection equals the plain one
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import check_scores

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


def rope_cfg(qsa, dims=64, base=10000.0, **kw):
    return qsa.default_config(flags=qsa.QSA_INDEX_ROPE, rope_dims=dims, rope_base=base, **kw)


@pytest.mark.parametrize("lengths,dims,base", [([1000, 37, 5000, 3], 64, 10000.0), ([262144], 64, 10000.0),
                                               ([4096, 777], 128, 1.0e6), ([2048], 8, 500.0)])
def test_compress_rope_matches_oracle(qsa, lengths, dims, base):
    g = torch.Generator().manual_seed(71)
    k_idx = torch.randn((sum(lengths), 128), generator=g).to(torch.bfloat16)
    cu_k, cu_b = cu(lengths)
    cfg = rope_cfg(qsa, dims, base)
    kc = qsa.compress_keys(k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1), cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    got = kc[:int(cu_b[-1])].float().cpu().double().numpy()
    got = got[:, 0, :] + got[:, 1, :]
    a = 0
    for s, L in enumerate(lengths):
        ref = oracle.compress(k_idx[a:a + L], 4, rope_dims=dims, rope_base=float(np.float32(base)))
        g_s = got[int(cu_b[s]):int(cu_b[s + 1])]
        assert g_s.shape == ref.shape
        assert np.all(np.abs(g_s - ref) <= 2e-5 * np.abs(ref) + 1e-6), np.abs(g_s - ref).max()
        a += L
    # without the flag nothing rotates
    plain = qsa.compress_keys(k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1))
    assert not torch.equal(plain[:int(cu_b[-1])], kc[:int(cu_b[-1])]) or dims == 0


def test_paged_compress_rope_equals_packed(qsa):
    lengths, page = [3000, 1024, 77], 64
    g = torch.Generator().manual_seed(72)
    k_idx = torch.randn((sum(lengths), 128), generator=g).to(torch.bfloat16)
    cu_k, cu_b = cu(lengths)
    cfg = rope_cfg(qsa)
    kc = qsa.compress_keys(k_idx.cuda(), cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg).cpu()
    npg = [(L + page - 1) // page for L in lengths]
    perm = torch.randperm(sum(npg), generator=g)
    table = torch.full((len(lengths), max(npg)), -1, dtype=torch.int32)
    k_pages = torch.zeros((sum(npg), page, 128), dtype=torch.bfloat16)
    p0, t0 = 0, 0
    for s, L in enumerate(lengths):
        for j in range(npg[s]):
            n = min(page, L - j * page)
            pid = int(perm[p0 + j])
            k_pages[pid, :n] = k_idx[t0 + j * page:t0 + j * page + n]
            table[s, j] = pid
        p0 += npg[s]
        t0 += L
    kc_pages = torch.zeros((sum(npg), page // 4, 2, 128), dtype=torch.bfloat16, device="cuda")
    qsa.compress_keys_paged(k_pages.cuda(), kc_pages, table.cuda(), cu_k, max(lengths), cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    kp = kc_pages.cpu()
    for s, L in enumerate(lengths):
        for b in range(L // 4):
            pid, row = int(table[s, (b * 4) // page]), ((b * 4) % page) // 4
            assert torch.equal(kp[pid, row], kc[int(cu_b[s]) + b]), (s, b)


@pytest.mark.parametrize("lq,lk", [([5000, 9, 300], [5000, 9, 300]), ([1, 1, 1], [131072, 7, 262144])])
def test_rope_queries_match_oracle(qsa, lq, lk):
    g = torch.Generator().manual_seed(73)
    q = torch.randn((sum(lq), 4, 128), generator=g).to(torch.bfloat16)
    cu_q, _ = cu(lq)
    cu_k, _ = cu(lk)
    cfg = rope_cfg(qsa)
    qg = q.cuda()
    qsa.rope_queries(qg, cu_q, cu_k, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    got = qg.cpu().double().numpy()
    pos = np.concatenate([np.arange(a) + (b - a) for a, b in zip(lq, lk)])
    ref = oracle.rope(q.double().numpy(), np.repeat(pos, 4), 64, 10000.0)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6), np.abs(got - ref).max()
    np.testing.assert_array_equal(got[..., 64:], q.double().numpy()[..., 64:])


def test_rope_queries_need_the_flag(qsa):
    q = torch.zeros((4, 4, 128), dtype=torch.bfloat16, device="cuda")
    cu_q = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    with pytest.raises(qsa.QSAError):
        qsa.rope_queries(q, cu_q, cu_q)


@pytest.mark.parametrize("lengths,k", [([8192], 512), ([3000, 1200], 64)])
def test_indexer_chain_with_rope(qsa, lengths, k):
    x = inputs.make_prefill(lengths, seed=74)
    cu_k, cu_b = cu(lengths)
    cfg = rope_cfg(qsa, budget_blocks=k)
    kc = qsa.compress_keys(x.k_idx.cuda(), cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    q_rot = x.q_idx.cuda()
    qsa.rope_queries(q_rot, cu_k, cu_k, cfg=cfg)
    max_len = max(lengths)
    ld = max(4, ((max_len - 1) // 4 + 3) // 4 * 4)
    total = sum(lengths)
    scores = qsa.index_scores(q_rot, x.w.cuda(), kc, cu_k, cu_k, cu_b, max_len, ld, cfg=cfg)
    sel_m = qsa.select_blocks(scores, cu_k, cu_k, total, cfg=cfg)
    sel_f = qsa.index_select(q_rot, x.w.cuda(), kc, cu_k, cu_k, cu_b, max_len, max_len, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    assert torch.equal(sel_f, sel_m)
    q_rot_h = q_rot.cpu()
    sc = scores.cpu().numpy()
    a = 0
    for L in lengths:
        kc_ref = oracle.compress(x.k_idx[a:a + L], 4, rope_dims=64, rope_base=10000.0)
        rows = np.unique(np.concatenate([np.arange(min(64, L)), np.arange(max(0, L - 64), L),
                                         np.random.default_rng(L).integers(0, L, 64)]))
        ref = oracle.index_scores(q_rot_h[a:a + L], x.w[a:a + L], kc_ref, L, L, 4, rows=rows, ld=ld)
        bt = rows // 4
        check_scores(sc[a + rows], ref, bt, k)
        a += L
