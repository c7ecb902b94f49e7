"""Decode with multi-token prediction: next_n queries per sequence share one
selection (qsa_index_select_mtp, qsa_sparse_attn_decode_mtp), through the C ABI,
against the fp64 oracle.

The selection is made from the scores of each sequence's last query with every
query's own block kept: bit-exact against the oracle's shared selection run on
the GPU's own exact scores, and within the near-threshold rule of the oracle's
selection on its own scores.  The attention of every (query, head) row over the
shared selection, cut to the row's tokens j <= t: max-abs <= 2e-2, mean-abs <= 1e-3
and lse within 2e-3 of the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import SCALE, bits, check_attn, check_selection_near_threshold

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


@pytest.mark.parametrize("batch,lo,hi,k,next_n", [(8, 300, 9000, 512, 4), (64, 16384, None, 512, 4),
                                                  (5, 4, 60, 16, 4), (6, 1000, 5000, 512, 2),
                                                  (3, 2000, 3000, 64, 3), (9, 100, 20000, 512, 1)])
def test_mtp_decode_step(qsa, batch, lo, hi, k, next_n):
    d = inputs.make_decode(batch, lo, hi, seed=61, next_n=next_n)
    cfg = qsa.default_config(budget_blocks=k)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1), cfg=cfg)
    max_len = max(d.seqlens)
    sel = qsa.index_select_mtp(d.q_idx.cuda(), d.w.cuda(), kc, cu_k, cu_b, next_n, max_len, cfg=cfg)
    q = d.q.cuda() if next_n > 1 else d.q.cuda()[:, None]
    o, lse = qsa.sparse_attn_decode_mtp(q, d.k_cache.cuda(), d.v_cache.cuda(), cu_k, sel, want_lse=True, cfg=cfg)
    # the exact GPU scores of each sequence's last query
    ld = max(4, ((max_len - 1) // 4 + 3) // 4 * 4)
    sc_g = qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc, cu_q, cu_k, cu_b, 1, ld, cfg=cfg)
    torch.cuda.synchronize()
    assert qsa.device_status(clear=True) == 0
    sel_g, sc_g = sel.cpu().numpy(), sc_g.cpu().numpy()
    o_g, lse_g = o.float().cpu().numpy(), lse.cpu().numpy()
    # bit-exact on the GPU's own scores (entries past each row's candidates are unspecified)
    sc64 = sc_g.astype(np.float64)
    for s, L in enumerate(d.seqlens):
        sc64[s, max(0, (L - 1) // 4):] = -np.inf
    np.testing.assert_array_equal(sel_g, oracle.select_shared(sc64, d.seqlens, next_n, k))
    cuh = cu_k.cpu().numpy()
    qh = d.q if next_n > 1 else d.q[:, None]
    for s, L in enumerate(d.seqlens):
        a, b = int(cuh[s]), int(cuh[s + 1])
        b_first = max(L - next_n, 0) // 4
        # against the oracle's own scores: only near-threshold blocks may differ
        kc_o = oracle.compress(bits(d.k_idx[a:b]), 4)
        sc_o = oracle.index_scores(d.q_idx[s:s + 1], d.w[s:s + 1], kc_o, 1, L, 4, [0], ld=ld)
        sel_o = oracle.select_shared(sc_o, [L], next_n, k)
        check_selection_near_threshold(sel_g[s:s + 1], sel_o, sc_o, [b_first], k - ((L - 1) // 4 - b_first))
        # every query of the step over the shared selection
        rows = list(range(next_n))
        ref_o, ref_lse = oracle.attend(qh[s], d.k_cache[a:b], d.v_cache[a:b], np.repeat(sel_g[s:s + 1], next_n, 0),
                                       next_n, L, 4, SCALE, rows)
        check_attn(o_g[s], ref_o)
        np.testing.assert_allclose(lse_g[s], ref_lse, rtol=0, atol=2e-3)


def test_mtp_next_n_1_selection_equals_decode(qsa):
    """next_n = 1 is the ordinary decode step: the same selection bit for bit."""
    d = inputs.make_decode(12, 500, 30000, seed=62)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(13, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=int(cu_b[-1]))
    max_len = max(d.seqlens)
    a = qsa.index_select_mtp(d.q_idx.cuda(), d.w.cuda(), kc, cu_k, cu_b, 1, max_len)
    b = qsa.index_select(d.q_idx.cuda(), d.w.cuda(), kc, cu_q, cu_k, cu_b, 1, max_len)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert qsa.device_status(clear=True) == 0


def test_mtp_step_cuda_graph(qsa):
    """qsa.MtpStep: the CUDA-graph replay of a multi-token step (compressed-block refresh,
    shared selection, attention) equals the same calls launched eagerly, bit for bit, and
    the refreshed blocks equal a full compression of the cache."""
    next_n = 4
    d = inputs.make_decode(6, 3000, 20000, seed=41, device="cuda", next_n=next_n)
    cu_k, cu_b = d.cu_seqlens_k, d.cu_blocks
    cfg = qsa.default_config()
    kc_full = qsa.compress_keys(d.k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    # the blocks the step's tokens touched start stale: the refresh must recompute them
    first = torch.tensor([(L - next_n) // 4 for L in d.seqlens], dtype=torch.int32, device="cuda")
    kcs = []
    for graph in (False, True):
        kc = kc_full.clone()
        for s in range(len(d.seqlens)):
            b0, nb = int(cu_b[s]), int(cu_b[s + 1]) - int(cu_b[s])
            lo = b0 + int(first[s])
            kc[lo:b0 + nb] = 0
        step = qsa.MtpStep(d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx, kc, cu_k, cu_b, max(d.seqlens),
                           refresh_blocks=first, cfg=cfg, graph=graph)
        for _ in range(2):
            o = step()
        torch.cuda.synchronize()
        kcs.append((kc, step.sel.clone(), o.clone()))
    assert torch.equal(kcs[0][0], kc_full) and torch.equal(kcs[1][0], kc_full)
    assert torch.equal(kcs[0][1], kcs[1][1])
    assert torch.equal(kcs[0][2], kcs[1][2])
    sel = qsa.index_select_mtp(d.q_idx, d.w, kc_full, cu_k, cu_b, next_n, max(d.seqlens), cfg=cfg)
    torch.cuda.synchronize()
    assert torch.equal(sel, kcs[0][1])
    assert qsa.device_status(clear=True) == 0


def test_mtp_selection_when_every_block_ties(qsa):
    """Every compressed key equal: the candidate list overflows, the row is selected from
    its exact scores in the same CTA, and the tie rule leaves a closed form: every query's
    own block (b_first .. b_last) forced, then the lowest blocks below b_first."""
    next_n, k = 4, 512
    lengths = [30002, 20001, 9, 2050]
    cfg = qsa.default_config(budget_blocks=k)
    g = torch.Generator(device="cuda")
    g.manual_seed(78)
    pat = torch.randn((4, 128), generator=g, device="cuda").to(torch.bfloat16)
    k_idx = torch.cat([pat.repeat((L + 3) // 4, 1)[:L] for L in lengths])
    q_idx = torch.randn((len(lengths), 4, 128), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.rand((len(lengths), 4), generator=g, device="cuda")
    cu_k, cu_b = cu(lengths)
    kc = qsa.compress_keys(k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    sel = qsa.index_select_mtp(q_idx, w, kc, cu_k, cu_b, next_n, max(lengths), cfg=cfg).cpu().numpy()
    for s, L in enumerate(lengths):
        b_first, b_last = max(L - next_n, 0) // 4, (L - 1) // 4
        nf = b_last - b_first + 1
        want = list(range(min(k - nf, b_first))) + list(range(b_first, b_first + nf))
        want += [-1] * (k - len(want))
        np.testing.assert_array_equal(sel[s], np.array(want, dtype=np.int32))
    assert qsa.device_status(clear=True) == 0
