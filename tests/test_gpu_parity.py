"""GPU (C ABI) vs fp64 oracle parity for every step of the QSA path.

Tolerances (fixed by the method's target bounds):
  scores     |g - o| <= 1e-2 * max(|o|, s*_t), s*_t = oracle's (k-1)-th best candidate score
  selection  bit-exact when both sides select on the same fp32 scores; on the GPU's own
             scores a block may differ only where the oracle's score is within 1e-2 of s*_t
  attention  max-abs <= 2e-2 and mean-abs <= 1e-3 against the oracle on the same selection
  compressor kc = hi + lo (compensated bf16 pair): |g - o| <= 2e-5 |o| + 1e-6
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import (SCALE, check_attn, check_scores, check_selection_invariants,
                           check_selection_near_threshold, kth_best,
                           sampled_rows)

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


def seq_slices(lengths):
    out, s = [], 0
    for L in lengths:
        out.append((s, s + L))
        s += L
    return out


def kc_value(kc):
    """hi + lo planes of the compressed keys, in fp64: [n_blocks, 128]."""
    assert kc.dtype == torch.bfloat16 and kc.dim() == 3
    return kc.double().sum(dim=1).cpu().numpy()


def status_ok(qsa):
    assert qsa.device_status(clear=True) == 0


# ---------------------------------------------------------------------------------------------
# compressor
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lengths", [[512], [1, 3, 4, 5, 37, 130, 701], [0, 9, 0, 4100]])
@pytest.mark.parametrize("normalise", [True, False])
def test_compress(qsa, lengths, normalise):
    x = inputs.make_prefill(lengths, seed=21)
    cu_k, cu_b = cu(lengths)
    cfg = qsa.default_config(flags=0 if normalise else qsa.QSA_COMPRESS_NO_NORM)
    nb = int(cu_b[-1])
    kc = qsa.compress_keys(x.k_idx.cuda(), cu_k, cu_b, cfg=cfg, n_blocks=nb)
    torch.cuda.synchronize()
    g = kc_value(kc)
    hi = kc[:, 0].double().cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(lengths)):
        ref = oracle.compress(x.k_idx[a:b], 4, normalise)
        got = g[int(cu_b[s]):int(cu_b[s + 1])]
        assert got.shape == ref.shape
        if ref.size:
            assert np.all(np.abs(got - ref) <= 2e-5 * np.abs(ref) + 1e-6)
            # the hi plane alone is the bf16 rounding of the value
            h = hi[int(cu_b[s]):int(cu_b[s + 1])]
            assert np.all(np.abs(h - ref) <= 2 ** -8 * np.abs(ref) + 1e-6)
    status_ok(qsa)


def test_compress_update_mode(qsa):
    lengths = [37, 4096, 129]
    x = inputs.make_prefill(lengths, seed=22)
    cu_k, cu_b = cu(lengths)
    k_idx = x.k_idx.cuda()
    full = qsa.compress_keys(k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]))
    part = torch.zeros_like(full)
    last = torch.tensor([L // 4 - 1 for L in lengths], dtype=torch.int32, device="cuda")
    qsa.compress_keys(k_idx, cu_k, cu_b, kc=part, blk_begin=last, max_new_blocks=2)
    torch.cuda.synchronize()
    for s in range(len(lengths)):
        row = int(cu_b[s + 1]) - 1
        assert torch.equal(part[row], full[row])
        if int(cu_b[s + 1]) - int(cu_b[s]) > 1:
            assert torch.count_nonzero(part[row - 1]) == 0
    status_ok(qsa)


# ---------------------------------------------------------------------------------------------
# indexer scores
# ---------------------------------------------------------------------------------------------

def gpu_scores(qsa, x, lengths, k, chunk=None, pad_ld=False):
    cu_k, cu_b = cu(lengths)
    total = sum(lengths)
    ld = max(1, (max(lengths) - 1) // 4)
    if pad_ld:
        ld = (ld + 3) // 4 * 4 + 4  # multiple of 4: whole-tile TMA stores
    kc = qsa.compress_keys(x.k_idx.cuda(), cu_k, cu_b, n_blocks=int(cu_b[-1]))
    q_idx, w = x.q_idx.cuda(), x.w.cuda()
    scores = torch.full((total, ld), float("nan"), dtype=torch.float32, device="cuda")
    chunk = chunk or total
    for r0 in range(0, total, chunk):
        r1 = min(total, r0 + chunk)
        qsa.index_scores(q_idx, w, kc, cu_k, cu_k, cu_b, max(lengths), ld, r0, r1, scores=scores[r0:r1])
    torch.cuda.synchronize()
    return kc, scores


@pytest.mark.parametrize("pad_ld", [False, True])
@pytest.mark.parametrize("lengths,chunk", [([512], None), ([1, 3, 4, 5, 37, 130, 701, 2], None),
                                           ([1000, 3000], 777), ([8192], 4096), ([5000, 70, 3000], 1000)])
def test_index_scores(qsa, lengths, chunk, pad_ld):
    k = 16 if max(lengths) <= 1024 else 512
    x = inputs.make_prefill(lengths, seed=23)
    kc, scores = gpu_scores(qsa, x, lengths, k, chunk, pad_ld)
    kc_g = kc_value(kc)
    sc = scores.cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(lengths)):
        L = b - a
        cb0 = sum(l // 4 for l in lengths[:s])
        rows = np.arange(L) if L <= 2048 else np.unique(np.r_[np.arange(64), np.arange(L - 64, L),
                                                                np.random.default_rng(0).integers(0, L, 256)])
        ref = oracle.index_scores(x.q_idx[a:b], x.w[a:b], kc_g[cb0:cb0 + L // 4], L, L, 4, rows,
                                  ld=sc.shape[1])
        bt = rows // 4
        g = sc[a + rows]
        check_scores(g, ref, bt, k)   # entries b >= b_t are unspecified
    status_ok(qsa)


def test_index_scores_decode_rows(qsa):
    """One query per sequence (the decode kernel) against caches of mixed length."""
    d = inputs.make_decode(6, 300, 9000, seed=24)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(len(d.seqlens) + 1, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=int(cu_b[-1]))
    ld = max(d.seqlens) // 4
    scores = torch.full((len(d.seqlens), ld), float("nan"), dtype=torch.float32, device="cuda")
    qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc, cu_q, cu_k, cu_b, 1, ld, scores=scores)
    torch.cuda.synchronize()
    kc_g, sc = kc_value(kc), scores.cpu().numpy()
    for s, L in enumerate(d.seqlens):
        cb0 = int(cu_b[s])
        ref = oracle.index_scores(d.q_idx[s:s + 1], d.w[s:s + 1], kc_g[cb0:cb0 + L // 4], 1, L, 4, [0], ld=ld)
        bt = (L - 1) // 4
        check_scores(sc[s:s + 1], ref, [bt], 512)
        assert np.all(np.isnan(sc[s, bt:]))
    status_ok(qsa)


# ---------------------------------------------------------------------------------------------
# selection
# ---------------------------------------------------------------------------------------------

def run_select(qsa, scores_f32, lengths_q, lengths_k, k):
    cu_q = torch.tensor(np.r_[0, np.cumsum(lengths_q)], dtype=torch.int32, device="cuda")
    cu_k = torch.tensor(np.r_[0, np.cumsum(lengths_k)], dtype=torch.int32, device="cuda")
    cfg = qsa.default_config(budget_blocks=k)
    s = torch.from_numpy(np.ascontiguousarray(scores_f32)).cuda()
    sel = qsa.select_blocks(s, cu_q, cu_k, int(sum(lengths_q)), cfg=cfg)
    torch.cuda.synchronize()
    return sel.cpu().numpy()


@pytest.mark.parametrize("case", ["random", "ties", "zeros", "negative"])
def test_select_bit_exact_on_oracle_scores(qsa, case):
    n, k = 2048, 64
    x = inputs.make_prefill([n], seed=25)
    w = x.w.clone()
    if case == "zeros":
        w.zero_()
    if case == "negative":
        w = w - 0.6
    kc = oracle.compress(x.k_idx, 4)
    sc = oracle.index_scores(x.q_idx, w, kc, n, n, 4, ld=(n - 1) // 4)
    if case == "ties":
        sc = np.round(sc * 2) / 2
    s32 = np.where(np.isfinite(sc), sc, 0).astype(np.float32)
    sel_g = run_select(qsa, s32, [n], [n], k)
    sel_o = oracle.select(s32.astype(np.float64), oracle.own_blocks(n, n, 4, None), k)
    np.testing.assert_array_equal(sel_g, sel_o)
    status_ok(qsa)


@pytest.mark.parametrize("bt,mod", [(40000, 7), (65535, 3), (65535, 0), (70000, 0), (70000, 3), (131071, 5)])
def test_select_long_rows(qsa, bt, mod):
    """Long rows, with heavy ties; beyond 65536 candidates the general path runs, its
    threshold ties spread over more than one 65536-key bitmap segment."""
    rng = np.random.default_rng(bt + mod)
    L = bt * 4 + 1
    row = rng.standard_normal(bt).astype(np.float32)
    if mod:
        row = (rng.integers(0, mod, bt)).astype(np.float32)
    sel_g = run_select(qsa, row[None, :], [1], [L], 512)
    sel_o = oracle.select(row[None, :].astype(np.float64), [bt], 512)
    np.testing.assert_array_equal(sel_g, sel_o)
    status_ok(qsa)


def test_select_short_rows_and_ragged_batch(qsa):
    lengths = [1, 2, 4, 5, 8, 9, 64, 65, 300]
    k = 8
    rng = np.random.default_rng(3)
    total = sum(lengths)
    ld = max(lengths) // 4 + 1
    s32 = rng.integers(0, 3, (total, ld)).astype(np.float32)
    sel_g = run_select(qsa, s32, lengths, lengths, k)
    bt = np.concatenate([np.arange(L) // 4 for L in lengths])
    sel_o = oracle.select(s32.astype(np.float64), bt, k)
    np.testing.assert_array_equal(sel_g, sel_o)
    status_ok(qsa)


# ---------------------------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------------------------

def run_chain(qsa, x, lengths, k, chunk=None, want_lse=True, kv_chunk=0):
    cfg = qsa.default_config(budget_blocks=k, kv_chunk_blocks=kv_chunk)
    pre = qsa.Prefill(lengths, chunk_rows=chunk or 16384, cfg=cfg)
    q, kk, v = x.q.cuda(), x.k.cuda(), x.v.cuda()
    sel = pre.index_select(x.q_idx.cuda(), x.w.cuda(), x.k_idx.cuda())
    o, lse = qsa.sparse_attn_prefill(q, kk, v, sel, pre.cu, pre.cu, want_lse=want_lse, cfg=cfg)
    torch.cuda.synchronize()
    return pre, sel, o, lse


def sample_rows(L, n_rand=128, seed=0):
    if L <= 600:
        return np.arange(L)
    rng = np.random.default_rng(seed)
    r = np.r_[np.arange(64), np.arange(L - 64, L), rng.integers(0, L, n_rand)]
    r = np.r_[r, r[r % 4 == 0][:16] + 3]
    return np.unique(r[(r >= 0) & (r < L)])


@pytest.mark.parametrize("lengths,k,kv_chunk", [([512], 16, 0), ([1, 3, 4, 5, 37, 130, 701, 2], 16, 0),
                                                ([3000], 512, 0), ([100, 2100], 64, 0),
                                                ([3000], 512, 64), ([1, 130, 701, 2100], 64, 37)])
def test_attention_on_gpu_selection(qsa, lengths, k, kv_chunk):
    """kv_chunk > 0 runs the L2-blocked schedule with tiny key chunks (many chunks per row)."""
    x = inputs.make_prefill(lengths, seed=26)
    pre, sel, o, lse = run_chain(qsa, x, lengths, k, kv_chunk=kv_chunk)
    sel_g, o_g, lse_g = sel.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(lengths)):
        L = b - a
        rows = sample_rows(L)
        # selection invariants
        for i in rows:
            bt = i // 4
            srow = sel_g[a + i]
            valid = srow[srow >= 0]
            assert len(valid) == min(k, bt + 1) and np.all(srow[len(valid):] == -1)
            assert np.all(np.diff(valid) > 0) and valid[-1] == bt
        ref_o, ref_lse = oracle.attend(x.q[a:b], x.k[a:b], x.v[a:b], sel_g[a + rows], L, L, 4, SCALE, rows)
        check_attn(o_g[a + rows], ref_o)
        np.testing.assert_allclose(lse_g[a + rows], ref_lse, rtol=0, atol=2e-3)
    status_ok(qsa)


def test_full_chain_tiny_config(qsa):
    """Batch 1, n = 512, budget 16 blocks, seed 0: every row end to end."""
    n, k = 512, 16
    x = inputs.make_prefill([n], seed=0)
    pre, sel, o, lse = run_chain(qsa, x, [n], k)
    ref = oracle.qsa_layer(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, 4, k)
    sel_g = sel.cpu().numpy()
    agree = check_selection_near_threshold(sel_g, ref["sel"], ref["scores"], np.arange(n) // 4, k)
    # near-ties may flip a few rows' choices, but nearly every row must agree exactly
    assert agree.mean() > 0.95, agree.mean()
    check_attn(o.float().cpu().numpy()[agree], ref["o"][agree])
    # the rows that differ: attention on the GPU's own selection still matches the oracle
    rows = np.nonzero(~agree)[0]
    if rows.size:
        ref_o, _ = oracle.attend(x.q, x.k, x.v, sel_g[rows], n, n, 4, SCALE, rows)
        check_attn(o.float().cpu().numpy()[rows], ref_o)
    status_ok(qsa)


def test_full_budget_equals_dense_n8192(qsa):
    """n = 8192 with a budget covering every block: QSA output = dense causal attention."""
    n, k = 8192, 2048
    x = inputs.make_prefill([n], seed=0)
    pre, sel, o, lse = run_chain(qsa, x, [n], k)
    rows = sample_rows(n, 96)
    ref_o, ref_lse = oracle.dense(x.q, x.k, x.v, n, n, SCALE, rows)
    check_attn(o.float().cpu().numpy()[rows], ref_o)
    np.testing.assert_allclose(lse.cpu().numpy()[rows], ref_lse, rtol=0, atol=2e-3)
    status_ok(qsa)


@pytest.mark.parametrize("kv_chunk", [0, 256])
def test_chain_n8192_budget512(qsa, kv_chunk):
    n, k = 8192, 512
    x = inputs.make_prefill([n], seed=0)
    pre, sel, o, lse = run_chain(qsa, x, [n], k, chunk=3000, kv_chunk=kv_chunk)
    rows = sample_rows(n, 160)
    sel_g = sel.cpu().numpy()
    kc = oracle.compress(x.k_idx, 4)
    sc = oracle.index_scores(x.q_idx, x.w, kc, n, n, 4, rows, ld=(n - 1) // 4)
    sel_o = oracle.select(sc, rows // 4, k)
    check_selection_near_threshold(sel_g[rows], sel_o, sc, rows // 4, k)
    ref_o, _ = oracle.attend(x.q, x.k, x.v, sel_g[rows], n, n, 4, SCALE, rows)
    check_attn(o.float().cpu().numpy()[rows], ref_o)
    status_ok(qsa)


# ---------------------------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------------------------

# batches below two per SM take the even schedule (rows cut in pieces: 200 rows of a few
# tiles put several rows in every CTA's share; one row of 125 tiles or two rows of one tile
# leave most shares empty); from 296 rows on every CTA attends whole rows
@pytest.mark.parametrize("batch,lo,hi,k", [(5, 1, 3000, 512), (64, 2000, 9000, 512), (3, 5000, 5000, 2048),
                                           (200, 1, 600, 64), (300, 1, 600, 64), (1, 8000, 8000, 2048),
                                           (2, 1, 50, 512)])
def test_decode_chain(qsa, batch, lo, hi, k):
    d = inputs.make_decode(batch, lo, hi, seed=27)
    cfg = qsa.default_config(budget_blocks=k)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1), cfg=cfg)
    ld = max(1, (max(d.seqlens) - 1) // 4)
    scores = torch.empty((batch, ld), dtype=torch.float32, device="cuda")
    qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc[: int(cu_b[-1])], cu_q, cu_k, cu_b, 1, ld, scores=scores, cfg=cfg)
    sel = qsa.select_blocks(scores, cu_q, cu_k, batch, cfg=cfg)
    o, lse = qsa.sparse_attn_decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_k, sel, want_lse=True, cfg=cfg)
    torch.cuda.synchronize()
    sel_g, o_g, lse_g = sel.cpu().numpy(), o.float().cpu().numpy(), lse.cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(d.seqlens)):
        L = b - a
        bt = (L - 1) // 4
        srow = sel_g[s]
        valid = srow[srow >= 0]
        assert len(valid) == min(k, bt + 1) and valid[-1] == bt and np.all(np.diff(valid) > 0)
        # the selection against the oracle's own, under the near-threshold rule
        kc_o = oracle.compress(d.k_idx[a:b], 4)
        sc_o = oracle.index_scores(d.q_idx[s:s + 1], d.w[s:s + 1], kc_o, 1, L, 4, [0], ld=max(1, ld))
        sel_o = oracle.select(sc_o, [bt], k)
        check_selection_near_threshold(srow[None], sel_o, sc_o, [bt], k)
        ref_o, ref_lse = oracle.attend(d.q[s:s + 1], d.k_cache[a:b], d.v_cache[a:b], srow[None], 1, L, 4, SCALE, [0])
        check_attn(o_g[s:s + 1], ref_o)
        np.testing.assert_allclose(lse_g[s], ref_lse[0], rtol=0, atol=2e-3)
    status_ok(qsa)


def paged_cache(kv, seqlens, page, seed, spare=5):
    """Scatter a packed [sum L, 2, 256] cache into a pool of pages in a seeded random
    order; returns the pool [n_pages, page, 2, 256] and the block table [B, max_pages]."""
    npg = [(L + page - 1) // page for L in seqlens]
    total = sum(npg) + spare
    perm = torch.randperm(total, generator=torch.Generator().manual_seed(seed))
    pool = torch.zeros((total, page) + tuple(kv.shape[1:]), dtype=kv.dtype)
    table = torch.full((len(seqlens), max(npg)), -1, dtype=torch.int32)
    a, nxt = 0, 0
    for s, L in enumerate(seqlens):
        for j in range(npg[s]):
            pid = int(perm[nxt])
            nxt += 1
            t0, t1 = j * page, min((j + 1) * page, L)
            pool[pid, : t1 - t0] = kv[a + t0 : a + t1]
            table[s, j] = pid
        a += L
    return pool, table


@pytest.mark.parametrize("batch,lo,hi,k,page", [(5, 1, 3000, 512, 16), (64, 2000, 9000, 512, 64),
                                                (300, 1, 600, 64, 4)])
def test_decode_paged(qsa, batch, lo, hi, k, page):
    """The paged decode reads the same K/V through a block table: equal to the packed
    decode (bit for bit where both run the even schedule) and to the oracle."""
    d = inputs.make_decode(batch, lo, hi, seed=31)
    cfg = qsa.default_config(budget_blocks=k)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1), cfg=cfg)
    ld = max(1, (max(d.seqlens) - 1) // 4)
    scores = torch.empty((batch, ld), dtype=torch.float32, device="cuda")
    qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc[: int(cu_b[-1])], cu_q, cu_k, cu_b, 1, ld, scores=scores, cfg=cfg)
    sel = qsa.select_blocks(scores, cu_q, cu_k, batch, cfg=cfg)
    o_p, lse_p = qsa.sparse_attn_decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_k, sel, want_lse=True,
                                        cfg=cfg)
    kp, table = paged_cache(d.k_cache, d.seqlens, page, seed=32)
    vp, _ = paged_cache(d.v_cache, d.seqlens, page, seed=32)
    o_g, lse_g = qsa.sparse_attn_decode_paged(d.q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), cu_k, sel,
                                              want_lse=True, cfg=cfg)
    torch.cuda.synchronize()
    og, lg = o_g.float().cpu().numpy(), lse_g.cpu().numpy()
    if batch < 296:  # both ran the even-schedule decode kernel on the same values
        assert torch.equal(o_g, o_p) and torch.equal(lse_g, lse_p)
    else:
        check_attn(og, o_p.float().cpu().numpy().astype(np.float64))
    sel_g = sel.cpu().numpy()
    for s, (a, b) in list(enumerate(seq_slices(d.seqlens)))[:: max(1, batch // 16)]:
        L = b - a
        ref_o, ref_lse = oracle.attend(d.q[s:s + 1], d.k_cache[a:b], d.v_cache[a:b], sel_g[s][None], 1, L, 4, SCALE,
                                       [0])
        check_attn(og[s:s + 1], ref_o)
        np.testing.assert_allclose(lg[s], ref_lse[0], rtol=0, atol=2e-3)
    status_ok(qsa)


# ---------------------------------------------------------------------------------------------
# dense causal attention (the comparison baseline)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("lengths", [[1], [77], [512], [1, 3, 130, 129, 700, 64]])
def test_dense_attention(qsa, lengths):
    x = inputs.make_prefill(lengths, seed=28)
    cu_q = torch.tensor(np.r_[0, np.cumsum(lengths)], dtype=torch.int32, device="cuda")
    o, lse = qsa.dense_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), cu_q, cu_q, max(lengths), want_lse=True)
    torch.cuda.synchronize()
    og, lg = o.float().cpu().numpy(), lse.cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(lengths)):
        L = b - a
        rows = sample_rows(L)
        ref_o, ref_l = oracle.dense(x.q[a:b], x.k[a:b], x.v[a:b], L, L, SCALE, rows)
        check_attn(og[a + rows], ref_o)
        np.testing.assert_allclose(lg[a + rows], ref_l, rtol=0, atol=2e-3)
    status_ok(qsa)


def test_dense_attention_decode_shape(qsa):
    """One query per sequence against its whole cache (L_q = 1 < L_k)."""
    d = inputs.make_decode(4, 100, 3000, seed=29)
    cu_k, _ = cu(d.seqlens)
    cu_q = torch.arange(5, dtype=torch.int32, device="cuda")
    o = qsa.dense_attn_prefill(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_q, cu_k, 1)
    torch.cuda.synchronize()
    og = o.float().cpu().numpy()
    for s, (a, b) in enumerate(seq_slices(d.seqlens)):
        L = b - a
        ref_o, _ = oracle.dense(d.q[s:s + 1], d.k_cache[a:b], d.v_cache[a:b], 1, L, SCALE, [0])
        check_attn(og[s:s + 1], ref_o)
    status_ok(qsa)


def test_dense_n8192_matches_full_budget_sparse(qsa):
    """Two independent GPU paths to the same number: dense causal attention and QSA with
    a budget covering every block; both against the oracle on sampled rows."""
    n = 8192
    x = inputs.make_prefill([n], seed=0)
    cu_q = torch.tensor([0, n], dtype=torch.int32, device="cuda")
    od = qsa.dense_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), cu_q, cu_q, n)
    _, _, osp, _ = run_chain(qsa, x, [n], 2048)
    torch.cuda.synchronize()
    d = (od.float() - osp.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 1e-3
    rows = sample_rows(n, 64)
    ref_o, _ = oracle.dense(x.q, x.k, x.v, n, n, SCALE, rows)
    check_attn(od.float().cpu().numpy()[rows], ref_o)
    status_ok(qsa)


@pytest.mark.parametrize("lengths,distinct,k", [([70001, 33000, 20000, 5], 300, 512), ([65540, 40000], 40, 512),
                                                 ([131072], 2000, 2048), ([9000, 17000], 3, 16),
                                                 ([30000, 20001, 7], 1, 512)])
def test_decode_refine_with_repeated_blocks(qsa, lengths, distinct, k):
    """The decode selection (hi-plane scan, exact rescoring of the near-threshold band,
    certain winners above it) against the exact scan and the plain selector, bit for bit,
    on caches whose blocks repeat a few patterns: equal scores by the hundreds sit at the
    threshold, so the tie rule (lower block first) decides most of the selection.  With a
    single pattern every block ties, the candidate list overflows and the row is selected
    from its exact scores inside the same CTA."""
    batch = len(lengths)
    cfg = qsa.default_config(budget_blocks=k)
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    pats = torch.randn((distinct, 4, 128), generator=g, device="cuda").to(torch.bfloat16)
    k_idx = torch.cat([pats[torch.randint(0, distinct, ((L + 3) // 4,), generator=g, device="cuda")]
                       .reshape(-1, 128)[:L] for L in lengths])
    q_idx = torch.randn((batch, 4, 128), generator=g, device="cuda").to(torch.bfloat16)
    w = torch.rand((batch, 4), generator=g, device="cuda")
    cu_k, cu_b = cu(lengths)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(k_idx, cu_k, cu_b, n_blocks=int(cu_b[-1]), cfg=cfg)
    fused = qsa.index_select(q_idx, w, kc, cu_q, cu_k, cu_b, 1, max(lengths), cfg=cfg)
    ld = max(4, ((max(lengths) - 1) // 4 + 3) // 4 * 4)
    scores = qsa.index_scores(q_idx, w, kc, cu_q, cu_k, cu_b, 1, ld, cfg=cfg)
    plain = qsa.select_blocks(scores, cu_q, cu_k, batch, cfg=cfg)
    torch.cuda.synchronize()
    assert torch.equal(fused, plain)
    sel = fused.cpu().numpy()
    check_selection_invariants(sel, [(L - 1) // 4 for L in lengths], k)
    if distinct == 1:  # every block ties (and the list overflows): the lowest k - 1 blocks and the own block
        for s_, L in enumerate(lengths):
            bt = (L - 1) // 4
            want = list(range(min(k - 1, bt))) + [bt] + [-1] * max(0, k - 1 - bt)
            np.testing.assert_array_equal(sel[s_], np.array(want[:k], dtype=np.int32))
    status_ok(qsa)


def test_decode_step_cuda_graph(qsa):
    """The CUDA-graph replay of a decode step equals the eager launches, bit for bit,
    and matches the oracle on the selection it made."""
    d = inputs.make_decode(8, 2000, 9000, seed=30)
    cu_k, cu_b = cu(d.seqlens)
    args = [t.cuda() for t in (d.q, d.q_idx, d.w, d.k_cache, d.v_cache, d.k_idx)]
    kc = qsa.compress_keys(args[5], cu_k, cu_b, n_blocks=int(cu_b[-1]))
    last = torch.tensor([L // 4 - 1 for L in d.seqlens], dtype=torch.int32, device="cuda")
    eager = qsa.DecodeStep(*args, kc, cu_k, cu_b, max(d.seqlens), refresh_blocks=last, graph=False)
    o_eager = eager().clone()
    sel_eager = eager.sel.clone()
    graphed = qsa.DecodeStep(*args, kc, cu_k, cu_b, max(d.seqlens), refresh_blocks=last, graph=True)
    for _ in range(3):
        o_graph = graphed()
    exact = qsa.DecodeStep(*args, kc, cu_k, cu_b, max(d.seqlens), refresh_blocks=last, graph=False, fused=False)
    o_exact = exact()
    torch.cuda.synchronize()
    assert torch.equal(graphed.sel, sel_eager)
    assert torch.equal(o_graph, o_eager)
    # the fused selection (hi-plane scan + exact window) equals the exact scan's
    assert torch.equal(exact.sel, sel_eager)
    assert torch.equal(o_exact, o_eager)
    sel_g = sel_eager.cpu().numpy()
    for s in (0, 7):
        a, b = int(cu_k[s]), int(cu_k[s + 1])
        ref_o, _ = oracle.attend(d.q[s:s + 1], d.k_cache[a:b], d.v_cache[a:b], sel_g[s:s + 1], 1, b - a, 4, SCALE, [0])
        check_attn(o_eager.float().cpu().numpy()[s:s + 1], ref_o)
    status_ok(qsa)


@pytest.mark.parametrize("batch,lo,hi,k,page", [(5, 1, 3000, 512, 16), (64, 2000, 9000, 512, 64),
                                                (9, 4100, 20000, 512, 256), (300, 1, 600, 64, 4)])
def test_paged_kc_decode_chain(qsa, batch, lo, hi, k, page):
    """The compressed keys and the decode indexer through the same block table as the
    paged K/V: compressed keys, selection and attention equal the packed path bit for bit."""
    d = inputs.make_decode(batch, lo, hi, seed=33)
    cfg = qsa.default_config(budget_blocks=k)
    cu_k, cu_b = cu(d.seqlens)
    cu_q = torch.arange(batch + 1, dtype=torch.int32, device="cuda")
    max_len = max(d.seqlens)
    # the packed chain
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=max(int(cu_b[-1]), 1), cfg=cfg)
    ld = max(4, ((max_len - 1) // 4 + 3) // 4 * 4)
    scores = torch.empty((batch, ld), dtype=torch.float32, device="cuda")
    qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc[: max(int(cu_b[-1]), 1)], cu_q, cu_k, cu_b, 1, ld, scores=scores,
                     cfg=cfg)
    sel_p = qsa.select_blocks(scores, cu_q, cu_k, batch, cfg=cfg)
    o_p = qsa.sparse_attn_decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_k, sel_p, cfg=cfg)
    # the paged chain: one table for k_idx, kc, K and V
    kip, table = paged_cache(d.k_idx, d.seqlens, page, seed=34)
    kp, _ = paged_cache(d.k_cache, d.seqlens, page, seed=34)
    vp, _ = paged_cache(d.v_cache, d.seqlens, page, seed=34)
    kip, table, kp, vp = kip.cuda(), table.cuda(), kp.cuda(), vp.cuda()
    kcp = torch.zeros((kip.shape[0], page // 4, 2, 128), dtype=torch.bfloat16, device="cuda")
    qsa.compress_keys_paged(kip, kcp, table, cu_k, max_len, cfg=cfg)
    sel_g = qsa.index_select_paged(d.q_idx.cuda(), d.w.cuda(), kcp, page, table, cu_k, max_len, cfg=cfg)
    o_g = qsa.sparse_attn_decode_paged(d.q.cuda(), kp, vp, table, cu_k, sel_g, cfg=cfg)
    torch.cuda.synchronize()
    # the compressed keys, row by row through the table
    tab = table.cpu().numpy()
    kcp_h, kc_h = kcp.cpu(), kc.cpu()
    for s, L in enumerate(d.seqlens):
        for b in range(L // 4):
            assert torch.equal(kcp_h[tab[s, (4 * b) // page], (4 * b % page) // 4], kc_h[int(cu_b[s]) + b]), (s, b)
    assert torch.equal(sel_g, sel_p)
    if batch < 296:  # both ran the even-schedule decode kernel on the same values
        assert torch.equal(o_g, o_p)
    else:
        check_attn(o_g.float().cpu().numpy(), o_p.float().cpu().numpy().astype(np.float64))
    # a decode step's refresh of the block just completed, into cleared pages
    last = torch.tensor([max(L // 4 - 1, 0) for L in d.seqlens], dtype=torch.int32, device="cuda")
    kcp2 = torch.zeros_like(kcp)
    qsa.compress_keys_paged(kip, kcp2, table, cu_k, max_len, blk_begin=last, max_new_blocks=1, cfg=cfg)
    torch.cuda.synchronize()
    kcp2_h = kcp2.cpu()
    for s, L in enumerate(d.seqlens):
        b = L // 4 - 1
        if b >= 0:
            pg, rw = tab[s, (4 * b) // page], (4 * b % page) // 4
            assert torch.equal(kcp2_h[pg, rw], kcp_h[pg, rw])
    status_ok(qsa)
