"""Failure paths on the GPU, in the forms that fault nothing.

* A selection holding ids outside 0 .. b_t (b_t + 1 and -5): the attention kernels
  skip those entries, raise QSA_ERR_DEVICE_CHECK in the sticky status word, and
  every row still equals the oracle on the ids that remain (an id past b_t only
  holds keys after the query, which the causal rule hides anyway).
* A bounded mbarrier wait that runs out: the QSA_DEBUG_CHECKS library
  (libqsa_debug.so, 20 ms waits) withholds the copies of one kc tile of the decode
  scan when qsa_debug_inject(1) is set.  Its consumer gives up, the call returns,
  the status word reads QSA_ERR_TIMEOUT, and the next call without the fault is
  correct.  It runs in a child process so the release library stays untouched.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs
from parity_common import SCALE, check_attn

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


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


def random_selection(bts, k, seed):
    """A valid selection per row: the own block b_t plus min(k - 1, b_t) distinct earlier
    blocks, ascending, padded with -1."""
    g = np.random.default_rng(seed)
    sel = np.full((len(bts), k), -1, dtype=np.int32)
    for i, bt in enumerate(bts):
        m = min(k - 1, bt)
        ids = np.sort(g.choice(bt, size=m, replace=False)) if m else np.zeros(0, dtype=np.int64)
        sel[i, :m + 1] = np.append(ids, bt)
    return sel


def corrupt(sel, bts, rows):
    """Rows `rows` get b_t + 1 at slot 1 and -5 at slot 3 (rows with at least 5 ids);
    returns the corrupted copy and the same rows with those slots dropped (-1)."""
    bad, clean = sel.copy(), sel.copy()
    for i in rows:
        assert (sel[i] >= 0).sum() >= 5
        bad[i, 1], bad[i, 3] = bts[i] + 1, -5
        clean[i, 1], clean[i, 3] = -1, -1
    return bad, clean


def test_prefill_out_of_range_ids_flag_device_check(qsa):
    lengths, k = [700, 1300], 64
    x = inputs.make_prefill(lengths, seed=91)
    cu_q, _ = cu(lengths)
    bts = np.concatenate([np.arange(L) // 4 for L in lengths])
    sel = random_selection(bts, k, seed=5)
    rows = [a + i for a, L in zip((0, 700), lengths) for i in (40, 333, L - 1)]
    bad, clean = corrupt(sel, bts, rows)
    qsa.device_status(clear=True)
    cfg = qsa.default_config(budget_blocks=k)
    o, lse = qsa.sparse_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), torch.from_numpy(bad).cuda(), cu_q, cu_q,
                                     want_lse=True, cfg=cfg)
    assert qsa.device_status(clear=True) == qsa.QSA_ERR_DEVICE_CHECK
    o_g, lse_g = o.float().cpu().numpy(), lse.cpu().numpy()
    for s, (a, L) in enumerate(zip((0, 700), lengths)):
        check = np.array(sorted(set([0, 17, 250, L - 2] + [r - a for r in rows if a <= r < a + L])))
        ref_o, ref_lse = oracle.attend(x.q[a:a + L], x.k[a:a + L], x.v[a:a + L], clean[a + check], L, L, 4, SCALE,
                                       check)
        check_attn(o_g[a + check], ref_o)
        np.testing.assert_allclose(lse_g[a + check], ref_lse, rtol=0, atol=2e-3)
    # the same call on the valid selection leaves the status word clear (a -1 among a row's
    # first min(k, b_t + 1) entries counts as out of range too)
    qsa.sparse_attn_prefill(x.q.cuda(), x.k.cuda(), x.v.cuda(), torch.from_numpy(sel).cuda(), cu_q, cu_q, cfg=cfg)
    assert qsa.device_status(clear=True) == 0


@pytest.mark.parametrize("paged", [False, True])
def test_decode_out_of_range_ids_flag_device_check(qsa, paged):
    batch, k = 6, 128
    d = inputs.make_decode(batch, 900, 5000, seed=92)
    cu_k, _ = cu(d.seqlens)
    bts = [(L - 1) // 4 for L in d.seqlens]
    sel = random_selection(bts, k, seed=6)
    rows = [0, 3, 5]
    bad, clean = corrupt(sel, bts, rows)
    qsa.device_status(clear=True)
    cfg = qsa.default_config(budget_blocks=k)
    if not paged:
        o, lse = qsa.sparse_attn_decode(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_k,
                                        torch.from_numpy(bad).cuda(), want_lse=True, cfg=cfg)
    else:
        page = 64
        npg = [(L + page - 1) // page for L in d.seqlens]
        table = torch.full((batch, max(npg)), -1, dtype=torch.int32)
        kp = torch.zeros((sum(npg), page, 2, 256), dtype=torch.bfloat16)
        vp = torch.zeros_like(kp)
        p0, t0 = 0, 0
        for s, L in enumerate(d.seqlens):
            for j in range(npg[s]):
                n = min(page, L - j * page)
                kp[p0 + j, :n] = d.k_cache[t0 + j * page:t0 + j * page + n]
                vp[p0 + j, :n] = d.v_cache[t0 + j * page:t0 + j * page + n]
                table[s, j] = p0 + j
            p0 += npg[s]
            t0 += L
        o, lse = qsa.sparse_attn_decode_paged(d.q.cuda(), kp.cuda(), vp.cuda(), table.cuda(), cu_k,
                                              torch.from_numpy(bad).cuda(), want_lse=True, cfg=cfg)
    assert qsa.device_status(clear=True) == qsa.QSA_ERR_DEVICE_CHECK
    o_g, lse_g = o.float().cpu().numpy(), lse.cpu().numpy()
    t0 = 0
    for s, L in enumerate(d.seqlens):
        ref_o, ref_lse = oracle.attend(d.q[s:s + 1], d.k_cache[t0:t0 + L], d.v_cache[t0:t0 + L], clean[s:s + 1], 1,
                                       L, 4, SCALE)
        check_attn(o_g[s:s + 1], ref_o)
        np.testing.assert_allclose(lse_g[s:s + 1], ref_lse, rtol=0, atol=2e-3)
        t0 += L


def test_mtp_out_of_range_ids_flag_device_check(qsa):
    batch, next_n, k = 4, 4, 64
    d = inputs.make_decode(batch, 600, 3000, seed=93, next_n=next_n)
    cu_k, _ = cu(d.seqlens)
    bts = [(L - 1) // 4 for L in d.seqlens]
    sel = random_selection(bts, k, seed=7)
    bad, clean = corrupt(sel, bts, [1, 2])
    qsa.device_status(clear=True)
    o, lse = qsa.sparse_attn_decode_mtp(d.q.cuda(), d.k_cache.cuda(), d.v_cache.cuda(), cu_k,
                                        torch.from_numpy(bad).cuda(), want_lse=True,
                                        cfg=qsa.default_config(budget_blocks=k))
    assert qsa.device_status(clear=True) == qsa.QSA_ERR_DEVICE_CHECK
    o_g = o.float().cpu().numpy()
    t0 = 0
    for s, L in enumerate(d.seqlens):
        rows = np.arange(L - next_n, L)
        ref_o, _ = oracle.attend(d.q[s], d.k_cache[t0:t0 + L], d.v_cache[t0:t0 + L],
                                 np.repeat(clean[s:s + 1], next_n, axis=0), next_n, L, 4, SCALE)
        check_attn(o_g[s], ref_o)
        assert rows.size == next_n
        t0 += L


CHILD = textwrap.dedent("""
    import sys, torch
    sys.path.insert(0, {root!r})
    from block_sparse_long_09_b200 import inputs, qsa
    assert qsa.LIB_PATH.endswith("libqsa_debug.so"), qsa.LIB_PATH
    d = inputs.make_decode(3, 20000, 30000, seed=94)
    a, b = [0], [0]
    for L in d.seqlens:
        a.append(a[-1] + L)
        b.append(b[-1] + L // 4)
    cu_k = torch.tensor(a, dtype=torch.int32, device="cuda")
    cu_b = torch.tensor(b, dtype=torch.int32, device="cuda")
    cu_q = torch.arange(4, dtype=torch.int32, device="cuda")
    kc = qsa.compress_keys(d.k_idx.cuda(), cu_k, cu_b, n_blocks=b[-1])
    args = (d.q_idx.cuda(), d.w.cuda(), kc, cu_q, cu_k, cu_b, 1, max(d.seqlens))
    qsa.device_status(clear=True)
    assert qsa.library().qsa_debug_inject(1) == qsa.QSA_OK
    qsa.index_select(*args)
    st = qsa.device_status(clear=True)
    assert st == qsa.QSA_ERR_TIMEOUT, st
    assert qsa.library().qsa_debug_inject(0) == qsa.QSA_OK
    sel = qsa.index_select(*args)
    assert qsa.device_status(clear=True) == 0
    # the exact scores and the plain selector give the same blocks
    ld = max(4, ((max(d.seqlens) - 1) // 4 + 3) // 4 * 4)
    sc = qsa.index_scores(d.q_idx.cuda(), d.w.cuda(), kc, cu_q, cu_k, cu_b, 1, ld)
    ref = qsa.select_blocks(sc, cu_q, cu_k, 3)
    assert torch.equal(sel, ref)
    assert qsa.device_status(clear=True) == 0
    print("CHILD-OK")
""")


def test_wait_timeout_returns_status_and_leaves_gpu_usable(qsa):
    from block_sparse_long_09_b200 import build
    build.build(debug=True)
    env = dict(os.environ, QSA_DEBUG_BUILD="1")
    p = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], env=env, capture_output=True, text=True,
                       timeout=600)
    assert p.returncode == 0 and "CHILD-OK" in p.stdout, p.stdout[-2000:] + p.stderr[-4000:]
    # and this process's library is unaffected
    assert qsa.library().qsa_debug_inject(1) == qsa.QSA_ERR_UNSUPPORTED
    assert qsa.device_status(clear=True) == 0
