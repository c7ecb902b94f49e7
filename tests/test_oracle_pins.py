"""Pins for the fp64 oracle, each against something other than the oracle itself.

Sources: "On the Design of Qwen3.8 Next Architecture" (reading notes), section 6:
the pooled-key equation (k̄_b), the indexer equation (I_ib), the budget sentence
(own causal block always kept, k-1 best complete blocks), and the expansion of
selected blocks to token indices for softmax attention.

The pins: hand-worked fixtures (tests/golden), a library routine (torch SDPA in
fp64) for the dense case, brute-force subset enumeration on tiny inputs, closed
forms (w = 0, v = const, q = 0, r = 1, identical rows) and an independently
ordered score computation.  Each is chosen so that a plausible slip in the oracle
(a dropped head, a wrong sign, a missing mask, an off-by-one block) fails.
"""
import itertools
import math
import os

import numpy as np
import pytest
import torch

import oracle
from block_sparse_long_09_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a) -> torch.Tensor:
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.double().numpy()


# --------------------------------------------------------------------------
# Compressor
# --------------------------------------------------------------------------

def test_compress_hand_fixture():
    rows, outs = [], []
    with open(os.path.join(GOLDEN, "compress_hand.txt")) as f:
        for line in f:
            if line.startswith("in "):
                rows.append([float(x) for x in line.split()[1:]])
            elif line.startswith("out "):
                outs.append([float(x) for x in line.split()[1:]])
    kc = oracle.compress(bf16(rows), r=4, normalise=True, eps=1e-6)
    assert kc.shape == (2, 4)
    np.testing.assert_allclose(kc, np.array(outs), rtol=0, atol=1e-15)


def test_compress_identical_rows_is_rmsnorm_of_row():
    g = torch.Generator().manual_seed(3)
    row = torch.randn(128, generator=g).to(torch.bfloat16)
    k_idx = row[None, :].repeat(4 * 5 + 3, 1)
    kc = oracle.compress(k_idx, r=4)
    x = f64(row)
    expect = x / math.sqrt(np.mean(x * x) + 1e-6)
    assert kc.shape == (5, 128)
    np.testing.assert_allclose(kc, np.tile(expect, (5, 1)), rtol=1e-14, atol=1e-14)


def test_compress_without_norm_is_block_mean():
    g = torch.Generator().manual_seed(4)
    k_idx = torch.randn(4 * 7 + 1, 128, generator=g).to(torch.bfloat16)
    kc = oracle.compress(k_idx, r=4, normalise=False)
    x = f64(k_idx)[: 4 * 7].reshape(7, 4, 128)
    np.testing.assert_allclose(kc, x.mean(axis=1), rtol=1e-15, atol=1e-15)


def test_compress_r1_norm_of_each_row():
    g = torch.Generator().manual_seed(5)
    k_idx = torch.randn(9, 128, generator=g).to(torch.bfloat16)
    kc = oracle.compress(k_idx, r=1)
    x = f64(k_idx)
    expect = x / np.sqrt((x * x).mean(axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(kc, expect, rtol=1e-14, atol=1e-14)


# --------------------------------------------------------------------------
# Indexer scores
# --------------------------------------------------------------------------

def _scores_by_einsum(q_idx, w, kc, Lq, Lk, r):
    """Independent loop order: all heads' dot products as one einsum, ReLU,
    weight, sum over heads, then the causal cut b < floor(t / r)."""
    q = f64(q_idx)                         # [Lq, H, d]
    dots = np.einsum("bd,ihd->ihb", kc, q)  # [Lq, H, nb]
    s = np.einsum("ih,ihb->ib", w.double().numpy(), np.maximum(dots, 0.0))
    t = (Lk - Lq) + np.arange(Lq)
    bt = t // r
    mask = np.arange(kc.shape[0])[None, :] >= bt[:, None]
    s[mask] = -np.inf
    return s


@pytest.mark.parametrize("n", [37, 64, 203])
def test_scores_match_independent_einsum(n):
    x = inputs.make_prefill([n], seed=1)
    kc = oracle.compress(x.k_idx, 4)
    ld = kc.shape[0]
    s = oracle.index_scores(x.q_idx, x.w, kc, n, n, 4, ld=ld)
    ref = _scores_by_einsum(x.q_idx, x.w, kc, n, n, 4)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(s))
    np.testing.assert_allclose(s[fin], ref[fin], rtol=1e-12, atol=1e-12)


def test_scores_w_one_is_unweighted_relu_sum():
    n = 48
    x = inputs.make_prefill([n], seed=2)
    w1 = torch.ones_like(x.w)
    kc = oracle.compress(x.k_idx, 4)
    s = oracle.index_scores(x.q_idx, w1, kc, n, n, 4, ld=kc.shape[0])
    q = f64(x.q_idx)
    for i in (5, 17, 47):
        bt = i // 4
        for b in range(bt):
            want = sum(max(0.0, float(np.dot(q[i, h], kc[b]))) for h in range(4))
            assert abs(s[i, b] - want) <= 1e-12 * max(1.0, abs(want))
        assert np.all(np.isneginf(s[i, bt:]))


def _read_scores_fixture():
    kc, q, w, s = {}, {}, {}, {}
    with open(os.path.join(GOLDEN, "scores_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or ":" not in line:
                continue
            head, vals = line.split(":")
            key = head.split()
            v = [float(x) for x in vals.split()]
            if key[0] == "kc":
                kc[int(key[1])] = v
            elif key[0] == "q":
                q[(int(key[1]), int(key[2]))] = v
            elif key[0] == "w":
                w[int(key[1])] = v
            elif key[0] == "s":
                s[(int(key[1]), int(key[2]))] = v[0]
    return kc, q, w, s


def test_scores_hand_fixture():
    """Hand-worked scores (tests/golden/scores_hand.txt): a negative dot that the
    ReLU must zero, unequal head weights, the own block and earlier rows at -inf."""
    kc_d, q_d, w_d, s_d = _read_scores_fixture()
    L, H, d = 12, 4, 4
    kc = np.array([kc_d[b] for b in range(3)], dtype=np.float64)
    q = np.zeros((L, H, d), dtype=np.float32)
    w = np.zeros((L, H), dtype=np.float32)
    for (t, h), v in q_d.items():
        q[t, h] = v
    for t, v in w_d.items():
        w[t] = v
    rows = sorted({t for t, _ in s_d})
    s = oracle.index_scores(bf16(q), torch.from_numpy(w), kc, L, L, 4, rows, ld=3)
    for n, t in enumerate(rows):
        for b in range(3):
            want = s_d[(t, b)]
            if math.isinf(want):
                assert np.isneginf(s[n, b]), (t, b, s[n, b])
            else:
                assert s[n, b] == want, (t, b, s[n, b], want)


def test_scores_decode_position():
    """Lq < Lk: query row i sits at t = Lk - Lq + i."""
    Lk, Lq = 41, 3
    x = inputs.make_prefill([Lk], seed=6)
    kc = oracle.compress(x.k_idx, 4)
    s_full = oracle.index_scores(x.q_idx, x.w, kc, Lk, Lk, 4, ld=kc.shape[0])
    s_tail = oracle.index_scores(x.q_idx[Lk - Lq:], x.w[Lk - Lq:], kc, Lq, Lk, 4, ld=kc.shape[0])
    np.testing.assert_array_equal(s_tail, s_full[Lk - Lq:])


# --------------------------------------------------------------------------
# Selection
# --------------------------------------------------------------------------

def test_select_hand_fixture():
    with open(os.path.join(GOLDEN, "select_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, sc, want = line.split("|")
            k, bt = (int(x) for x in head.split())
            scores = [float(x) for x in sc.split()]
            want = [int(x) for x in want.split()]
            row = np.full((1, max(1, bt + 1)), -np.inf)
            row[0, :bt] = scores
            got = oracle.select(row, [bt], k)
            assert got[0].tolist() == want, line


def _brute_select(scores, bt, k):
    """Enumerate every subset of the candidates of size min(k-1, bt); keep the
    largest score sum, and among equal sums the lexicographically smallest
    ascending index list; then add the own block."""
    m = min(k - 1, bt)
    best_sum, best = None, None
    for comb in itertools.combinations(range(bt), m):
        s = sum(scores[b] for b in comb)
        if best_sum is None or s > best_sum or (s == best_sum and list(comb) < best):
            best_sum, best = s, list(comb)
    out = sorted(best + [bt])
    return out + [-1] * (k - len(out))


@pytest.mark.parametrize("k", [2, 3, 4])
def test_select_matches_brute_force(k):
    rng = np.random.default_rng(10 + k)
    for bt in range(0, 9):
        for _ in range(6):
            # small integers make exact ties common
            scores = rng.integers(0, 4, size=bt).astype(np.float64)
            row = np.full((1, 9), -np.inf)
            row[0, :bt] = scores
            got = oracle.select(row, [bt], k)[0].tolist()
            assert got == _brute_select(scores, bt, k), (bt, scores, got)


def test_select_w_zero_closed_form():
    n, k = 160, 8
    x = inputs.make_prefill([n], seed=7)
    kc = oracle.compress(x.k_idx, 4)
    s = oracle.index_scores(x.q_idx, torch.zeros_like(x.w), kc, n, n, 4, ld=kc.shape[0])
    bt = oracle.own_blocks(n, n, 4, None)
    sel = oracle.select(s, bt, k)
    for i in range(n):
        b = bt[i]
        want = sorted(set(range(min(k - 1, b))) | {b})
        assert sel[i].tolist() == want + [-1] * (k - len(want))


def test_select_invariants_tiny_config():
    n, k = 512, 16
    x = inputs.make_prefill([n], seed=0)
    res = oracle.qsa_layer(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, 4, k,
                           rows=np.arange(0, n, 7))
    rows = np.arange(0, n, 7)
    for j, i in enumerate(rows):
        bt = i // 4
        s = res["sel"][j]
        valid = s[s >= 0]
        assert np.all(s[len(valid):] == -1)
        assert len(valid) == min(k, bt + 1)
        assert np.all(np.diff(valid) > 0)
        assert valid[-1] == bt and valid.max() <= bt
        # the chosen candidates beat every unchosen one (or tie with a higher index)
        chosen = set(valid[:-1].tolist())
        sc = res["scores"][j]
        worst = min(((sc[b], -b) for b in chosen), default=None)
        for b in range(bt):
            if b not in chosen and worst is not None:
                assert (sc[b], -b) < worst


# --------------------------------------------------------------------------
# Attention
# --------------------------------------------------------------------------

def _masked_dense_numpy(q, k, v, t, tokens, scale):
    """Separately written: full logits over keys 0..t, -inf where a key is not
    in ``tokens``, softmax, weighted sum of v.  One query row, all heads."""
    qn, kn, vn = f64(q), f64(k), f64(v)
    Hq, Hkv = qn.shape[0], kn.shape[1]
    grp = Hq // Hkv
    mask = np.full(t + 1, -np.inf)
    mask[sorted(tokens)] = 0.0
    o = np.zeros((Hq, qn.shape[1]))
    lse = np.zeros(Hq)
    for h in range(Hq):
        g = h // grp
        lg = kn[: t + 1, g, :] @ qn[h] * scale + mask
        m = lg.max()
        p = np.exp(lg - m)
        o[h] = p @ vn[: t + 1, g, :] / p.sum()
        lse[h] = m + math.log(p.sum())
    return o, lse


def test_attend_matches_masked_dense_on_brute_force_selection():
    n, r, k = 32, 4, 3
    x = inputs.make_prefill([n], seed=11)
    kc = oracle.compress(x.k_idx, r)
    s = oracle.index_scores(x.q_idx, x.w, kc, n, n, r, ld=kc.shape[0])
    bt = oracle.own_blocks(n, n, r, None)
    sel = np.array([_brute_select(s[i, : bt[i]], int(bt[i]), k) for i in range(n)], dtype=np.int32)
    np.testing.assert_array_equal(sel, oracle.select(s, bt, k))
    rows = np.array([0, 3, 4, 9, 15, 22, 31])
    o, lse = oracle.attend(x.q, x.k, x.v, sel[rows], n, n, r, 1 / 16, rows)
    for j, i in enumerate(rows):
        toks = [b * r + u for b in sel[i] if b >= 0 for u in range(r) if b * r + u <= i]
        oref, lref = _masked_dense_numpy(x.q[i], x.k, x.v, int(i), toks, 1 / 16)
        np.testing.assert_allclose(o[j], oref, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(lse[j], lref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n", [64, 101])
def test_sparse_equals_dense_when_budget_covers_all(n):
    x = inputs.make_prefill([n], seed=12)
    res = oracle.qsa_layer(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, 4, budget=n // 4 + 2)
    od, ld = oracle.dense(x.q, x.k, x.v, n, n, 1 / 16)
    np.testing.assert_allclose(res["o"], od, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(res["lse"], ld, rtol=1e-12, atol=1e-13)


def test_dense_matches_torch_sdpa_fp64():
    n = 96
    x = inputs.make_prefill([n], seed=13)
    od, lse = oracle.dense(x.q, x.k, x.v, n, n, 1 / 16)
    q = x.q.double().permute(1, 0, 2)[None]                     # [1, 24, n, 256]
    k = x.k.double().repeat_interleave(12, dim=1).permute(1, 0, 2)[None]
    v = x.v.double().repeat_interleave(12, dim=1).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True, scale=1 / 16)
    np.testing.assert_allclose(od, ref[0].permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-12)
    lg = torch.einsum("hid,hjd->hij", q[0], k[0]) / 16
    lg = lg.masked_fill(torch.ones(n, n, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(lse, torch.logsumexp(lg, -1).T.numpy(), rtol=1e-12, atol=1e-12)


def test_r1_full_budget_is_dense():
    n = 40
    x = inputs.make_prefill([n], seed=14)
    res = oracle.qsa_layer(x.q, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, r=1, budget=n)
    od, _ = oracle.dense(x.q, x.k, x.v, n, n, 1 / 16)
    np.testing.assert_allclose(res["o"], od, rtol=1e-12, atol=1e-13)


def test_constant_v_gives_constant_output():
    n, k = 80, 4
    x = inputs.make_prefill([n], seed=15)
    c = torch.randn(2, 256, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    v = c[None].repeat(n, 1, 1)
    res = oracle.qsa_layer(x.q, x.k, v, x.q_idx, x.k_idx, x.w, n, n, 4, k)
    want = np.repeat(f64(c), 12, axis=0)  # head h uses group h // 12
    for j in range(n):
        np.testing.assert_allclose(res["o"][j], want, rtol=1e-13, atol=1e-13)


def test_zero_q_gives_mean_of_selected_values():
    n, k = 72, 3
    x = inputs.make_prefill([n], seed=16)
    q0 = torch.zeros_like(x.q)
    res = oracle.qsa_layer(q0, x.k, x.v, x.q_idx, x.k_idx, x.w, n, n, 4, k)
    vn = f64(x.v)
    for i in range(n):
        toks = [b * 4 + u for b in res["sel"][i] if b >= 0 for u in range(4) if b * 4 + u <= i]
        mean = vn[toks].mean(axis=0)                   # [2, 256]
        np.testing.assert_allclose(res["o"][i], np.repeat(mean, 12, axis=0), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(res["lse"][i], math.log(len(toks)), rtol=1e-13, atol=1e-13)


def test_duplicate_and_padding_entries_are_ignored():
    n = 40
    x = inputs.make_prefill([n], seed=17)
    rows = np.array([39])
    a = np.array([[1, 3, 9, -1, -1]], dtype=np.int32)
    b = np.array([[9, 1, 1, 3, -1]], dtype=np.int32)
    oa, la = oracle.attend(x.q, x.k, x.v, a, n, n, 4, 1 / 16, rows)
    ob, lb = oracle.attend(x.q, x.k, x.v, b, n, n, 4, 1 / 16, rows)
    np.testing.assert_array_equal(oa, ob)
    np.testing.assert_array_equal(la, lb)


# --------------------------------------------------------------------------
# Shared selection of a multi-token decode step
# --------------------------------------------------------------------------

def test_select_shared_hand_fixture():
    with open(os.path.join(GOLDEN, "select_shared_hand.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            head, scores, expect = line.split("|")
            k, next_n, L = (int(x) for x in head.split())
            sc = [float(x) for x in scores.split()]
            row = np.full((1, max(1, (L - 1) // 4)), -np.inf)
            row[0, :len(sc)] = sc
            got = oracle.select_shared(row, [L], next_n, k)
            assert got[0].tolist() == [int(x) for x in expect.split()], (line, got)


@pytest.mark.parametrize("L", [1, 4, 5, 17, 40, 203])
def test_select_shared_next_n_1_is_select(L):
    rng = np.random.default_rng(L)
    bt = (L - 1) // 4
    sc = rng.integers(0, 4, (1, max(1, bt))).astype(np.float64)
    for k in (1, 2, 5, 16):
        np.testing.assert_array_equal(oracle.select_shared(sc, [L], 1, k), oracle.select(sc, [bt], k))


@pytest.mark.parametrize("next_n", [2, 3, 4])
def test_select_shared_brute_force(next_n):
    """Every subset of the candidates below the first forced block: the max-sum subset,
    lexicographically smallest among equal sums, plus the forced own blocks."""
    rng = np.random.default_rng(next_n)
    for trial in range(40):
        L = int(rng.integers(1, 36))
        k = int(rng.integers(2, 6))
        b_first, b_last = max(L - next_n, 0) // 4, (L - 1) // 4
        nf = b_last - b_first + 1
        sc = rng.integers(0, 3, (1, max(1, (L - 1) // 4))).astype(np.float64)
        m = min(b_first, k - nf)
        best = None
        for sub in itertools.combinations(range(b_first), m):
            key = (-sum(sc[0, b] for b in sub), sub)
            if best is None or key < best:
                best = key
        want = sorted(list(best[1]) + list(range(b_first, b_last + 1)))
        want += [-1] * (k - len(want))
        got = oracle.select_shared(sc, [L], next_n, k)[0].tolist()
        assert got == want, (L, k, next_n, sc, got, want)


# ---------------------------------------------------------------- partial RoPE of the pooled key

def _rope_cases():
    out = []
    for line in open(os.path.join(GOLDEN, "rope_hand.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        head, x, want = (part.split() for part in line.split("|"))
        out.append((int(head[0]), int(head[1]), float(head[2]), np.array(x, float), np.array(want, float)))
    return out


def test_rope_hand_fixture():
    cases = _rope_cases()
    assert len(cases) == 2
    for pos, rd, base, x, want in cases:
        np.testing.assert_allclose(oracle.rope(x[None], [pos], rd, base)[0], want, rtol=0, atol=1e-12)


def test_rope_identity_cases_and_norm():
    g = np.random.default_rng(11)
    x = g.standard_normal((9, 128))
    np.testing.assert_array_equal(oracle.rope(x, np.zeros(9, np.int64), 64, 1e4), x)  # position 0
    np.testing.assert_array_equal(oracle.rope(x, np.arange(9) * 4, 0, 1e4), x)       # no rotated dims
    y = oracle.rope(x, np.arange(9) * 1000 + 7, 64, 1e4)
    np.testing.assert_array_equal(y[:, 64:], x[:, 64:])                              # only the first 64 dims
    np.testing.assert_allclose(np.linalg.norm(y[:, :64], axis=1), np.linalg.norm(x[:, :64], axis=1), rtol=1e-12)


def test_rope_dot_depends_on_relative_position_only():
    # <R(p) a, R(s) b> = <R(p + D) a, R(s + D) b>: a wrong pairing, sign or frequency index
    # breaks either this or the hand fixture
    g = np.random.default_rng(12)
    a, b = g.standard_normal((2, 64))
    for p, s, D in [(3, 0, 5), (1000, 17, 12345), (40, 40, 262140)]:
        d0 = oracle.rope(a[None], [p], 64, 1e4)[0] @ oracle.rope(b[None], [s], 64, 1e4)[0]
        d1 = oracle.rope(a[None], [p + D], 64, 1e4)[0] @ oracle.rope(b[None], [s + D], 64, 1e4)[0]
        assert abs(d0 - d1) <= 1e-9 * (np.abs(a) @ np.abs(b))
    # and it does depend on the offset p - s
    d0 = oracle.rope(a[None], [5], 64, 1e4)[0] @ oracle.rope(b[None], [0], 64, 1e4)[0]
    d1 = oracle.rope(a[None], [6], 64, 1e4)[0] @ oracle.rope(b[None], [0], 64, 1e4)[0]
    assert abs(d0 - d1) > 1e-6


def test_compress_rope_pools_before_rotating():
    # the page's order: average-pool the r keys, then rotate the pooled key at b r; it differs
    # from pooling keys that were each rotated at their own position
    g = torch.Generator().manual_seed(13)
    k = torch.randn((64, 128), generator=g).to(torch.bfloat16)
    kc = oracle.compress(k, 4, rope_dims=64, rope_base=1e4)
    plain = oracle.compress(k, 4)
    np.testing.assert_allclose(kc, oracle.rope(plain, np.arange(16) * 4, 64, 1e4), rtol=0, atol=1e-12)
    kk = k.double().numpy()
    per_token = oracle.rope(kk, np.arange(64), 64, 1e4).reshape(16, 4, 128).mean(axis=1)
    per_token /= np.sqrt((per_token ** 2).mean(axis=1, keepdims=True) + 1e-6)
    assert np.abs(per_token - kc).max() > 1e-3
    # RMSNorm (unit gain) commutes with the rotation: rotating before or after the norm agrees
    mean = kk.reshape(16, 4, 128).mean(axis=1)
    rot_then_norm = oracle.rope(mean, np.arange(16) * 4, 64, 1e4)
    rot_then_norm /= np.sqrt((rot_then_norm ** 2).mean(axis=1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(kc, rot_then_norm, rtol=0, atol=1e-12)
