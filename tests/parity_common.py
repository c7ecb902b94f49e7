"""Tolerance checks shared by the GPU-vs-oracle parity tests.

The bounds are the method's acceptance bounds:
  scores     |g - o| <= 1e-2 * max(|o|, s*_t), s*_t = the oracle's (k-1)-th best
             candidate score of row t (the row max when there are fewer candidates)
  selection  on the GPU's own scores a block may differ from the oracle's choice only
             where the oracle's score lies within 1e-2 (relative) of s*_t
  attention  max-abs <= 2e-2 and mean-abs <= 1e-3 against the oracle on the same selection
"""
import numpy as np

SCALE = 1.0 / 16.0


def kth_best(scores_row, bt, k):
    """The (k-1)-th best candidate score of a row (the row max when fewer candidates)."""
    if bt == 0:
        return 0.0
    cand = np.sort(scores_row[:bt])[::-1]
    return float(cand[k - 2]) if bt >= k - 1 and k >= 2 else float(cand[0])


def check_scores(g, o, bt, k):
    """The score tolerance: relative where it matters, floored at the row's k-th score."""
    for n in range(g.shape[0]):
        b = int(bt[n])
        if b == 0:
            continue
        s_star = abs(kth_best(o[n], b, k))
        err = np.abs(g[n, :b] - o[n, :b])
        bound = 1e-2 * np.maximum(np.abs(o[n, :b]), s_star) + 1e-6
        bad = np.nonzero(err > bound)[0]
        assert bad.size == 0, (n, bad[:5], g[n, bad[:5]], o[n, bad[:5]])


def check_selection_near_threshold(sel_g, sel_o, scores_o, bt, k):
    """The GPU selects on its own scores: a block may differ from the oracle's choice
    only where the oracle's score is within 1e-2 (relative) of the row's k-th best.
    Returns the mask of rows whose selections agree exactly."""
    agree = np.all(sel_g == sel_o, axis=1)
    for n in np.nonzero(~agree)[0]:
        s_star = kth_best(scores_o[n], int(bt[n]), k)
        diff = set(sel_g[n].tolist()) ^ set(sel_o[n].tolist())
        for b in diff:
            assert 0 <= b < bt[n], (n, b)
            assert abs(scores_o[n, b] - s_star) < 1e-2 * abs(s_star) + 1e-9, (n, b, scores_o[n, b], s_star)
    return agree


def check_selection_invariants(sel_rows, bt, k):
    """Ascending, unique, own block last, count min(k, b_t + 1), -1 padding."""
    for n in range(sel_rows.shape[0]):
        srow = sel_rows[n]
        valid = srow[srow >= 0]
        assert len(valid) == min(k, int(bt[n]) + 1), (n, len(valid))
        assert np.all(srow[len(valid):] == -1)
        assert np.all(np.diff(valid) > 0) and valid[-1] == bt[n]


def check_attn(g, o):
    d = np.abs(np.asarray(g, dtype=np.float64) - o)
    assert d.max() <= 2e-2, d.max()
    assert d.mean() <= 1e-3, d.mean()


def sampled_rows(L, seed=0, n_rand=256):
    """The sampled-row set of the large workloads: the first 64 rows, the last 64,
    n_rand seeded random rows, and with every random row the first and last row of
    its micro-block (t mod 4 = 0 and 3)."""
    rng = np.random.default_rng(seed)
    r = rng.integers(0, L, n_rand)
    blk = r - r % 4
    rows = np.r_[np.arange(min(64, L)), np.arange(max(0, L - 64), L), r, blk, np.minimum(blk + 3, L - 1)]
    return np.unique(rows)


def bits(t):
    """bf16 tensor -> numpy uint16 bit patterns (on the host)."""
    import torch
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def mean_blocks_differing(sel_g, sel_o):
    """Mean over rows of the number of selected blocks that differ between two selections."""
    d = [len(set(a.tolist()) ^ set(b.tolist())) / 2.0 for a, b in zip(sel_g, sel_o)]
    return float(np.mean(d)) if d else 0.0
