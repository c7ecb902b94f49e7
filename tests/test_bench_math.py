"""The work counts behind the bench's roofline fractions, checked on the CPU.

Each helper is compared with a brute-force count on small cases and with the
closed-form totals of the benchmarked workloads: the prefill of 262 144 tokens at
k = 512 gathers 1.094 TB of K/V and its indexer scores 8.59e9 (row, block) pairs
(8.80e12 flop at 1024 flop each), and a decode step of batch 64 at 131 072 tokens
scans 537 MB of hi planes and gathers 268 MB.
"""
import importlib.util
import os

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)  # defines functions only; main() runs under __main__
    return mod


def brute_tokens(n, r, k):
    total = 0
    for t in range(n):
        bt = t // r
        blocks = list(range(bt + 1))[-k:] if bt + 1 <= k else list(range(k - 1)) + [bt]
        for b in blocks:  # complete blocks give r tokens, the own block only those <= t
            total += sum(1 for j in range(b * r, b * r + r) if j <= t)
    return total


@pytest.mark.parametrize("n,r,k", [(1, 4, 512), (50, 4, 4), (203, 4, 16), (97, 1, 8)])
def test_selected_tokens_brute_force(bench, n, r, k):
    assert bench.selected_tokens(n, r, k) == brute_tokens(n, r, k)


@pytest.mark.parametrize("n", [0, 1, 4, 5, 101, 4096])
def test_index_pairs_brute_force(bench, n):
    assert bench.index_pairs(n) == sum(t // 4 for t in range(n))


def test_prefill_totals_at_262144(bench):
    n = 262144
    pairs = bench.index_pairs(n)
    assert pairs == n * (n - 4) // 8  # sum of floor(t / 4) over t < n, n a multiple of 4
    assert abs(pairs - 8.59e9) / 8.59e9 < 1e-3
    assert abs(1024 * pairs - 8.80e12) / 8.80e12 < 2e-3
    tok = bench.selected_tokens(n)
    # a row t >= 2044 attends 511 full blocks and the t mod 4 + 1 tokens of its own block
    # (2045 .. 2048); the first 2044 rows attend fewer
    assert tok == sum(min(511, t // 4) * 4 + t % 4 + 1 for t in range(n))
    assert 2030 * n < tok < 2048 * n
    gather = bench.gather_bytes_per_query(tok)
    assert abs(gather - 1.09442e12) / 1.09442e12 < 1e-4
    assert abs(4 * 24 * 256 * tok - 1.3133e13) / 1.3133e13 < 1e-3  # the attention's flops


def test_decode_bytes_at_131072(bench):
    total, kc, gather = bench.decode_bytes([131072] * 64, 256)
    assert kc == 64 * (131072 // 4) * 256 == 536870912           # the hi planes, 256 B per block
    assert gather == 64 * 2048 * 2048 == 268435456              # 2048 tokens x (K + V) x 2 heads x 512 B
    assert total == kc + gather + 64 * ((131072 - 1) // 4) * 8  # plus one fp32 score written and read per block
    # a short sequence attends every token it has
    _, _, g_short = bench.decode_bytes([7], 256)
    assert g_short == bench.gather_bytes_per_query(7)
    assert np.isclose(bench.gather_bytes_per_query(1), 2048)
