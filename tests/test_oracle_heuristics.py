"""Pins of the comparison selectors (uniform eviction, random drop) of the
Forcing-KV page ("与基线对比及工程启示", first item): Philox4x64-10 against
numpy's Philox bit generator, the selections against brute force and closed
forms."""
import itertools

import numpy as np
import pytest

from oracle import fkv_heuristics as fh


def _numpy_block(ctr, key):
    """numpy's Philox returns the block of counter c + 1 first: start it at c - 1."""
    c = sum(int(v) << (64 * i) for i, v in enumerate(ctr))
    k = sum(int(v) << (64 * i) for i, v in enumerate(key))
    g = np.random.Philox(counter=(c - 1) % (1 << 256), key=k)
    return tuple(int(v) for v in g.random_raw(4))


@pytest.mark.parametrize("ctr,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((1, 0, 0, 0), (0, 0)),
    ((7, 3, 0, 0), (12345, 0)),
    ((2**64 - 1, 2**64 - 1, 2**64 - 1, 2**64 - 1), (2**64 - 1, 2**64 - 1)),
])
def test_philox_matches_numpy(ctr, key):
    assert fh.philox4x64_10(ctr, key) == _numpy_block(ctr, key)


def test_philox_matches_numpy_random_inputs():
    rng = np.random.default_rng(17)
    for _ in range(50):
        ctr = tuple(int(v) for v in rng.integers(0, 2**64, 4, dtype=np.uint64, endpoint=False))
        key = tuple(int(v) for v in rng.integers(0, 2**64, 2, dtype=np.uint64, endpoint=False))
        assert fh.philox4x64_10(ctr, key) == _numpy_block(ctr, key)


def test_priorities_grid_and_spread():
    u = fh.priorities(seed=99, lh=3, n=4000)
    assert np.all((u >= 0) & (u < 1)) and np.all(u * 2**24 == np.floor(u * 2**24))
    assert abs(u.mean() - 0.5) < 0.02 and abs(u.var() - 1 / 12) < 0.01
    assert not np.array_equal(u[:100], fh.priorities(seed=99, lh=4, n=100))
    assert not np.array_equal(u[:100], fh.priorities(seed=98, lh=3, n=100))


@pytest.mark.parametrize("n,k", [(18, 13), (18, 18), (18, 1), (18, 0), (7, 3), (18720, 14040), (5, 5)])
def test_uniform_keep_is_evenly_spaced(n, k):
    kept = fh.uniform_keep(n, k)
    assert len(kept) == k and len(set(kept.tolist())) == k
    if k:
        assert kept[0] == 0 and kept[-1] < n and np.all(np.diff(kept) > 0)
        gaps = np.diff(np.append(kept, n))           # the last gap wraps to n
        assert set(gaps.tolist()) <= {n // k, -(-n // k)}
    if k and n % k == 0:
        assert np.array_equal(kept, np.arange(0, n, n // k))


def test_random_keep_is_the_best_subset_by_brute_force():
    n, k, seed = 9, 4, 5
    for lh in range(6):
        u = fh.priorities(seed, lh, n)
        best = max(itertools.combinations(range(n), k), key=lambda c: sum(u[i] for i in c))
        assert fh.random_keep(seed, lh, n, k).tolist() == sorted(best)


def test_token_mode_keeps_sink_and_recent():
    N, S, R, C = 200, 24, 16, 50
    for policy in ("uniform", "random"):
        kept = fh.head_keep(policy, granularity="token", seed=3, lh=1, k=C, N=N, sink=S, recent=R)
        assert len(kept) == S + C + R and np.all(np.diff(kept) > 0)
        assert set(range(S)) <= set(kept.tolist()) and set(range(N - R, N)) <= set(kept.tolist())
        mid = kept[S:S + C]
        assert np.all((mid >= S) & (mid < N - R))
    assert np.array_equal(fh.head_keep("uniform", granularity="token", seed=0, lh=0, k=C, N=N,
                                       sink=S, recent=R)[S:S + C], S + fh.uniform_keep(N - S - R, C))
