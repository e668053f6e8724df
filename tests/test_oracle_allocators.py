"""Oracle pins for the allocators of MILO §4.3 and §5.3 beyond the entropy rule.

§4.3 describes the allocation as greedy: start at the minimum rank and give each remaining
rank unit to the block with the largest marginal gain.  §5.3 compares entropy allocation with
uniform and random allocation under the same total budget.  These tests pin the oracle's
versions: hand-derived worked examples (tests/golden), exact optimality of the greedy on small
problems (brute force over every rank vector), invariants, and the baselines' definitions.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import WORKLOADS, gen_block_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "greedy_alloc_worked_examples.json")


def _shares(sigma):
    e = np.asarray(sigma, dtype=np.float64) ** 2
    t = e.sum(axis=1, keepdims=True)
    return np.divide(e, t, out=np.zeros_like(e), where=t > 0)


def _captured(sigma, ranks):
    s = _shares(sigma)
    return sum(s[b, :r].sum() for b, r in enumerate(ranks))


def test_greedy_worked_examples():
    for case in json.load(open(GOLDEN))["cases"]:
        got = oracle.allocate_ranks_greedy(case["sigma"], case["R"], case["r_min"], case["d"])
        assert list(got) == case["ranks"], case["name"]


@pytest.mark.parametrize("seed", range(12))
def test_greedy_is_optimal_by_brute_force(seed):
    """The greedy maximises the captured energy shares Σ_b Σ_{i<=r_b} g_b(i) over every rank vector
    with Σ r = R and r_min <= r <= d (each block's shares are non-increasing, so greedy is exact)."""
    rng = np.random.default_rng(seed)
    nb, d, r_min = 3, 6, 1
    sigma = np.sort(rng.exponential(1.0, size=(nb, d)) ** rng.uniform(0.5, 3.0, size=(nb, 1)), axis=1)[:, ::-1]
    R = int(rng.integers(nb * r_min + 1, nb * d))
    got = oracle.allocate_ranks_greedy(sigma, R, r_min, d)
    best = max(_captured(sigma, r) for r in itertools.product(range(r_min, d + 1), repeat=nb) if sum(r) == R)
    assert got.sum() == R
    assert _captured(sigma, got) == pytest.approx(best, rel=1e-12)


@pytest.mark.parametrize("seed", range(6))
def test_greedy_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    nb, d = int(rng.integers(2, 40)), int(rng.choice([64, 128]))
    r_min = int(rng.integers(1, 8))
    sigma = np.sort(rng.exponential(1.0, size=(nb, d)), axis=1)[:, ::-1]
    R = int(rng.integers(nb * r_min, nb * d))
    r = oracle.allocate_ranks_greedy(sigma, R, r_min, d)
    assert r.sum() == R and r.min() >= r_min and r.max() <= d
    assert np.array_equal(oracle.allocate_ranks_greedy(sigma * 7.5, R, r_min, d), r)  # scale-free shares
    assert list(oracle.allocate_ranks_greedy(sigma, nb * r_min, r_min, d)) == [r_min] * nb
    assert list(oracle.allocate_ranks_greedy(sigma, nb * d + 3, r_min, d)) == [d] * nb
    with pytest.raises(oracle.BudgetError):
        oracle.allocate_ranks_greedy(sigma, nb * r_min - 1, r_min, d)


def test_greedy_gives_slower_decay_more_rank_noise_free():
    wl = WORKLOADS["tiny"]
    taus = [1.5, 3.0, 6.0, 12.0]
    sig = np.array([oracle.block_svd(gen_block_f64(wl, 0, 0, 0, b, t, noise_std=0.0))[0] for b, t in enumerate(taus)])
    n, d = wl.block_size, wl.head_dim
    R = oracle.rank_total(0.5, len(taus) * n, n, d)
    r = oracle.allocate_ranks_greedy(sig, R, 4, d)
    assert r.sum() == R and np.all(np.diff(r) >= 0)


def test_uniform_baseline():
    assert list(oracle.allocate_ranks_uniform(4, 10, 1, 8)) == [3, 3, 2, 2]
    assert list(oracle.allocate_ranks_uniform(3, 12, 4, 64)) == [4, 4, 4]
    assert list(oracle.allocate_ranks_uniform(2, 40, 4, 16)) == [16, 16]
    # the same as the entropy rule's water-filling with equal weights
    for nb, R in [(5, 23), (64, 3276), (7, 7 * 128 - 1)]:
        want = oracle.allocate_ranks(np.ones(nb), R, 4, 128)[0]
        assert np.array_equal(oracle.allocate_ranks_uniform(nb, R, 4, 128), want)


def test_random_baseline_is_a_valid_seeded_allocation():
    a = oracle.allocate_ranks_random(64, 3276, 4, 128, np.random.default_rng(5))
    b = oracle.allocate_ranks_random(64, 3276, 4, 128, np.random.default_rng(5))
    assert np.array_equal(a, b) and a.sum() == 3276 and a.min() >= 4 and a.max() <= 128
    assert not np.array_equal(a, oracle.allocate_ranks_uniform(64, 3276, 4, 128))


def test_greedy_cut_gap_predicts_stability():
    """Perturbing every share by less than half the cut gap leaves the greedy ranks unchanged; the
    gap is the difference between the smallest share taken and the largest share left."""
    rng = np.random.default_rng(11)
    nb, d, r_min = 8, 16, 2
    sigma = np.sort(rng.exponential(1.0, size=(nb, d)) ** 1.5, axis=1)[:, ::-1]
    R = 60
    r = oracle.allocate_ranks_greedy(sigma, R, r_min, d)
    gap = oracle.greedy_cut_gap(sigma, R, r_min, d)
    s = _shares(sigma)
    taken = [s[b, i] for b in range(nb) for i in range(r_min, r[b])]
    left = [s[b, i] for b in range(nb) for i in range(r[b], d)]
    assert gap == pytest.approx(min(taken) - max(left), abs=1e-15)
    assert gap > 0
    for k in range(20):
        # multiplicative noise on the energies that moves every share by less than gap / 2
        eps = 0.2 * gap * rng.uniform(-1, 1, size=sigma.shape)
        e = sigma ** 2
        s2 = e / e.sum(axis=1, keepdims=True) + eps
        sig2 = np.sqrt(np.maximum(s2, 0) * e.sum(axis=1, keepdims=True))
        assert np.array_equal(oracle.allocate_ranks_greedy(sig2, R, r_min, d), r)
    assert oracle.greedy_cut_gap(sigma, nb * r_min, r_min, d) == float("inf")


# ---------------------------------------------------------------- rules and budget scope of a whole layer

def _tiny_layer(scale_v=1.0):
    from synth import from_storage, gen_layer
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    return wl, from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype) * scale_v


def test_layer_scope_worked_example():
    """Hand-derived: 2 pools x 2 blocks, d = 8, r_min = 1, weights [1, 2 | 3, 2].
    Layer budget 12: lam = 12 / 8 = 1.5, quotas [1.5, 3, 4.5, 3], floors sum 11, the one extra unit goes to
    the largest fractional part (0.5, a tie between blocks 0 and 2, to the lower index): [2, 3 | 4, 3].
    Per pool, 6 each: pool 0 lam = 2, quotas [2, 4]; pool 1 lam = 1.2, quotas [3.6, 2.4], floors 5, the
    extra unit to fraction 0.6: [2, 4 | 4, 2]."""
    sig = np.ones((4, 8))
    r, q = oracle.allocate_blocks("weights", sig, 12, 1, 8, weights=[1, 2, 3, 2])
    assert list(r) == [2, 3, 4, 3] and np.allclose(q, [1.5, 3, 4.5, 3])
    r0, _ = oracle.allocate_blocks("weights", sig[:2], 6, 1, 8, weights=[1, 2])
    r1, _ = oracle.allocate_blocks("weights", sig[2:], 6, 1, 8, weights=[3, 2])
    assert list(r0) + list(r1) == [2, 4, 4, 2]


def test_pool_scope_entropy_is_compress_layer():
    wl, K, V = _tiny_layer()
    a = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    b = oracle.compress_layer_rule(K, V, wl.block_size, 0.5, wl.r_min, "entropy", "pool")
    for t in ("K", "V"):
        for pa, pb in zip(a[t], b[t]):
            assert np.array_equal(pa["ranks"], pb["ranks"])
            assert np.allclose(pa["quotas"], pb["quotas"], rtol=0, atol=1e-12)
            for ua, ub in zip(pa["U"], pb["U"]):
                assert np.array_equal(ua, ub)


@pytest.mark.parametrize("rule", ["entropy", "greedy", "uniform"])
def test_layer_scope_invariants(rule):
    wl, K, V = _tiny_layer()
    n, d, T = wl.block_size, wl.head_dim, wl.context
    R = oracle.rank_total(0.5, T, n, d)
    lay = oracle.compress_layer_rule(K, V, n, 0.5, wl.r_min, rule, "layer")
    ranks = np.array([p["ranks"] for t in ("K", "V") for p in lay[t]])
    assert lay["R_total"] == ranks.sum() == 2 * wl.kv_heads * R
    assert ranks.min() >= wl.r_min and ranks.max() <= d
    if rule != "uniform":  # entropy and energy shares do not change when a pool is scaled
        lay2 = oracle.compress_layer_rule(K * 3.0, V, n, 0.5, wl.r_min, rule, "layer")
        ranks2 = np.array([p["ranks"] for t in ("K", "V") for p in lay2[t]])
        assert np.array_equal(ranks, ranks2)
    else:
        P, nb = ranks.shape
        want = np.full(P * nb, (P * R) // (P * nb))
        want[: (P * R) % (P * nb)] += 1
        assert np.array_equal(ranks.ravel(), want)


@pytest.mark.parametrize("rule", ["entropy", "greedy"])
def test_layer_scope_with_identical_pools_matches_pool_scope(rule):
    """When every pool holds the same data, sharing the budget over the layer changes nothing: the quotas
    (or shares) repeat per pool, and the tie-break by index hands each repeated unit to every pool alike."""
    wl, K, _ = _tiny_layer()
    n = wl.block_size
    a = oracle.compress_layer_rule(K, K, n, 0.5, wl.r_min, rule, "pool")
    b = oracle.compress_layer_rule(K, K, n, 0.5, wl.r_min, rule, "layer")
    for t in ("K", "V"):
        for pa, pb in zip(a[t], b[t]):
            assert np.array_equal(pa["ranks"], pb["ranks"])


def test_layer_scope_greedy_is_optimal_by_brute_force():
    """Over a layer the greedy still maximises the captured energy shares (brute force, 2 pools x 2 blocks)."""
    rng = np.random.default_rng(7)
    d, r_min = 5, 1
    sigma = np.sort(rng.exponential(1.0, size=(4, d)) ** 2.0, axis=1)[:, ::-1]
    for R in range(5, 4 * d):
        got, _ = oracle.allocate_blocks("greedy", sigma, R, r_min, d)
        best = max(_captured(sigma, r) for r in itertools.product(range(r_min, d + 1), repeat=4) if sum(r) == R)
        assert got.sum() == R
        assert _captured(sigma, got) == pytest.approx(best, rel=1e-12)


def test_weights_rule_with_equal_weights_is_uniform():
    sig = np.ones((64, 128))
    r, _ = oracle.allocate_blocks("weights", sig, 3276, 4, 128, weights=np.full(64, 9.0))
    assert np.array_equal(r, oracle.allocate_ranks_uniform(64, 3276, 4, 128))
