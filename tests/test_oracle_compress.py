"""Pins of the oracle's compression half: SVD truncation, entropy, budget, allocation.

Each check is fixed by mathematics, not by re-running the oracle's own formula:
the generator's exact noise-free spectra, the Eckart–Young theorem, closed-form
entropies, hand-derived allocations, an independent Jacobi SVD and a bisection
root finder.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import WORKLOADS, gen_block_f64, gen_pool_f64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _geometric_block(tau, k=40, n=256, d=64, seed_block=0):
    wl = WORKLOADS["tiny"]
    return gen_block_f64(wl, 0, 0, 0, seed_block, tau, noise_std=0.0, signal_rank=k)


# ---------------------------------------------------------------- SVD / truncation

@pytest.mark.parametrize("tau", [2.0, 5.0, 16.0])
def test_singular_values_match_generator(tau):
    x = _geometric_block(tau)
    sigma, bvec = oracle.block_svd(x)
    want = np.exp(-np.arange(1, 41) / tau)
    assert np.allclose(sigma[:40], want, rtol=1e-11, atol=1e-15)
    assert np.all(sigma[40:] < 1e-13)
    assert np.allclose(bvec.T @ bvec, np.eye(64), atol=1e-12)


@pytest.mark.parametrize("tau,r", [(4.0, 3), (8.0, 10), (16.0, 25)])
def test_eckart_young_error_from_generator_spectrum(tau, r):
    """‖X − U Bᵀ‖_F² equals the discarded energy Σ_{i>r} e^{−2i/τ} (known from the generator)."""
    x = _geometric_block(tau)
    sigma, bvec = oracle.block_svd(x)
    u = x @ bvec[:, :r]
    err = np.linalg.norm(x - u @ bvec[:, :r].T)
    want = math.sqrt(sum(math.exp(-2.0 * i / tau) for i in range(r + 1, 41)))
    assert err == pytest.approx(want, rel=1e-9)
    # token-side factor carries the singular values: Uᵀ U = diag(σ_1..σ_r)²
    assert np.allclose(u.T @ u, np.diag(np.exp(-2.0 * np.arange(1, r + 1) / tau)), atol=1e-12)


def test_truncation_beats_random_subspaces():
    rng = np.random.default_rng(3)
    x = gen_block_f64(WORKLOADS["tiny"], 0, 0, 1, 2, 6.0)
    sigma, bvec = oracle.block_svd(x)
    r = 12
    best = np.linalg.norm(x - x @ bvec[:, :r] @ bvec[:, :r].T)
    for _ in range(20):
        qm, _ = np.linalg.qr(bvec[:, :r] + 0.05 * rng.standard_normal((64, r)))
        assert np.linalg.norm(x - x @ qm @ qm.T) >= best - 1e-15


def test_lapack_matches_handwritten_jacobi():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((48, 16)) @ np.diag(np.exp(-np.arange(16) / 3.0))
    s1, b1 = oracle.block_svd(x)
    s2, b2, sweeps = oracle.hestenes_svd(x)
    assert sweeps < 30
    assert np.allclose(s1, s2, rtol=1e-12, atol=1e-15)
    for r in (1, 5, 11):
        p1 = b1[:, :r] @ b1[:, :r].T
        p2 = b2[:, :r] @ b2[:, :r].T
        assert np.allclose(p1, p2, atol=1e-9)


def test_compress_pool_factors_reconstruct_projection():
    wl = WORKLOADS["tiny"]
    x = gen_pool_f64(wl, 0, 0, 0)
    pool = oracle.compress_pool(x, wl.block_size, 0.5, wl.r_min)
    rec = oracle.reconstruct_pool(pool)
    for b, r in enumerate(pool["ranks"]):
        xb = x[b * 256:(b + 1) * 256]
        err = np.linalg.norm(xb - rec[b * 256:(b + 1) * 256])
        tail = math.sqrt(float(np.sum(pool["sigma"][b][r:] ** 2)))
        assert err == pytest.approx(tail, rel=1e-9)


# ---------------------------------------------------------------- entropy

def _geometric_entropy(tau, k):
    rho = math.exp(-2.0 / tau)
    z = rho * (1.0 - rho ** k) / (1.0 - rho)
    mean_i = 1.0 / (1.0 - rho) - k * rho ** k / (1.0 - rho ** k)
    return math.log(z) - math.log(rho) * mean_i


def test_entropy_closed_form_geometric():
    spec = json.load(open(os.path.join(GOLDEN, "entropy_closed_forms.json")))
    for case in spec["geometric"]["cases"]:
        tau, k = case["tau"], case["k"]
        x = _geometric_block(tau, k=min(k, 64), n=256, d=64) if k <= 64 else None
        if x is None:
            wl = WORKLOADS["qwen2.5-7b-layer"]
            x = gen_block_f64(wl, 0, 0, 0, 0, tau, noise_std=0.0)
        h = oracle.spectral_entropy(oracle.block_svd(x)[0])
        assert h == pytest.approx(_geometric_entropy(tau, k), rel=1e-9, abs=1e-11)


def test_entropy_flat_and_rank_one():
    spec = json.load(open(os.path.join(GOLDEN, "entropy_closed_forms.json")))
    rng = np.random.default_rng(0)
    for k in spec["flat"]["k"]:
        g, _ = np.linalg.qr(rng.standard_normal((96, k)))
        h, _ = np.linalg.qr(rng.standard_normal((64, k)))
        x = 0.37 * g @ h.T
        assert oracle.spectral_entropy(oracle.block_svd(x)[0]) == pytest.approx(math.log(k), abs=1e-10)
    assert oracle.spectral_entropy(np.zeros(8)) == 0.0


def test_entropy_scale_invariant():
    x = gen_block_f64(WORKLOADS["tiny"], 0, 0, 0, 1, 9.0)
    h1 = oracle.spectral_entropy(oracle.block_svd(x)[0])
    h2 = oracle.spectral_entropy(oracle.block_svd(1234.5 * x)[0])
    assert h1 == pytest.approx(h2, rel=1e-12)


# ---------------------------------------------------------------- budget and allocation

def test_rank_total_is_half_memory():
    # 7B layer: 32768 tokens, d 128, blocks of 512 -> 3276 rank units of (512+128) numbers each
    assert oracle.rank_total(0.5, 32768, 512, 128) == 3276
    assert 3276 * (512 + 128) <= 0.5 * 32768 * 128 < 3277 * (512 + 128)
    assert oracle.rank_total(0.5, 1024, 256, 64) == 102


def test_allocation_worked_examples():
    spec = json.load(open(os.path.join(GOLDEN, "alloc_worked_examples.json")))
    for case in spec["cases"]:
        ranks, quotas, lam = oracle.allocate_ranks(case["w"], case["R"], case["r_min"], case["d"])
        assert list(ranks) == case["ranks"], case["name"]
        assert np.allclose(quotas, case["quotas"], atol=1e-12), case["name"]
        if case["lam"] is not None:
            assert lam == pytest.approx(case["lam"], rel=1e-12)


def test_allocation_budget_error():
    with pytest.raises(oracle.BudgetError):
        oracle.allocate_ranks([1.0, 2.0, 3.0], 11, 4, 64)


def _bisect_lam(w, R, r_min, d):
    lo, hi = 0.0, d / min(w) * 2
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        if np.clip(mid * w, r_min, d).sum() < R:
            lo = mid
        else:
            hi = mid
    return 0.5 * (lo + hi)


@pytest.mark.parametrize("seed", range(6))
def test_allocation_invariants_random(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(2, 200))
    d = int(rng.choice([64, 128]))
    r_min = int(rng.integers(1, 8))
    w = np.exp(rng.uniform(0.0, math.log(d), nb))
    R = int(rng.integers(nb * r_min, nb * d))
    ranks, q, lam = oracle.allocate_ranks(w, R, r_min, d)
    assert ranks.sum() == R
    assert ranks.min() >= r_min and ranks.max() <= d
    assert np.all(np.abs(ranks - q) < 1.0)
    assert q.sum() == pytest.approx(R, rel=1e-12)
    assert lam == pytest.approx(_bisect_lam(w, R, r_min, d), rel=1e-9)
    perm = rng.permutation(nb)
    r2, _, _ = oracle.allocate_ranks(w[perm], R, r_min, d)
    frac = q - np.floor(q)
    if len(set(np.round(frac, 9))) == nb:  # permutation equivariance holds when no fractional ties
        assert np.array_equal(r2, ranks[perm])
    # larger weight never gets a smaller rank
    order = np.argsort(w)
    assert np.all(np.diff(q[order]) >= -1e-12)


def test_allocation_full_rank_budget():
    ranks, q, _ = oracle.allocate_ranks([1.0, 2.0, 50.0], 3 * 64, 4, 64)
    assert list(ranks) == [64, 64, 64]


def test_pool_allocation_monotone_in_tau_noise_free():
    wl = WORKLOADS["tiny"]
    taus = [1.5, 3.0, 6.0, 12.0]
    x = np.concatenate([gen_block_f64(wl, 0, 0, 0, b, t, noise_std=0.0) for b, t in enumerate(taus)])
    pool = oracle.compress_pool(x, 256, 0.5, 4)
    assert np.all(np.diff(pool["entropy"]) > 0)
    assert np.all(np.diff(pool["ranks"]) >= 0)
    assert pool["ranks"].sum() == pool["R"]


def test_pool_ranks_scale_invariant():
    wl = WORKLOADS["tiny"]
    x = gen_pool_f64(wl, 0, 0, 1)
    a = oracle.compress_pool(x, 256, 0.5, 4)["ranks"]
    b = oracle.compress_pool(7.25 * x, 256, 0.5, 4)["ranks"]
    assert np.array_equal(a, b)
    assert int(a.sum()) * (256 + 64) <= 0.5 * 1024 * 64


def test_tiefree_taus_give_wide_cut():
    wl = WORKLOADS["qwen2.5-0.5b-layer"]
    taus = oracle.tiefree_taus(wl, 0, 0.5, 0.02)
    from synth import from_storage, gen_layer
    L = gen_layer(wl, 0, taus=taus)
    for t in ("K", "V"):
        for h in range(wl.kv_heads):
            pool = oracle.compress_pool(from_storage(L[t][h], wl.dtype), wl.block_size, 0.5, wl.r_min)
            gap, _ = oracle.cut_gap(pool["quotas"], pool["R"])
            assert gap >= 0.02
