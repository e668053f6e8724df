"""GPU parity of milo_compress against the oracle.

Acceptance: integer ranks bit-exact (on generator inputs whose allocation has a
cut gap of at least delta(wl) rank units, checked against the GPU's own quota
error), per-block compression error within 1e-3
relative of the Eckart–Young optimum (on the GPU's fp32 eigenvectors, before the
storage cast), and end-to-end decode within 2e-2 (bf16) / 1e-4 (fp32) of the
oracle's fp64 pipeline.
"""
import functools
import math

import numpy as np
import pytest

import oracle
from milo_testutil import assert_close, factor_arrays, from_torch, to_torch, untok_slabs
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
DELTA = 0.02  # cut gap of the generator inputs, rank units


def delta(wl):
    """Cut gap required of a workload's generator inputs.  With nb blocks the fractional parts of the
    quotas are about 1/nb apart, so a fixed 0.02 is unreachable for long pools (256 blocks); 1/nb keeps
    a margin of more than ten times the fp32 quota error measured on the GPU (about 2e-4 rank units),
    and every test asserts that error below half the gap it relies on."""
    return min(DELTA, 1.0 / wl.num_blocks)
E2E_TOL = {"f32": 1e-4, "bf16": 2e-2}


@functools.lru_cache(maxsize=3)
def _inputs_and_oracle(name, beta, layer):
    """Tie-free generator inputs and the oracle's compression of them (cached across tests)."""
    wl = WORKLOADS[name]
    taus = oracle.tiefree_taus(wl, layer, beta, delta(wl))
    L = gen_layer(wl, layer, taus=taus)
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    ref = oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min)
    return L, ref


def _compress_both(name, beta=None, layer=0, keep=True):
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    beta = wl.budgets[0] if beta is None else beta
    L, ref = _inputs_and_oracle(name, beta, layer)
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, beta, wl.r_min,
                      keep_intermediates=keep)
    return wl, dt, L, K, V, ref, f


def _ref_pools(ref):
    out = []
    for h in range(len(ref["K"])):
        out += [ref["K"][h], ref["V"][h]]
    return out


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_ranks_bit_exact_and_eckart_young(name):
    wl, dt, L, K, V, ref, f = _compress_both(name)
    code, bits = f.status()
    assert code == 0, bits
    got = factor_arrays(f)
    pools = _ref_pools(ref)
    want_ranks = np.array([p["ranks"] for p in pools])
    # quota error of the fp32 eigen-decomposition, in rank units (must stay below DELTA / 2)
    qerr = np.abs(got["quotas"] - np.array([p["quotas"] for p in pools])).max()
    print(f"{name}: max |quota_gpu - quota_oracle| = {qerr:.2e}")
    assert qerr < delta(wl) / 2
    assert np.array_equal(got["ranks"], want_ranks)
    n, d = wl.block_size, wl.head_dim
    for p, pool in enumerate(pools):
        X = (K if p % 2 == 0 else V)[p // 2]
        lam_max = pool["sigma"][:, 0] ** 2
        assert np.all(np.abs(got["eigvals"][p] - pool["sigma"] ** 2) <= 2e-5 * lam_max[:, None])
        for b in range(wl.num_blocks):
            r = int(want_ranks[p, b])
            xb = X[b * n:(b + 1) * n]
            bv = got["eigvecs"][p, b, :r].T  # d × r
            err = np.linalg.norm(xb - xb @ bv @ bv.T)
            opt = math.sqrt(float(np.sum(pool["sigma"][b][r:] ** 2)))
            if r < d:
                assert (err - opt) / opt <= 1e-3, (p, b, err, opt)
            else:
                # full rank: the optimum is 0; fp32 eigenvectors are orthonormal to ~1e-6, so allow 1e-4 |X_b|
                assert err <= 1e-4 * np.linalg.norm(xb), (p, b, err)


def test_stored_factors_reconstruct_near_optimum_7b():
    wl, dt, L, K, V, ref, f = _compress_both("qwen2.5-7b-layer")
    got = factor_arrays(f)
    n = wl.block_size
    pools = _ref_pools(ref)
    worst = 0.0
    for p in range(len(pools)):
        X = (K if p % 2 == 0 else V)[p // 2]
        for b in range(wl.num_blocks):
            r0, r1 = got["row_offsets"][p, b], got["row_offsets"][p, b + 1]
            u = untok_slabs(got["tok"][r0 * n:r1 * n], n, r1 - r0)
            rec = u @ got["dim"][r0:r1]
            xb = X[b * n:(b + 1) * n]
            opt = math.sqrt(float(np.sum(pools[p]["sigma"][b][r1 - r0:] ** 2)))
            err = np.linalg.norm(xb - rec)
            # bf16 storage of both factors adds about 2^-8 of the block norm on top of the optimum
            assert err <= opt + 2.0 ** -8 * np.linalg.norm(xb)
            worst = max(worst, (err - opt) / np.linalg.norm(xb))
    print(f"stored-bf16 excess error over the optimum, max relative to |X_b|: {worst:.2e}")


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_end_to_end_decode(name):
    import decode_attention_milo_b200 as milo
    wl, dt, L, K, V, ref, f = _compress_both(name, keep=False)
    S = wl.suffix
    out = from_torch(milo.decode_attn(to_torch(L["q"], dt), f, to_torch(L["K_suf"], dt) if S else None,
                                      to_torch(L["V_suf"], dt) if S else None))
    want = oracle.decode_attention(from_storage(L["q"], dt), ref, from_storage(L["K_suf"], dt),
                                   from_storage(L["V_suf"], dt))
    assert_close(out, want, E2E_TOL[dt], f"{name} end to end")


def test_full_rank_budget_reproduces_attention_7b():
    """Budget (n+d)/n gives every block rank d: the decode must equal plain attention on K, V."""
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS["qwen2.5-7b-layer"]
    L = gen_layer(wl)
    dt = wl.dtype
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, 1.25, wl.r_min)
    assert np.all(f.ranks() == wl.head_dim)
    q = L["q"][:4]
    Ks, Vs = L["K_suf"][:4], L["V_suf"][:4]
    out = from_torch(milo.decode_attn(to_torch(q, dt), f, to_torch(Ks, dt), to_torch(Vs, dt)))
    want = oracle.decode_attention_dense(from_storage(q, dt), from_storage(L["K"], dt), from_storage(L["V"], dt),
                                         from_storage(Ks, dt), from_storage(Vs, dt))
    assert_close(out, want, E2E_TOL[dt], "full rank vs dense attention")


def test_sweep_limit_reports_no_convergence():
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    f = milo.compress(to_torch(L["K"], "f32"), to_torch(L["V"], "f32"), wl.block_size, 0.5, wl.r_min,
                      max_sweeps=1)
    code, bits = f.status()
    assert code == 4 and bits & 1


STACK_CASES = [("qwen2.5-7b-stack", 0.5), ("qwen2.5-32b-stack", 0.25), ("qwen2.5-32b-stack", 0.5),
               ("qwen2.5-32b-stack", 0.75)]


def _tile_sample(wl):
    """Queries at the first and last item of every row tile of the decode (128 // G queries per tile)."""
    ipt = min(wl.batch, 128 // wl.group)
    s = set()
    for t0 in range(0, wl.batch, ipt):
        s |= {t0, min(wl.batch, t0 + ipt) - 1}
    return sorted(s)


@pytest.mark.parametrize("name,beta", STACK_CASES)
def test_stack_layer_ranks_and_end_to_end(name, beta):
    """One full layer of a stacked workload (each layer is an independent call): ranks bit-exact, then GPU
    decode of the whole batch and suffix on the GPU's own factors against the oracle's fp64 pipeline, on
    queries that span every row tile."""
    import decode_attention_milo_b200 as milo
    wl, dt, L, K, V, ref, f = _compress_both(name, beta=beta, layer=1, keep=True)
    assert f.status()[0] == 0
    pools = _ref_pools(ref)
    qerr = np.abs(factor_arrays(f)["quotas"] - np.array([p["quotas"] for p in pools])).max()
    print(f"{name} beta={beta}: max |quota_gpu - quota_oracle| = {qerr:.2e}")
    assert qerr < delta(wl) / 2
    want_ranks = np.array([p["ranks"] for p in pools])
    assert np.array_equal(f.ranks(), want_ranks)
    out = from_torch(milo.decode_attn(to_torch(L["q"], dt), f, to_torch(L["K_suf"], dt),
                                      to_torch(L["V_suf"], dt)))
    assert f.status()[0] == 0
    idx = _tile_sample(wl)
    want = oracle.decode_attention(from_storage(L["q"][idx], dt), ref, from_storage(L["K_suf"][idx], dt),
                                   from_storage(L["V_suf"][idx], dt))
    assert_close(out[idx], want, E2E_TOL[dt], f"{name} beta {beta} end to end")


@pytest.mark.parametrize("name", ["qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_compression_is_deterministic(name):
    """Three compressions of one layer give the same bytes: ranks, eigenpairs and both factors.  A race
    between the eigensolver's warps shows up here as last-bit differences in the eigenpairs of some blocks,
    which the ranks and the error bounds above do not see."""
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    K, V = to_torch(L["K"], wl.dtype), to_torch(L["V"], wl.dtype)
    runs = []
    for _ in range(3):
        f = milo.compress(K, V, wl.block_size, wl.budgets[0], wl.r_min, keep_intermediates=True)
        a = factor_arrays(f)
        assert f.status()[0] == 0
        f.close()
        runs.append(a)
    for key in ("ranks", "row_offsets", "tok", "dim", "eigvals", "eigvecs"):
        for other in runs[1:]:
            same = np.array_equal(runs[0][key], other[key])
            assert same, f"{name}: {key} differs between two compressions of the same layer"
