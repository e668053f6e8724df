"""Pins of the oracle's pre-RoPE decode (oracle/rope.py): the rotation against its complex-number form, the
properties that define a rotary embedding, and the decode against plain attention over rotated keys."""
import math

import numpy as np
import pytest

import oracle
from milo_testutil import stored_layer
from synth import WORKLOADS, from_storage, gen_layer


def _rope_complex(x, positions, theta):
    """RoPE written as complex multiplication: pair (i, i + d/2) is z = x_i + 1j·x_{i+d/2}, turned by e^{1j·φ_i}."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    z = x[:, :d // 2] + 1j * x[:, d // 2:]
    freqs = np.array([theta ** (-2.0 * i / d) for i in range(d // 2)])
    z = z * np.exp(1j * np.outer(np.asarray(positions, dtype=np.float64), freqs))
    return np.concatenate([z.real, z.imag], axis=1)


def test_hand_example():
    # d = 4, base 100: pair (0, 2) turns by pos·1, pair (1, 3) by pos·0.1; at position 1:
    # (1, 3) → (cos 1 − 3 sin 1, 3 cos 1 + sin 1) and (2, 4) → (2 cos .1 − 4 sin .1, 4 cos .1 + 2 sin .1)
    got = oracle.apply_rope([[1.0, 2.0, 3.0, 4.0]], [1], 100.0)[0]
    want = [-1.9841106, 1.5906747, 2.4623779, 4.1796835]
    assert np.allclose(got, want, atol=1e-6)


@pytest.mark.parametrize("d,theta", [(8, 10000.0), (64, 1e6), (128, 1e6)])
def test_matches_complex_form(d, theta):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((50, d))
    pos = rng.integers(0, 200000, 50)
    assert np.allclose(oracle.apply_rope(x, pos, theta), _rope_complex(x, pos, theta), rtol=0, atol=1e-9)


def test_position_zero_is_identity_and_norms_are_kept():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((20, 16))
    assert np.array_equal(oracle.apply_rope(x, np.zeros(20), 1e6), x)
    y = oracle.apply_rope(x, np.arange(20) * 997, 1e6)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_scores_depend_on_relative_position_only():
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal((1, 32)), rng.standard_normal((1, 32))
    for m, n in [(5, 3), (1000, 17), (70000, 69999)]:
        lhs = float((oracle.apply_rope(a, [m], 1e6) @ oracle.apply_rope(b, [n], 1e6).T)[0, 0])
        rhs = float((oracle.apply_rope(a, [m - n], 1e6) @ b.T)[0, 0])
        assert math.isclose(lhs, rhs, rel_tol=1e-9, abs_tol=1e-9)


def _full_rank_layer(name="tiny"):
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    K, V = from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype)
    lay = oracle.compress_layer(K, V, wl.block_size, 1.25, wl.r_min)  # rank d everywhere: exact keys
    return wl, L, K, V, lay


@pytest.mark.parametrize("theta", [1e4, 1e6])
def test_decode_equals_attention_over_rotated_keys(theta):
    """At full rank the factors reproduce K exactly, so the decode must equal plain softmax attention over the
    keys rotated (in complex form) at their absolute positions 0 .. T − 1: a block-local position, a
    rotated value or a wrong pairing fails this."""
    wl, L, K, V, lay = _full_rank_layer()
    q = from_storage(L["q"], wl.dtype)
    Ks, Vs = from_storage(L["K_suf"], wl.dtype), from_storage(L["V_suf"], wl.dtype)
    got = oracle.decode_attention_rope(q, lay, Ks, Vs, theta)
    Kr = np.stack([_rope_complex(K[h], np.arange(wl.context), theta) for h in range(wl.kv_heads)])
    want = oracle.decode_attention_dense(q, Kr, V, Ks, Vs)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-11)


def test_selected_blocks_keep_their_positions():
    wl, L, K, V, lay = _full_rank_layer()
    q = from_storage(L["q"], wl.dtype)
    Ks, Vs = from_storage(L["K_suf"], wl.dtype), from_storage(L["V_suf"], wl.dtype)
    nb, n = wl.num_blocks, wl.block_size
    mask = np.zeros((wl.kv_heads, nb), dtype=bool)
    mask[:, 1::2] = True
    got = oracle.decode_attention_rope(q, lay, Ks, Vs, 1e6, block_mask=mask)
    rows = np.concatenate([np.arange(b * n, (b + 1) * n) for b in range(nb) if mask[0, b]])
    Kr = np.stack([_rope_complex(K[h][rows], rows, 1e6) for h in range(wl.kv_heads)])
    want = oracle.decode_attention_dense(q, Kr, V[:, rows], Ks, Vs)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-11)


def test_low_rank_decode_uses_the_stored_factors():
    """Below full rank the decode equals dense attention over the rotated reconstruction U_b·B_bᵀ."""
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    K, V = from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype)
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, wl.budgets[0], wl.r_min), "bf16")
    q = from_storage(L["q"], wl.dtype)
    Ks, Vs = from_storage(L["K_suf"], wl.dtype), from_storage(L["V_suf"], wl.dtype)
    got = oracle.decode_attention_rope(q, lay, Ks, Vs, 1e6)
    Kr = np.stack([_rope_complex(oracle.reconstruct_pool(lay["K"][h]), np.arange(wl.context), 1e6)
                   for h in range(wl.kv_heads)])
    Vd = np.stack([oracle.reconstruct_pool(lay["V"][h]) for h in range(wl.kv_heads)])
    want = oracle.decode_attention_dense(q, Kr, Vd, Ks, Vs)
    assert np.allclose(got, want, rtol=1e-9, atol=1e-11)
