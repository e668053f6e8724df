"""Pins of the oracle's 8-bit factor storage (oracle/quant.py): hand-derived codes, the rounding bound of
asymmetric quantisation, the exact identity of the folded scales, and decode over the 8-bit factors
against plain attention over the dequantized keys and values."""
import numpy as np
import pytest

import oracle
from milo_testutil import stored_layer
from synth import WORKLOADS, from_storage, gen_layer


def test_codes_hand_example():
    # lo = -1, hi = 3: a = 4/255; (0 + 1)/a = 63.75 rounds to 64, so codes -128, 64 - 128, 127
    c, a, lo = oracle.quantize_channel([-1.0, 0.0, 3.0])
    assert list(c) == [-128, -64, 127]
    assert a == np.float32(4.0) / np.float32(255.0) and lo == -1.0


def test_codes_of_a_ramp_are_exact():
    # 256 equally spaced values 0, 0.5, ..., 127.5: a = 0.5 and every value is a code point
    x = 0.5 * np.arange(256)
    c, a, lo = oracle.quantize_channel(x)
    assert a == 0.5 and lo == 0.0
    assert np.array_equal(c.astype(int), np.arange(256) - 128)
    assert np.array_equal(oracle.dequantize_channel(c, a, lo), x)


def test_round_half_to_even():
    # lo = 0, hi = 255: a = 1, so x = 2.5 and 3.5 sit exactly between two codes
    c, a, _ = oracle.quantize_channel([0.0, 2.5, 3.5, 255.0])
    assert a == 1.0 and list(c) == [-128, 2 - 128, 4 - 128, 127]


def test_constant_channel():
    c, a, lo = oracle.quantize_channel(np.full(7, -0.375))
    assert a == 0.0 and np.all(c == -128)
    assert np.all(oracle.dequantize_channel(c, a, lo) == -0.375)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_extremes_and_rounding_bound(seed):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(512) * 3.0).astype(np.float32)
    c, a, lo = oracle.quantize_channel(x)
    assert c[np.argmin(x)] == -128 and c[np.argmax(x)] == 127
    err = np.abs(oracle.dequantize_channel(c, a, lo) - x.astype(np.float64))
    # round to nearest: within half a step (plus the fp32 rounding of (x - lo)/a)
    assert err.max() <= 0.5 * float(a) * (1 + 1e-5) + 1e-6 * float(np.abs(x).max())


def test_folded_scales_reproduce_the_dequantized_block():
    rng = np.random.default_rng(3)
    n, r, d = 256, 9, 64
    u = rng.standard_normal((n, r)) * rng.uniform(0.1, 10, r)
    b = np.linalg.qr(rng.standard_normal((d, r)))[0]
    q = oracle.quantize_block(u, b)
    assert q["U_aug"].shape == (n, r + 1) and q["B_aug"].shape == (d, r + 1)
    assert np.all(q["U_aug"][:, r] == 1.0)
    lhs = q["U_aug"] @ q["B_aug"].T
    rhs = q["u_hat"] @ b.T
    assert np.allclose(lhs, rhs, rtol=0, atol=1e-12 * np.abs(rhs).max())
    # and the dequantized factor is within half a step of the original, channel by channel
    assert np.all(np.abs(q["u_hat"] - u) <= 0.5 * q["scale"].astype(np.float64) * (1 + 1e-5) + 1e-5)


def _quantized_tiny(beta=None):
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    K, V = from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype)
    beta = wl.budgets[0] if beta is None else beta
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min), "bf16")
    return wl, L, lay, oracle.quantize_layer(lay)


def test_symmetric_codes_hand_example():
    # max |x| = 2: a = 2/127; 1/a = 63.5 rounds to 64 (half to even), 0.5/a = 31.75 rounds to 32
    c, a = oracle.quantize_channel_symmetric([-2.0, 1.0, 0.5, 2.0])
    assert list(c) == [-127, 64, 32, 127]
    assert a == np.float32(2.0) / np.float32(127.0)
    c, a = oracle.quantize_channel_symmetric(np.zeros(5))
    assert a == 0.0 and np.all(c == 0)


def test_full_rank_block_takes_the_symmetric_form():
    rng = np.random.default_rng(4)
    n, d = 256, 16
    u = rng.standard_normal((n, d)) * rng.uniform(0.1, 10, d)
    b = np.linalg.qr(rng.standard_normal((d, d)))[0]
    q = oracle.quantize_block(u, b)
    assert q["U_aug"].shape == (n, d) and q["B_aug"].shape == (d, d)  # no extra component at rank d
    assert np.all(np.abs(q["codes"].astype(int)) <= 127)
    assert np.allclose(q["U_aug"] @ q["B_aug"].T, q["u_hat"] @ b.T, rtol=0, atol=1e-12 * np.abs(u).max())
    assert np.all(np.abs(q["u_hat"] - u) <= 0.5 * q["scale"].astype(np.float64) * (1 + 1e-5) + 1e-5)
    for j in range(d):  # the largest magnitude of each channel maps to ±127
        t = np.argmax(np.abs(u[:, j]))
        assert abs(int(q["codes"][t, j])) == 127


def test_quantized_layer_ranks_and_shapes():
    _, _, lay, ql = _quantized_tiny()
    for t in ("K", "V"):
        for p, qp in zip(lay[t], ql[t]):
            d = p["B"][0].shape[0]
            want = np.where(np.asarray(p["ranks"]) < d, np.asarray(p["ranks"]) + 1, np.asarray(p["ranks"]))
            assert np.array_equal(qp["ranks"], want)
            for u, qu, qb in zip(p["U"], qp["U"], qp["B"]):
                r = u.shape[1]
                extra = 1 if r < d else 0
                assert qu.shape == (u.shape[0], r + extra) and qb.shape[1] == r + extra
                assert np.all((qu[:, :r] >= -128) & (qu[:, :r] <= 127))
                if extra:
                    assert np.all(qu[:, -1] == 1)


@pytest.mark.parametrize("beta", [None, 0.75, 1.25])
def test_decode_over_8bit_factors_is_attention_over_dequantized_cache(beta):
    """Rank-space decode on (codes, folded B) equals plain softmax attention over the dense keys and values
    rebuilt from the dequantized token factors: a dropped zero-point column, a wrong sign of the offset or a
    scale on the wrong side changes the keys and fails this.  Budgets: every block below full rank
    (asymmetric), some blocks at full rank (both forms), every block at full rank (symmetric)."""
    wl, L, lay, ql = _quantized_tiny(beta)
    d = wl.head_dim
    full = sum(int(np.sum(np.asarray(p["ranks"]) == d)) for t in ("K", "V") for p in lay[t])
    print(f"budget {beta}: {full} blocks at full rank")
    q = from_storage(L["q"], wl.dtype)
    Ks, Vs = from_storage(L["K_suf"], wl.dtype), from_storage(L["V_suf"], wl.dtype)
    got = oracle.decode_attention(q, ql, Ks, Vs)
    Kd = np.stack([np.concatenate([uh @ b.T for uh, b in zip(qp["u_hat"], p["B"])]) for qp, p in zip(ql["K"], lay["K"])])
    Vd = np.stack([np.concatenate([uh @ b.T for uh, b in zip(qp["u_hat"], p["B"])]) for qp, p in zip(ql["V"], lay["V"])])
    want = oracle.decode_attention_dense(q, Kd, Vd, Ks, Vs)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-12)
    # and 8-bit storage moves the output only a little from the unquantized factors' decode
    base = oracle.decode_attention(q, lay, Ks, Vs)
    assert np.linalg.norm(got - base) <= 2e-2 * np.linalg.norm(base)
