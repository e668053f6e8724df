"""Pins of the oracle's decode attention: brute force, library softmax attention, closed forms."""
import math

import numpy as np
import pytest
import torch

import oracle
from synth import WORKLOADS, from_storage, gen_layer, gen_queries


def _brute_force(q, K, V, K_suf, V_suf, scale):
    """Pure-Python loops: softmax over prefix ∪ suffix with math.exp, one query row at a time."""
    Bq, Hq, d = q.shape
    H = K.shape[0]
    G = Hq // H
    out = np.zeros_like(q)
    for i in range(Bq):
        for hq in range(Hq):
            h = hq // G
            keys = list(K[h]) + list(K_suf[i, h])
            vals = list(V[h]) + list(V_suf[i, h])
            s = [scale * sum(float(a) * float(b) for a, b in zip(q[i, hq], k)) for k in keys]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            tot = sum(e)
            for c in range(d):
                out[i, hq, c] = sum(ej * float(v[c]) for ej, v in zip(e, vals)) / tot
    return out


def _sdpa(q, K, V, K_suf, V_suf, scale):
    """torch's scaled_dot_product_attention in fp64 on CPU, one (query, head) at a time."""
    Bq, Hq, d = q.shape
    H = K.shape[0]
    G = Hq // H
    out = np.zeros_like(q)
    for i in range(Bq):
        for hq in range(Hq):
            h = hq // G
            k = torch.from_numpy(np.concatenate([K[h], K_suf[i, h]]))[None, None]
            v = torch.from_numpy(np.concatenate([V[h], V_suf[i, h]]))[None, None]
            qq = torch.from_numpy(q[i, hq])[None, None, None]
            out[i, hq] = torch.nn.functional.scaled_dot_product_attention(qq, k, v, scale=scale)[0, 0, 0].numpy()
    return out


def _tiny_inputs(suffix=0, batch=1):
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    K = from_storage(L["K"], "f32")
    V = from_storage(L["V"], "f32")
    q = from_storage(L["q"], "f32")
    rng = np.random.default_rng(5)
    if batch != 1:
        q = rng.standard_normal((batch, 2, 64))
    Ks = 0.01 * rng.standard_normal((batch, 1, suffix, 64))
    Vs = 0.01 * rng.standard_normal((batch, 1, suffix, 64))
    return wl, K, V, q, Ks, Vs


def test_rank_space_equals_brute_force_on_reconstruction():
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=24, batch=2)
    lay = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    Kr = oracle.reconstruct_pool(lay["K"][0])[None]
    Vr = oracle.reconstruct_pool(lay["V"][0])[None]
    scale = 1.0 / 8.0
    got = oracle.decode_attention(q, lay, Ks, Vs)
    want = _brute_force(q, Kr, Vr, Ks, Vs, scale)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-15)
    assert np.allclose(oracle.decode_attention_dense(q, Kr, Vr, Ks, Vs), want, rtol=1e-11, atol=1e-15)


def test_full_rank_compression_is_exact_attention():
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=8)
    beta = (wl.block_size + wl.head_dim) / wl.block_size  # R = nb * d
    lay = oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min)
    assert all(int(r) == 64 for r in lay["K"][0]["ranks"])
    got = oracle.decode_attention(q, lay, Ks, Vs)
    want = _sdpa(q, K, V, Ks, Vs, 1.0 / 8.0)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-14)


def test_sharp_scores_match_library_attention():
    """Large logits exercise the max subtraction; compare with torch's attention on the reconstruction."""
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=16)
    lay = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    Kr = oracle.reconstruct_pool(lay["K"][0])[None]
    Vr = oracle.reconstruct_pool(lay["V"][0])[None]
    scale = 4000.0
    got = oracle.decode_attention(q, lay, Ks, Vs, scale=scale)
    assert np.allclose(got, _sdpa(q, Kr, Vr, Ks, Vs, scale), rtol=1e-9, atol=1e-13)


def test_identical_keys_give_mean_of_values():
    wl = WORKLOADS["tiny"]
    rng = np.random.default_rng(11)
    key = rng.standard_normal(64)
    K = np.tile(key, (1, 1024, 1))
    V = rng.standard_normal((1, 1024, 64))
    Ks = np.tile(key, (1, 1, 5, 1))
    Vs = rng.standard_normal((1, 1, 5, 64))
    beta = 1.25
    lay = oracle.compress_layer(K, V, 256, beta, 4)
    q = rng.standard_normal((1, 2, 64))
    got = oracle.decode_attention(q, lay, Ks, Vs)
    mean = np.concatenate([V[0], Vs[0, 0]]).mean(axis=0)
    assert np.allclose(got[0, 0], mean, atol=1e-12) and np.allclose(got[0, 1], mean, atol=1e-12)


def test_dominant_token_returns_its_value():
    rng = np.random.default_rng(12)
    K = 1e-3 * rng.standard_normal((1, 512, 64))
    V = rng.standard_normal((1, 512, 64))
    q = rng.standard_normal((1, 1, 64))
    K[0, 300] = 50.0 * q[0, 0] / np.linalg.norm(q[0, 0])
    lay = oracle.compress_layer(K, V, 256, 1.25, 4)
    Ks = np.zeros((1, 1, 0, 64))
    got = oracle.decode_attention(q, lay, Ks, Ks)
    assert np.allclose(got[0, 0], V[0, 300], atol=1e-9)


def test_gqa_head_mapping_with_constant_values():
    """Constant values c_h on KV head h: every query head hq must return c_{hq // G} exactly."""
    rng = np.random.default_rng(13)
    H, G, d, T = 3, 4, 64, 512
    K = rng.standard_normal((H, T, d))
    consts = rng.standard_normal((H, d))
    V = np.broadcast_to(consts[:, None, :], (H, T, d)).copy()
    Ks = rng.standard_normal((2, H, 7, d))
    Vs = np.broadcast_to(consts[None, :, None, :], (2, H, 7, d)).copy()
    lay = oracle.compress_layer(K, V, 256, 0.5, 4)
    q = rng.standard_normal((2, H * G, d))
    got = oracle.decode_attention(q, lay, Ks, Vs)
    for hq in range(H * G):
        assert np.allclose(got[:, hq], consts[hq // G], atol=1e-12)


def test_scale_argument():
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=4)
    lay = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    a = oracle.decode_attention(q, lay, Ks, Vs, scale=0.0)
    b = oracle.decode_attention(q, lay, Ks, Vs, scale=1.0 / 8.0)
    c = oracle.decode_attention(q, lay, Ks, Vs, scale=0.5)
    assert np.array_equal(a, b)
    assert not np.allclose(b, c)


# ---------------------------------------------------------------- block selection (§4.4: selected blocks only)

def test_block_selection_equals_attention_over_the_selected_blocks():
    """Selecting blocks {0, 2} of four equals brute-force softmax over those blocks' reconstructed rows and
    the suffix; selecting every block equals the unmasked decode."""
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=12, batch=2)
    lay = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    n = wl.block_size
    Kr = oracle.reconstruct_pool(lay["K"][0])
    Vr = oracle.reconstruct_pool(lay["V"][0])
    mask = [[True, False, True, False]]
    rows = np.concatenate([np.arange(b * n, (b + 1) * n) for b in (0, 2)])
    got = oracle.decode_attention(q, lay, Ks, Vs, block_mask=mask)
    want = _brute_force(q, Kr[rows][None], Vr[rows][None], Ks, Vs, 1.0 / 8.0)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-15)
    every = oracle.decode_attention(q, lay, Ks, Vs, block_mask=[[True] * 4])
    assert np.array_equal(every, oracle.decode_attention(q, lay, Ks, Vs))


def test_block_selection_full_rank_is_exact_attention_on_the_selected_rows():
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=8)
    beta = (wl.block_size + wl.head_dim) / wl.block_size
    lay = oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min)
    n = wl.block_size
    got = oracle.decode_attention(q, lay, Ks, Vs, block_mask=[[False, True, False, False]])
    want = _sdpa(q, K[:, n:2 * n], V[:, n:2 * n], Ks, Vs, 1.0 / 8.0)
    assert np.allclose(got, want, rtol=1e-10, atol=1e-14)


def test_no_block_selected_leaves_the_suffix():
    wl, K, V, q, Ks, Vs = _tiny_inputs(suffix=5)
    lay = oracle.compress_layer(K, V, wl.block_size, 0.5, wl.r_min)
    got = oracle.decode_attention(q, lay, Ks, Vs, block_mask=[[False] * 4])
    want = _sdpa(q, K[:, :0], V[:, :0], Ks, Vs, 1.0 / 8.0)
    assert np.allclose(got, want, rtol=1e-12, atol=1e-15)
