"""The seeded generator: reproducible, shaped like the workloads, exact noise-free spectra."""
import numpy as np
import pytest
import torch

from synth import WORKLOADS, block_taus, f64_to_bf16_bits, gen_block_f64, gen_layer, gen_queries


def test_block_reproducible_and_independent():
    wl = WORKLOADS["qwen2.5-0.5b-layer"]
    a = gen_block_f64(wl, 0, 1, 0, 5, 4.0)
    b = gen_block_f64(wl, 0, 1, 0, 5, 4.0)
    c = gen_block_f64(wl, 0, 1, 0, 6, 4.0)
    assert np.array_equal(a, b)
    assert not np.allclose(a, c)
    assert a.shape == (wl.block_size, wl.head_dim)


def test_noise_free_spectrum_is_exact():
    wl = WORKLOADS["qwen2.5-7b-layer"]
    x = gen_block_f64(wl, 0, 0, 0, 3, 7.5, noise_std=0.0)
    s = np.linalg.svd(x, compute_uv=False)
    k = wl.signal_rank
    want = np.exp(-np.arange(1, k + 1) / 7.5)
    assert np.allclose(s[:k], want, rtol=1e-12, atol=1e-14)
    assert np.all(s[k:] < 1e-13)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_tau_ranges(name):
    wl = WORKLOADS[name]
    t = block_taus(wl, 0, 0)
    assert t.shape == (wl.num_blocks,)
    kind = wl.tau[0]
    if kind == "fixed":
        assert list(t[:4]) == [2.0, 4.0, 8.0, 16.0]
    elif kind == "bimodal":
        assert np.sum((t >= 1.0) & (t <= 4.0)) == wl.num_blocks // 2
        assert np.sum((t >= 32.0) & (t <= 96.0)) == wl.num_blocks - wl.num_blocks // 2
    else:
        assert t.min() >= wl.tau[1] and t.max() <= wl.tau[2]


def test_bf16_cast_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(10000) * 10.0 ** rng.integers(-6, 6, 10000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e38]])
    mine = f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)


def test_tiny_layer_shapes():
    wl = WORKLOADS["tiny"]
    L = gen_layer(wl)
    assert L["K"].shape == (1, 1024, 64) and L["K"].dtype == np.float32
    assert L["q"].shape == (1, 2, 64)
    assert L["K_suf"].shape == (1, 1, 0, 64)
    q = gen_queries(wl, 0)
    assert abs(q.std() - 1.0) < 0.3


def test_token_slab_packing_roundtrip():
    import sys, os
    sys.path.insert(0, os.path.dirname(__file__))
    from milo_testutil import tok_slabs, untok_slabs
    rng = np.random.default_rng(2)
    u = rng.standard_normal((512, 37))
    flat = tok_slabs(u)
    assert flat.shape == (4 * 37, 128)
    # element (j, t) sits at (t // 128) * (r * 128) + j * 128 + t % 128
    j, t = 11, 300
    assert flat.reshape(-1)[(t // 128) * 37 * 128 + j * 128 + t % 128] == u[t, j]
    assert np.array_equal(untok_slabs(flat.reshape(-1), 512, 37), u)
