"""GPU parity of the decode over pre-RoPE key factors (milo_decode_attn_rope) against the oracle.

Acceptance: relative L2 <= 5e-3 over the output and every row within ROW_FACTOR times that, the bf16 decode
bound: the rotated keys are rebuilt in fp32 and stored in bf16, the rounding a bf16 key cache has.
"""
import functools

import numpy as np
import pytest

import oracle
from milo_testutil import assert_close, from_torch, pack_factors, stored_layer, to_torch
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
TOL = 5e-3


@functools.lru_cache(maxsize=2)
def _layer(name, beta):
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    K, V = from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype)
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min), wl.dtype)
    ranks, tok, dim = pack_factors(lay, wl.dtype)
    f = milo.import_factors(milo.BF16, wl.kv_heads, wl.context, wl.head_dim, wl.block_size, wl.r_min, ranks, tok,
                            dim)
    return wl, L, lay, f


def _check(name, beta, theta, batch=None, suffix=None, mask=None, sample=None):
    import decode_attention_milo_b200 as milo
    wl, L, lay, f = _layer(name, beta)
    q, Ks, Vs = L["q"], L["K_suf"], L["V_suf"]
    if batch is not None:
        q, Ks, Vs = q[:batch], Ks[:batch], Vs[:batch]
    if suffix is not None:
        Ks, Vs = Ks[:, :, :suffix], Vs[:, :, :suffix]
    S = Ks.shape[2]
    out = from_torch(milo.decode_attn_rope(to_torch(q, "bf16"), f, to_torch(Ks, "bf16") if S else None,
                                           to_torch(Vs, "bf16") if S else None, theta=theta, block_mask=mask))
    code, bits = f.status()
    assert code == 0, bits
    idx = np.arange(q.shape[0]) if sample is None else np.asarray(sample)
    want = oracle.decode_attention_rope(from_storage(q[idx], "bf16"), lay, from_storage(Ks[idx], "bf16"),
                                        from_storage(Vs[idx], "bf16"), theta, block_mask=mask)
    assert_close(out[idx], want, TOL, f"rope {name} theta {theta} batch {batch} suffix {suffix}")


@pytest.mark.parametrize("name,theta", [("qwen2.5-0.5b-layer", 1e6), ("qwen2.5-7b-layer", 1e6),
                                        ("qwen2.5-7b-layer", 1e4)])
def test_rope_decode_matches_oracle(name, theta):
    _check(name, WORKLOADS[name].budgets[0], theta)


@pytest.mark.parametrize("batch,suffix", [(3, 7), (40, 100), (1, 0)])
def test_rope_decode_ragged_7b(batch, suffix):
    _check("qwen2.5-7b-layer", 0.5, 1e6, batch, suffix)


def test_rope_decode_with_selection_7b():
    wl = WORKLOADS["qwen2.5-7b-layer"]
    mask = np.random.default_rng(11).random((wl.kv_heads, wl.num_blocks)) < 0.4
    _check("qwen2.5-7b-layer", 0.5, 1e6, mask=mask)


def test_rope_decode_32b_stack_layer():
    """Blocks of 1024 tokens, 65 536 positions, GQA 5, three row tiles, suffix 512 (queries at both ends of
    every row tile checked)."""
    wl = WORKLOADS["qwen2.5-32b-stack"]
    ipt = min(wl.batch, 128 // wl.group)
    sample = sorted({t for t0 in range(0, wl.batch, ipt) for t in (t0, min(wl.batch, t0 + ipt) - 1)})
    _check("qwen2.5-32b-stack", 0.5, 1e6, sample=sample)


def test_rope_and_plain_decode_alternate_on_one_object():
    """The plan is rebuilt when the mode changes: a rank-space decode between two rotated ones stays right."""
    import decode_attention_milo_b200 as milo
    wl, L, lay, f = _layer("qwen2.5-0.5b-layer", 0.5)
    q, Ks, Vs = (to_torch(L[k], "bf16") for k in ("q", "K_suf", "V_suf"))
    a = from_torch(milo.decode_attn_rope(q, f, Ks, Vs, theta=1e6))
    plain = from_torch(milo.decode_attn(q, f, Ks, Vs))
    b = from_torch(milo.decode_attn_rope(q, f, Ks, Vs, theta=1e6))
    assert np.array_equal(a, b)
    want = oracle.decode_attention(from_storage(L["q"], "bf16"), lay, from_storage(L["K_suf"], "bf16"),
                                   from_storage(L["V_suf"], "bf16"))
    assert_close(plain, want, TOL, "plain decode between rotated ones")
