"""GPU parity of milo_decode_attn against the oracle, fed the oracle's own stored factors.

Acceptance: relative L2 over the whole output <= 1e-5 (fp32) and <= 5e-3 (bf16), the
bounds stated for decode fed the oracle's factors.
"""
import numpy as np
import pytest

import oracle
from milo_testutil import from_torch, pack_factors, rel_l2, stored_layer, to_torch
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-5, "bf16": 5e-3}


def _setup(name, beta=None, batch=None, suffix=None, q_scale=1.0, seed_override=None):
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    beta = wl.budgets[0] if beta is None else beta
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min), dt)
    q = L["q"]
    Ks, Vs = L["K_suf"], L["V_suf"]
    if batch is not None and batch > q.shape[0]:
        # more queries than the workload draws: append sign-flipped, rescaled copies (distinct rows, each
        # with its own copy of a suffix)
        from synth import to_storage
        reps = -(-batch // q.shape[0])
        qf = from_storage(q, dt)
        q = to_storage(np.concatenate([qf * (-0.6) ** k for k in range(reps)]), dt)
        Ks, Vs = np.concatenate([Ks] * reps), np.concatenate([Vs] * reps)
    if batch is not None:
        q, Ks, Vs = q[:batch], Ks[:batch], Vs[:batch]
    if suffix is not None:
        Ks, Vs = Ks[:, :, :suffix], Vs[:, :, :suffix]
    if q_scale != 1.0:
        from synth import to_storage
        q = to_storage(from_storage(q, dt) * q_scale, dt)
    ranks, tok, dim = pack_factors(lay, dt)
    f = milo.import_factors(milo.F32 if dt == "f32" else milo.BF16, wl.kv_heads, wl.context, wl.head_dim,
                            wl.block_size, wl.r_min, ranks, tok, dim)
    return wl, dt, lay, f, q, Ks, Vs


def _run(wl, dt, lay, f, q, Ks, Vs, scale=0.0):
    import decode_attention_milo_b200 as milo
    tq = to_torch(q, dt)
    S = Ks.shape[2]
    tks = to_torch(Ks, dt) if S else None
    tvs = to_torch(Vs, dt) if S else None
    out = from_torch(milo.decode_attn(tq, f, tks, tvs, scale=scale))
    code, bits = f.status()
    assert code == 0, bits
    want = oracle.decode_attention(from_storage(q, dt), lay, from_storage(Ks, dt), from_storage(Vs, dt),
                                   scale=scale)
    return out, want


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_decode_matches_oracle(name):
    wl, dt, lay, f, q, Ks, Vs = _setup(name)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert rel_l2(out, want) <= TOL[dt]


def test_decode_sharp_softmax_7b():
    """q scaled so the logits have std ~4: exercises the running-max rescaling."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", q_scale=60.0)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert rel_l2(out, want) <= TOL[dt]


@pytest.mark.parametrize("batch,suffix", [(1, 0), (3, 7), (16, 0), (5, 129)])
def test_decode_ragged_shapes_7b(batch, suffix):
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", batch=batch, suffix=suffix)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert rel_l2(out, want) <= TOL[dt]


@pytest.mark.parametrize("batch,suffix", [(40, 100), (19, 0)])
def test_decode_several_row_tiles_7b(batch, suffix):
    """More query rows than one 128-row tile per KV head (GQA group 7: 18 queries per tile)."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", batch=batch, suffix=suffix)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert rel_l2(out, want) <= TOL[dt]


def test_decode_explicit_scale_tiny():
    wl, dt, lay, f, q, Ks, Vs = _setup("tiny")
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, scale=0.75)
    assert rel_l2(out, want) <= TOL[dt]


@pytest.mark.parametrize("beta", [0.0 + 4 * (512 + 128) * 64 / (32768 * 128), 1.25])
def test_decode_extreme_budgets_7b(beta):
    """All blocks at r_min, and all blocks at full rank d."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", beta=beta, batch=4, suffix=32)
    ranks = lay["K"][0]["ranks"]
    assert np.all(ranks == 4) or np.all(ranks == 128)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert rel_l2(out, want) <= TOL[dt]
