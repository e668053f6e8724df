"""GPU parity of the 8-bit factor storage (milo_factors_quantize) and of the decode over it.

Acceptance: the int8 codes bit-exact against the oracle's quantiser applied to the GPU's own bf16 factors
(both sides take the integer decisions in fp32); the folded bf16 dimension factors within bf16 rounding of
the oracle's fp64 fold; and the decode over 8-bit factors within 5e-3 relative L2 (and ROW_FACTOR times that
per output row) of the oracle's decode over the same stored factors.
"""
import functools

import numpy as np
import pytest

import oracle
from milo_testutil import (assert_close, factor_arrays, from_torch, layer_from_arrays, pack_factors_8bit,
                           stored_layer, stored_layer_8bit, to_torch, untok_slabs)
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
TOL = 5e-3


@functools.lru_cache(maxsize=2)
def _layer(name):
    wl = WORKLOADS[name]
    return wl, gen_layer(wl)


@functools.lru_cache(maxsize=3)
def _oracle_8bit(name, beta):
    wl, L = _layer(name)
    K, V = from_storage(L["K"], wl.dtype), from_storage(L["V"], wl.dtype)
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min), "bf16")
    return stored_layer_8bit(oracle.quantize_layer(lay))


def _import_8bit(name, beta):
    import decode_attention_milo_b200 as milo
    wl, _ = _layer(name)
    ql = _oracle_8bit(name, beta)
    ranks, tok, dim = pack_factors_8bit(ql)
    f = milo.import_factors(milo.I8, wl.kv_heads, wl.context, wl.head_dim, wl.block_size, wl.r_min, ranks,
                            tok, dim)
    return ql, f


def _queries(name, batch=None, suffix=None):
    wl, L = _layer(name)
    q, Ks, Vs = L["q"], L["K_suf"], L["V_suf"]
    if batch is not None:
        q, Ks, Vs = q[:batch], Ks[:batch], Vs[:batch]
    if suffix is not None:
        Ks, Vs = Ks[:, :, :suffix], Vs[:, :, :suffix]
    return q, Ks, Vs


def _decode(f, q, Ks, Vs, dt="bf16", mask=None):
    import decode_attention_milo_b200 as milo
    S = Ks.shape[2]
    args = (to_torch(q, dt), f, to_torch(Ks, dt) if S else None, to_torch(Vs, dt) if S else None)
    out = milo.decode_attn(*args) if mask is None else milo.decode_attn_select(args[0], f, mask, *args[2:])
    code, bits = f.status()
    assert code == 0, bits
    return from_torch(out)


def _tile_sample(wl, batch):
    ipt = min(batch, 128 // wl.group)
    s = set()
    for t0 in range(0, batch, ipt):
        s |= {t0, min(batch, t0 + ipt) - 1}
    return sorted(s)


@pytest.mark.parametrize("name", ["qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_quantize_codes_bit_exact(name):
    import decode_attention_milo_b200 as milo
    wl, L = _layer(name)
    dt = wl.dtype
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, wl.budgets[0], wl.r_min)
    qf = milo.quantize(f)
    code, bits = qf.status()
    assert code == 0, bits
    got, gq = factor_arrays(f), factor_arrays(qf)
    assert gq["desc"]["dtype"] == milo.I8
    d = wl.head_dim
    want_ranks = np.where(got["ranks"] < d, got["ranks"] + 1, got["ranks"])
    assert np.array_equal(gq["ranks"], want_ranks)
    P, nb = got["ranks"].shape
    flat = np.concatenate([[0], np.cumsum(want_ranks.reshape(-1))])
    assert np.array_equal(gq["row_offsets"][:, :nb], flat[:-1].reshape(P, nb))
    assert np.array_equal(gq["row_offsets"][:, nb], flat[nb::nb])
    print(f"{name}: {int(np.sum(got['ranks'] == d))} of {P * nb} blocks at full rank (symmetric form)")
    ql = oracle.quantize_layer(layer_from_arrays(got))
    n = wl.block_size
    pools = [p for h in range(len(ql["K"])) for p in (ql["K"][h], ql["V"][h])]
    worst = 0.0
    for p, pool in enumerate(pools):
        for b in range(nb):
            r0, r1 = int(gq["row_offsets"][p, b]), int(gq["row_offsets"][p, b + 1])
            codes = untok_slabs(gq["codes"][r0 * n:r1 * n].astype(np.int64), n, r1 - r0)
            assert np.array_equal(codes, pool["U"][b].astype(np.int64)), (p, b)
            want = pool["B"][b].T  # (r+1) × d, fp64 fold of the GPU's own factors
            # bf16 rounding of the result, plus fp32 accumulation of the offset row over r terms
            src = layer_from_arrays(got)["K" if p % 2 == 0 else "V"][p // 2]["B"][b]
            off = pool["lo"][b].astype(np.float64) + 128.0 * pool["scale"][b].astype(np.float64)
            acc_bound = np.abs(src) @ np.abs(off)
            bound = 2.0 ** -8 * np.abs(want)
            if r1 - r0 > got["ranks"][p, b]:  # the asymmetric form's offset row, accumulated in fp32
                bound[-1] += 2.0 ** -20 * acc_bound
            err = np.abs(gq["dim"][r0:r1] - want)
            assert np.all(err <= bound + 1e-30), (p, b, float((err - bound).max()))
            worst = max(worst, float((err / np.maximum(np.abs(want), 1e-30)).max()))
    print(f"{name}: folded dimension factors, max relative deviation {worst:.2e}")


@pytest.mark.parametrize("name,batch,suffix", [("qwen2.5-0.5b-layer", None, None), ("qwen2.5-7b-layer", None, None),
                                               ("qwen2.5-7b-layer", 3, 7), ("qwen2.5-7b-layer", 40, 100)])
def test_decode_8bit_matches_oracle(name, batch, suffix):
    wl, _ = _layer(name)
    ql, f = _import_8bit(name, wl.budgets[0])
    q, Ks, Vs = _queries(name, batch, suffix)
    out = _decode(f, q, Ks, Vs)
    want = oracle.decode_attention(from_storage(q, "bf16"), ql, from_storage(Ks, "bf16"), from_storage(Vs, "bf16"))
    assert_close(out, want, TOL, f"8-bit {name} batch {batch} suffix {suffix}")


def test_decode_8bit_32b_stack_layer():
    """Blocks of 1024 tokens (8 chunks each), GQA 5, three row tiles, suffix 512, on 8-bit factors."""
    wl, _ = _layer("qwen2.5-32b-stack")
    ql, f = _import_8bit("qwen2.5-32b-stack", 0.5)
    q, Ks, Vs = _queries("qwen2.5-32b-stack")
    out = _decode(f, q, Ks, Vs)
    idx = _tile_sample(wl, wl.batch)
    want = oracle.decode_attention(from_storage(q[idx], "bf16"), ql, from_storage(Ks[idx], "bf16"),
                                   from_storage(Vs[idx], "bf16"))
    assert_close(out[idx], want, TOL, "8-bit 32b stack layer")


def test_end_to_end_8bit_7b():
    """GPU compress → GPU quantise → GPU decode, against the oracle's decode over the GPU's own 8-bit factors,
    and (looser, the quantisation error itself) against the oracle's decode over the unquantised factors."""
    import decode_attention_milo_b200 as milo
    wl, L = _layer("qwen2.5-7b-layer")
    dt = wl.dtype
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, wl.budgets[0], wl.r_min)
    qf = milo.quantize(f)
    q, Ks, Vs = _queries("qwen2.5-7b-layer")
    out = _decode(qf, q, Ks, Vs)
    qv, Kv, Vv = from_storage(q, dt), from_storage(Ks, dt), from_storage(Vs, dt)
    want = oracle.decode_attention(qv, layer_from_arrays(factor_arrays(qf)), Kv, Vv)
    assert_close(out, want, TOL, "8-bit end to end")
    base = oracle.decode_attention(qv, layer_from_arrays(factor_arrays(f)), Kv, Vv)
    rel = np.linalg.norm(out - base) / np.linalg.norm(base)
    print(f"8-bit storage vs bf16 factors, decode relative L2: {rel:.2e}")
    assert rel <= 2e-2


def test_select_and_noalloc_on_8bit_factors():
    import torch
    import decode_attention_milo_b200 as milo
    wl, _ = _layer("qwen2.5-7b-layer")
    ql, f = _import_8bit("qwen2.5-7b-layer", wl.budgets[0])
    q, Ks, Vs = _queries("qwen2.5-7b-layer")
    rng = np.random.default_rng(5)
    mask = rng.random((wl.kv_heads, wl.num_blocks)) < 0.5
    out = _decode(f, q, Ks, Vs, mask=mask)
    want = oracle.decode_attention(from_storage(q, "bf16"), ql, from_storage(Ks, "bf16"), from_storage(Vs, "bf16"),
                                   block_mask=mask)
    assert_close(out, want, TOL, "8-bit block selection")
    tq, tk, tv = to_torch(q, "bf16"), to_torch(Ks, "bf16"), to_torch(Vs, "bf16")
    a = milo.decode_attn(tq, f, tk, tv)
    b = milo.decode_attn_noalloc(tq, f, tk, tv)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_full_rank_8bit_0_5b():
    """Every block at rank d: every block takes the symmetric form (no extra component)."""
    import decode_attention_milo_b200 as milo
    wl, L = _layer("qwen2.5-0.5b-layer")
    dt = wl.dtype
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, 1.25, wl.r_min)
    assert np.all(f.ranks() == wl.head_dim)
    qf = milo.quantize(f)
    assert np.all(qf.ranks() == wl.head_dim)
    q, Ks, Vs = _queries("qwen2.5-0.5b-layer")
    out = _decode(qf, q, Ks, Vs)
    want = oracle.decode_attention(from_storage(q, dt), layer_from_arrays(factor_arrays(qf)), from_storage(Ks, dt),
                                   from_storage(Vs, dt))
    assert_close(out, want, TOL, "8-bit full rank")
