"""GPU parity of milo_decode_attn against the oracle, fed the oracle's own stored factors.

Acceptance: relative L2 over the whole output <= 1e-5 (fp32) and <= 5e-3 (bf16), the
bounds stated for decode fed the oracle's factors, and every output row (one query and
head) within ROW_FACTOR times that bound.

The stacked workloads (Qwen2.5-7B and -32B shapes) decode one full layer on the GPU, with
the whole batch and suffix, and are checked on a sample of queries that spans every row
tile (the oracle computes those rows one by one).
"""
import functools

import numpy as np
import pytest

import oracle
from milo_testutil import assert_close, from_torch, pack_factors, stored_layer, to_torch
from synth import WORKLOADS, from_storage, gen_layer, to_storage

pytestmark = pytest.mark.gpu
TOL = {"f32": 1e-5, "bf16": 5e-3}


@functools.lru_cache(maxsize=2)
def _layer(name):
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    dt = wl.dtype
    return wl, L, from_storage(L["K"], dt), from_storage(L["V"], dt)


@functools.lru_cache(maxsize=3)
def _oracle_layer(name, beta):
    wl, L, K, V = _layer(name)
    return stored_layer(oracle.compress_layer(K, V, wl.block_size, beta, wl.r_min), wl.dtype)


def _setup(name, beta=None, batch=None, suffix=None, q_scale=1.0):
    import decode_attention_milo_b200 as milo
    wl, L, _, _ = _layer(name)
    dt = wl.dtype
    beta = wl.budgets[0] if beta is None else beta
    lay = _oracle_layer(name, beta)
    q = L["q"]
    Ks, Vs = L["K_suf"], L["V_suf"]
    if batch is not None and batch > q.shape[0]:
        # more queries than the workload draws: append sign-flipped, rescaled copies (distinct rows, each
        # with its own copy of a suffix)
        reps = -(-batch // q.shape[0])
        qf = from_storage(q, dt)
        q = to_storage(np.concatenate([qf * (-0.6) ** k for k in range(reps)]), dt)
        Ks, Vs = np.concatenate([Ks] * reps), np.concatenate([Vs] * reps)
    if batch is not None:
        q, Ks, Vs = q[:batch], Ks[:batch], Vs[:batch]
    if suffix is not None:
        Ks, Vs = Ks[:, :, :suffix], Vs[:, :, :suffix]
    if q_scale != 1.0:
        q = to_storage(from_storage(q, dt) * q_scale, dt)
    ranks, tok, dim = pack_factors(lay, dt)
    f = milo.import_factors(milo.F32 if dt == "f32" else milo.BF16, wl.kv_heads, wl.context, wl.head_dim,
                            wl.block_size, wl.r_min, ranks, tok, dim)
    return wl, dt, lay, f, q, Ks, Vs


def _run(wl, dt, lay, f, q, Ks, Vs, scale=0.0, sample=None):
    """GPU decode of the whole batch; the oracle on the queries in `sample` (all when None)."""
    import decode_attention_milo_b200 as milo
    tq = to_torch(q, dt)
    S = Ks.shape[2]
    tks = to_torch(Ks, dt) if S else None
    tvs = to_torch(Vs, dt) if S else None
    out = from_torch(milo.decode_attn(tq, f, tks, tvs, scale=scale))
    code, bits = f.status()
    assert code == 0, bits
    idx = np.arange(q.shape[0]) if sample is None else np.asarray(sample)
    want = oracle.decode_attention(from_storage(q[idx], dt), lay, from_storage(Ks[idx], dt),
                                   from_storage(Vs[idx], dt), scale=scale)
    return out[idx], want


def _tile_sample(wl, batch):
    """Queries at the first and last item of every row tile (GQA group G: 128 // G queries per tile)."""
    ipt = min(batch, 128 // wl.group)
    s = set()
    for t0 in range(0, batch, ipt):
        s |= {t0, min(batch, t0 + ipt) - 1}
    return sorted(s)


@pytest.mark.parametrize("name", ["tiny", "qwen2.5-0.5b-layer", "qwen2.5-7b-layer"])
def test_decode_matches_oracle(name):
    wl, dt, lay, f, q, Ks, Vs = _setup(name)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], name)


@pytest.mark.parametrize("name,q_scale", [("qwen2.5-7b-layer", 60.0), ("qwen2.5-0.5b-layer", 60.0)])
def test_decode_sharp_softmax(name, q_scale):
    """q scaled so the logits have std ~4: exercises the running-max rescaling (d = 128 and d = 64)."""
    wl, dt, lay, f, q, Ks, Vs = _setup(name, q_scale=q_scale)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], f"{name} q x {q_scale}")


@pytest.mark.parametrize("batch,suffix", [(1, 0), (3, 7), (16, 0), (5, 129)])
def test_decode_ragged_shapes_7b(batch, suffix):
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", batch=batch, suffix=suffix)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], f"batch {batch} suffix {suffix}")


@pytest.mark.parametrize("batch,suffix", [(3, 7), (8, 0)])
def test_decode_ragged_shapes_d64(batch, suffix):
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-0.5b-layer", batch=batch, suffix=suffix)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], f"d=64 batch {batch} suffix {suffix}")


@pytest.mark.parametrize("batch,suffix", [(40, 100), (19, 0)])
def test_decode_several_row_tiles_7b(batch, suffix):
    """More query rows than one 128-row tile per KV head (GQA group 7: 18 queries per tile)."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", batch=batch, suffix=suffix)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], f"batch {batch} suffix {suffix}")


def test_decode_explicit_scale_tiny():
    wl, dt, lay, f, q, Ks, Vs = _setup("tiny")
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, scale=0.75)
    assert_close(out, want, TOL[dt], "tiny scale 0.75")


@pytest.mark.parametrize("beta", [0.0 + 4 * (512 + 128) * 64 / (32768 * 128), 1.25])
def test_decode_extreme_budgets_7b(beta):
    """All blocks at r_min, and all blocks at full rank d."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", beta=beta, batch=4, suffix=32)
    ranks = lay["K"][0]["ranks"]
    assert np.all(ranks == 4) or np.all(ranks == 128)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs)
    assert_close(out, want, TOL[dt], f"beta {beta:.4f}")


def test_decode_7b_stack_layer():
    """One layer of the Qwen2.5-7B stack: 256 blocks of 512, batch 32 (two row tiles per KV head), suffix 256."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-stack")
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, sample=_tile_sample(wl, wl.batch))
    assert_close(out, want, TOL[dt], "7b stack layer")


@pytest.mark.parametrize("beta", [0.25, 0.5, 0.75])
def test_decode_32b_stack_layer(beta):
    """One layer of the Qwen2.5-32B stack: blocks of 1024 (8 chunks each), 8 KV / 40 query heads (GQA 5:
    25 queries per row tile, three tiles), batch 64, suffix 512."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-32b-stack", beta=beta)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, sample=_tile_sample(wl, wl.batch))
    assert_close(out, want, TOL[dt], f"32b stack layer beta {beta}")


def test_decode_32b_stack_sharp_softmax():
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-32b-stack", beta=0.5, q_scale=60.0)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, sample=_tile_sample(wl, wl.batch))
    assert_close(out, want, TOL[dt], "32b stack layer q x 60")


def test_decode_large_batch_7b():
    """A batch of 300 queries with 256-token suffixes: 17 row tiles per KV head and some 1200 suffix segments,
    more segments than a CTA's staged work record holds, so that CTAs also read the global segment tables."""
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer", batch=300)
    out, want = _run(wl, dt, lay, f, q, Ks, Vs, sample=[0, 17, 18, 151, 287, 288, 299])
    assert_close(out, want, TOL[dt], "batch 300")


def test_back_to_back_calls_with_inputs_written_just_before():
    """Each call's q is written by a kernel right before it on the same stream, and the calls follow each
    other with no synchronisation (the decode is launched as a programmatic dependent of the kernel before
    it, and reuses the partials the previous call's combine reads): twelve such calls equal the same calls
    run one at a time."""
    import torch
    import decode_attention_milo_b200 as milo
    wl, dt, lay, f, q, Ks, Vs = _setup("qwen2.5-7b-layer")
    tq, tk, tv = to_torch(q, dt), to_torch(Ks, dt), to_torch(Vs, dt)
    scales = [1.0 + 0.25 * k for k in range(12)]
    ref = []
    for sc in scales:
        qq = tq * sc
        torch.cuda.synchronize()
        ref.append(milo.decode_attn(qq, f, tk, tv))
        torch.cuda.synchronize()
    buf = torch.empty_like(tq)
    outs = []
    for sc in scales:
        torch.mul(tq, sc, out=buf)  # a kernel that writes q right before the decode on the same stream
        outs.append(milo.decode_attn(buf, f, tk, tv))
    torch.cuda.synchronize()
    for k, (a, b) in enumerate(zip(outs, ref)):
        assert torch.equal(a, b), k
    assert f.status()[0] == 0
