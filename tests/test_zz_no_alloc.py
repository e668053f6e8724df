"""milo_decode_attn_noalloc: the decode for callers that cannot allocate device memory.

Such callers (a serving engine whose allocator owns all device memory and forbids side
allocations; a latency-critical path that cannot take the device-wide synchronisation of
cudaMalloc) get an entry point that keeps its work list and partials in one fixed device
array instead of allocating them.  These tests call it through the C ABI and check it
against milo_decode_attn on the same inputs, two calls in a row: both run the same kernels
on the same work list, so the outputs must be identical bit for bit.  One test also checks
it directly against the oracle, and one runs a large shape and then a smaller one with
another head dimension, to show that nothing left in the shared array leaks into a later
call.

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest

import oracle
from milo_testutil import assert_close, from_torch, pack_factors, stored_layer, to_torch
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
TOL = 5e-3  # relative L2 of the bf16 decode fed the oracle's factors


def _compressed(name):
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    dt = wl.dtype
    L = gen_layer(wl)
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, wl.budgets[0], wl.r_min)
    return wl, dt, L, f


def test_noalloc_matches_decode_attn_on_two_calls():
    import torch

    import decode_attention_milo_b200 as milo
    wl, dt, L, f = _compressed("qwen2.5-7b-layer")
    ks, vs = to_torch(L["K_suf"], dt), to_torch(L["V_suf"], dt)
    q1 = to_torch(L["q"], dt)
    q2 = (q1.float() * -0.75).to(torch.bfloat16).contiguous()  # a second, different query batch
    out1, out2 = torch.empty_like(q1), torch.empty_like(q2)
    # two calls in a row on a factor object that was never decoded before
    milo.decode_attn_noalloc(q1, f, ks, vs, out=out1)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    milo.decode_attn_noalloc(q2, f, ks, vs, out=out2)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before  # the call itself took no device memory
    assert f.status()[0] == 0
    want1 = milo.decode_attn(q1, f, ks, vs)
    want2 = milo.decode_attn(q2, f, ks, vs)
    torch.cuda.synchronize()
    assert f.status()[0] == 0
    assert torch.equal(out1, want1)
    assert torch.equal(out2, want2)
    assert not torch.equal(out1, out2)


def test_noalloc_matches_oracle():
    """Fed the oracle's own stored factors, the no-alloc decode is held to the decode bound directly."""
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS["qwen2.5-7b-layer"]
    dt = wl.dtype
    L = gen_layer(wl)
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, wl.budgets[0], wl.r_min), dt)
    ranks, tok, dim = pack_factors(lay, dt)
    f = milo.import_factors(milo.BF16, wl.kv_heads, wl.context, wl.head_dim, wl.block_size, wl.r_min, ranks,
                            tok, dim)
    got = from_torch(milo.decode_attn_noalloc(to_torch(L["q"], dt), f, to_torch(L["K_suf"], dt),
                                              to_torch(L["V_suf"], dt)))
    assert f.status()[0] == 0
    want = oracle.decode_attention(from_storage(L["q"], dt), lay, from_storage(L["K_suf"], dt),
                                   from_storage(L["V_suf"], dt))
    assert_close(got, want, TOL, "noalloc vs oracle")


def test_noalloc_large_then_small_shape():
    """A large call (7B layer, d = 128) and then a smaller one (0.5B layer, d = 64) through the same array,
    each identical to milo_decode_attn."""
    import torch

    import decode_attention_milo_b200 as milo
    for name in ("qwen2.5-7b-layer", "qwen2.5-0.5b-layer", "qwen2.5-7b-layer"):
        wl, dt, L, f = _compressed(name)
        q, ks, vs = to_torch(L["q"], dt), to_torch(L["K_suf"], dt), to_torch(L["V_suf"], dt)
        got = milo.decode_attn_noalloc(q, f, ks, vs)
        want = milo.decode_attn(q, f, ks, vs)
        torch.cuda.synchronize()
        assert f.status()[0] == 0
        assert torch.equal(got, want), name
        f.close()


def test_noalloc_rejects_shapes_beyond_its_array():
    import torch

    import decode_attention_milo_b200 as milo
    wl, dt, L, f = _compressed("qwen2.5-7b-layer")
    q = torch.zeros((4096, wl.q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(milo.MiloError) as exc:
        milo.decode_attn_noalloc(q, f)
    assert exc.value.code == 2  # MILO_ERR_UNSUPPORTED: work list and partials exceed the fixed array
