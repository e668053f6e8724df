"""milo_decode_attn_noalloc: the decode for callers that cannot allocate device memory.

Such callers (code running while a stream is captured in global mode, where cudaMalloc is not
allowed; engines whose allocator owns all device memory) get an entry point that keeps its work
list and partials in one fixed device array instead of allocating them.  These tests call it
through the C ABI and check it against milo_decode_attn on the same inputs, two calls in a row,
within the bf16 decode tolerance used by the other decode tests.

The file name sorts last so that a run stopping at the first failure has run every other test.
"""
import numpy as np
import pytest

from milo_testutil import from_torch, rel_l2, to_torch
from synth import WORKLOADS, gen_layer

pytestmark = pytest.mark.gpu
TOL = 5e-3  # relative L2 of the bf16 decode


def _layer():
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS["qwen2.5-7b-layer"]
    dt = wl.dtype
    L = gen_layer(wl)
    f = milo.compress(to_torch(L["K"], dt), to_torch(L["V"], dt), wl.block_size, wl.budgets[0], wl.r_min)
    return wl, dt, L, f


def test_noalloc_matches_decode_attn_on_two_calls():
    import torch

    import decode_attention_milo_b200 as milo
    wl, dt, L, f = _layer()
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
    got1, got2 = from_torch(out1), from_torch(out2)
    want1 = from_torch(milo.decode_attn(q1, f, ks, vs))
    want2 = from_torch(milo.decode_attn(q2, f, ks, vs))
    assert f.status()[0] == 0
    assert rel_l2(got1, want1) <= TOL
    assert rel_l2(got2, want2) <= TOL
    assert not np.allclose(got1, got2)


def test_noalloc_rejects_shapes_beyond_its_array():
    import torch

    import decode_attention_milo_b200 as milo
    wl, dt, L, f = _layer()
    q = torch.zeros((4096, wl.q_heads, wl.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(milo.MiloError) as exc:
        milo.decode_attn_noalloc(q, f)
    assert exc.value.code == 2  # MILO_ERR_UNSUPPORTED: work list and partials exceed the fixed array
