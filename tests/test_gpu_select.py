"""GPU parity of block selection (milo_decode_attn_select) against the oracle.

MILO §4.4: at decode time the selected blocks are retrieved and attended sparsely.  The selection
is a [H][nb] mask per KV head, shared by every query of the head; the decode skips the blocks
it leaves out through its work list.  Fed the oracle's stored factors, the output is held to the
decode bound (relative L2 5e-3 bf16, every row within 4x of it).
"""
import functools

import numpy as np
import pytest

import oracle
from milo_testutil import assert_close, from_torch, pack_factors, stored_layer, to_torch
from synth import WORKLOADS, from_storage, gen_layer

pytestmark = pytest.mark.gpu
TOL = 5e-3


@functools.lru_cache(maxsize=1)
def _setup(name):
    import decode_attention_milo_b200 as milo
    wl = WORKLOADS[name]
    L = gen_layer(wl)
    dt = wl.dtype
    K, V = from_storage(L["K"], dt), from_storage(L["V"], dt)
    lay = stored_layer(oracle.compress_layer(K, V, wl.block_size, wl.budgets[0], wl.r_min), dt)
    ranks, tok, dim = pack_factors(lay, dt)
    f = milo.import_factors(milo.BF16, wl.kv_heads, wl.context, wl.head_dim, wl.block_size, wl.r_min, ranks, tok,
                            dim)
    return wl, L, lay, f


def _masks(wl):
    rng = np.random.default_rng(31 + wl.wid)
    H, nb = wl.kv_heads, wl.num_blocks
    one = np.zeros((H, nb), dtype=bool)
    one[np.arange(H), rng.integers(0, nb, size=H)] = True
    return {"half": rng.uniform(size=(H, nb)) < 0.5,
            "one block": one,
            "tail": np.arange(nb)[None, :].repeat(H, 0) >= nb - 3,
            "none": np.zeros((H, nb), dtype=bool)}


@pytest.mark.parametrize("which", ["half", "one block", "tail", "none"])
def test_select_matches_oracle_7b(which):
    import decode_attention_milo_b200 as milo
    wl, L, lay, f = _setup("qwen2.5-7b-layer")
    dt = wl.dtype
    mask = _masks(wl)[which]
    q, ks, vs = to_torch(L["q"], dt), to_torch(L["K_suf"], dt), to_torch(L["V_suf"], dt)
    got = from_torch(milo.decode_attn_select(q, f, mask, ks, vs))
    assert f.status()[0] == 0
    want = oracle.decode_attention(from_storage(L["q"], dt), lay, from_storage(L["K_suf"], dt),
                                   from_storage(L["V_suf"], dt), block_mask=mask)
    assert_close(got, want, TOL, f"select {which}")


def test_select_all_blocks_equals_decode_attn_and_masks_can_change():
    """Selecting every block gives milo_decode_attn's output bit for bit; alternating masks on one factor object
    rebuilds the work list each time and stays correct."""
    import torch

    import decode_attention_milo_b200 as milo
    wl, L, lay, f = _setup("qwen2.5-7b-layer")
    dt = wl.dtype
    q, ks, vs = to_torch(L["q"], dt), to_torch(L["K_suf"], dt), to_torch(L["V_suf"], dt)
    full = milo.decode_attn_select(q, f, np.ones((wl.kv_heads, wl.num_blocks), dtype=bool), ks, vs)
    plain = milo.decode_attn(q, f, ks, vs)
    torch.cuda.synchronize()
    assert torch.equal(full, plain)
    masks = _masks(wl)
    for which in ("half", "tail", "half"):
        got = from_torch(milo.decode_attn_select(q, f, masks[which], ks, vs))
        want = oracle.decode_attention(from_storage(L["q"], dt), lay, from_storage(L["K_suf"], dt),
                                       from_storage(L["V_suf"], dt), block_mask=masks[which])
        assert_close(got, want, TOL, f"select {which} again")


def test_select_without_suffix_rejects_an_empty_head():
    import decode_attention_milo_b200 as milo
    wl, L, lay, f = _setup("qwen2.5-7b-layer")
    dt = wl.dtype
    mask = np.ones((wl.kv_heads, wl.num_blocks), dtype=bool)
    mask[1] = False
    with pytest.raises(milo.MiloError) as exc:
        milo.decode_attn_select(to_torch(L["q"], dt), f, mask)
    assert exc.value.code == 1
