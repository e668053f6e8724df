"""The decode work list (host logic of the bf16 tensor-core decode), checked on CPU.

The decode of page "MILO" §4.4 visits every 128-token chunk of every compressed block once per
(KV head, row tile), and every chunk of every query's uncompressed suffix once per (query, KV head);
the work list cuts that sequence into one run per CTA.  These tests check, through the C ABI
(milo_decode_worklist, no GPU), that every chunk is covered exactly once and in order, that the
partial-slot ranges the combine step reads match the segments, and that the runs are contiguous.
"""
import numpy as np
import pytest

pytestmark = []

# (kv heads, q heads, head dim, block size, blocks, batch, suffix)
SHAPES = {
    "qwen2.5-0.5b-layer": (2, 14, 64, 512, 32, 8, 64),
    "qwen2.5-7b-layer": (4, 28, 128, 512, 64, 16, 256),
    "qwen2.5-32b-layer": (8, 40, 128, 1024, 64, 64, 512),
    "ragged": (4, 28, 128, 512, 8, 5, 129),
    "no-suffix": (4, 28, 128, 512, 8, 3, 0),
}


def _ranks(H, nb, d, seed):
    rng = np.random.default_rng(seed)
    return rng.integers(4, d + 1, size=(2 * H, nb), dtype=np.int32)


def _check(wl, H, Hq, d, n, nb, B, S, ctas):
    G = Hq // H
    cpb, nsc = n // 128, -(-S // 128)
    ipt = min(B, 128 // G)
    nrt = -(-B // ipt)
    assert wl["items_per_tile"] == ipt and wl["tiles"] == nrt
    segs, first = wl["segs"], wl["seg_first"]
    assert len(first) == min(ctas, H * nrt * nb * cpb + B * H * nsc) + 1
    assert first[0] == 0 and first[-1] == len(segs) and np.all(np.diff(first) >= 0)
    assert np.array_equal(segs[:, 5], np.arange(len(segs)))  # partial slot = segment index
    covered = {}
    for kind, h, tile, c0, c1, pid, rows, _ in segs:
        assert 0 <= c0 < c1
        if kind == 0:
            assert c1 <= nb * cpb and rows == min(ipt, B - tile * ipt) * G
        else:
            assert kind == 1 and c1 <= nsc and rows == G
        covered.setdefault((kind, h, tile), []).append((c0, c1, pid))
    # every chunk exactly once, segments of one group consecutive and in order
    for h in range(H):
        for t in range(nrt):
            runs = covered.pop((0, h, t))
            assert runs[0][0] == 0 and runs[-1][1] == nb * cpb
            assert all(a[1] == b[0] and a[2] + 1 == b[2] for a, b in zip(runs, runs[1:]))
            lo, hi = wl["pre_range"][h * nrt + t]
            assert (lo, hi) == (runs[0][2], runs[-1][2] + 1)
    for i in range(B):
        for h in range(H):
            lo, hi = wl["suf_range"][i * H + h]
            if nsc == 0:
                assert lo == hi
                continue
            runs = covered.pop((1, h, i))
            assert runs[0][0] == 0 and runs[-1][1] == nsc
            assert all(a[1] == b[0] and a[2] + 1 == b[2] for a, b in zip(runs, runs[1:]))
            assert (lo, hi) == (runs[0][2], runs[-1][2] + 1)
    assert not covered  # nothing else


@pytest.mark.parametrize("name", sorted(SHAPES))
@pytest.mark.parametrize("ctas", [148, 37, 1])
def test_worklist_covers_every_chunk_once(name, ctas):
    import decode_attention_milo_b200 as milo
    H, Hq, d, n, nb, B, S = SHAPES[name]
    wl = milo.decode_worklist(_ranks(H, nb, d, 7), n, d, B, Hq, S, ctas)
    _check(wl, H, Hq, d, n, nb, B, S, ctas)


def test_worklist_gives_every_cta_work():
    import decode_attention_milo_b200 as milo
    H, Hq, d, n, nb, B, S = SHAPES["qwen2.5-7b-layer"]
    wl = milo.decode_worklist(_ranks(H, nb, d, 3), n, d, B, Hq, S, 148)
    assert np.all(np.diff(wl["seg_first"]) >= 1)


def test_worklist_rejects_bad_arguments():
    import decode_attention_milo_b200 as milo
    r = _ranks(4, 8, 128, 1)
    with pytest.raises(milo.MiloError) as e:
        milo.decode_worklist(np.where(r == r[0, 0], 0, r), 512, 128, 4, 28, 0, 148)  # a rank of 0
    assert e.value.code == 1
    with pytest.raises(milo.MiloError) as e:
        milo.decode_worklist(r, 512, 96, 4, 28, 0, 148)  # head dim not built
    assert e.value.code in (1, 2)
    with pytest.raises(milo.MiloError) as e:
        milo.decode_worklist(r, 500, 128, 4, 28, 0, 148)  # block size not a multiple of 128
    assert e.value.code == 2
