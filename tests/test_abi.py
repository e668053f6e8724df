"""The C-ABI library loads, exports every symbol its header declares, and rejects bad arguments
before touching the GPU (these calls return before any CUDA call, so they run on CPU)."""
import ctypes
import os
import re

import pytest

import decode_attention_milo_b200 as milo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(milo_\w+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol():
    lib = milo.load_library()
    names = _declared()
    assert {"milo_compress", "milo_decode_attn"} <= names
    for n in names:
        assert hasattr(lib, n), n
    assert lib.milo_abi_version() == 4
    assert lib.milo_status_string(0) == b"ok"
    assert lib.milo_status_string(3).startswith(b"budget")


def _compress(lib, **kw):
    args = dict(K=1, V=1, dtype=1, H=4, T=32768, d=128, n=512, budget=0.5, r_min=4, sweeps=0, flags=0)
    args.update(kw)
    out = ctypes.c_void_p(123)
    code = lib.milo_compress(ctypes.c_void_p(args["K"]) if args["K"] else None,
                             ctypes.c_void_p(args["V"]) if args["V"] else None,
                             args["dtype"], args["H"], args["T"], args["d"], args["n"], args["budget"],
                             args["r_min"], args["sweeps"], args["flags"], None, ctypes.byref(out))
    assert out.value is None  # *out cleared on error
    return code


@pytest.mark.parametrize("kw,code", [
    (dict(K=0), 1), (dict(dtype=7), 1), (dict(H=0), 1), (dict(d=96), 2), (dict(d=0), 1),
    (dict(T=32769), 1), (dict(n=100), 1), (dict(n=64), 1), (dict(r_min=0), 1), (dict(r_min=129), 1),
    (dict(budget=0.0), 1), (dict(budget=float("nan")), 1), (dict(sweeps=-1), 1), (dict(flags=8), 1),
    (dict(budget=0.001), 3),
    (dict(T=8193 * 512, H=1), 2),  # more blocks per pool than the allocation step holds in shared memory
    (dict(dtype=2), 1),            # 8-bit describes factor objects only, never the cache
])
def test_compress_rejects_bad_arguments(kw, code):
    assert _compress(milo.load_library(), **kw) == code


def _compress_rule(lib, rule=0, scope=0, weights=None, **kw):
    args = dict(K=1, V=1, dtype=1, H=4, T=32768, d=128, n=512, budget=0.5, r_min=4)
    args.update(kw)
    out = ctypes.c_void_p(123)
    w = None if weights is None else weights.ctypes.data_as(ctypes.c_void_p)
    code = lib.milo_compress_rule(ctypes.c_void_p(args["K"]), ctypes.c_void_p(args["V"]), args["dtype"], args["H"],
                                  args["T"], args["d"], args["n"], args["budget"], args["r_min"], 0, 0, rule, scope,
                                  w, None, ctypes.byref(out))
    assert out.value is None
    return code


def test_compress_rule_rejects_bad_arguments():
    import numpy as np
    lib = milo.load_library()
    w = np.ones(2 * 4 * 64)
    assert _compress_rule(lib, rule=4) == 1                      # unknown rule
    assert _compress_rule(lib, scope=2) == 1                     # unknown scope
    assert _compress_rule(lib, rule=3) == 1                      # weights rule without weights
    assert _compress_rule(lib, rule=0, weights=w) == 1           # weights given to another rule
    bad = w.copy()
    bad[5] = 0.0
    assert _compress_rule(lib, rule=3, weights=bad) == 1         # weights must be > 0
    bad[5] = float("nan")
    assert _compress_rule(lib, rule=3, weights=bad) == 1
    # a layer-wide budget allocates over all 2H·nb blocks at once: 16 heads x 2 x 512 blocks is too many
    assert _compress_rule(lib, scope=1, H=16, T=512 * 512) == 2
    assert _compress_rule(lib, rule=1, budget=0.001) == 3


def test_decode_rejects_null_arguments():
    lib = milo.load_library()
    assert lib.milo_decode_attn(None, 1, 2, None, None, None, 0, 0.0, None, None) == 1
    assert lib.milo_factors_ranks(None, None) == 1
    assert lib.milo_factors_status(None, None) == 1
    lib.milo_factors_destroy(None)


def test_import_rejects_ranks_out_of_range():
    import numpy as np
    lib = milo.load_library()
    tok = np.zeros(64 * 512, dtype=np.uint16)
    for bad in (0, 65):
        ranks = np.array([[4, bad], [4, 4]], dtype=np.int32)
        out = ctypes.c_void_p()
        code = lib.milo_factors_import(1, 1, 1024, 64, 512, 4, ranks.ctypes.data_as(ctypes.c_void_p),
                                       tok.ctypes.data_as(ctypes.c_void_p), tok.ctypes.data_as(ctypes.c_void_p),
                                       None, ctypes.byref(out))
        assert code == 1


def test_every_status_code_has_a_string():
    lib = milo.load_library()
    seen = set()
    for code in range(8):
        s = lib.milo_status_string(code)
        assert s and s not in seen, code
        seen.add(s)
    assert lib.milo_status_string(99)  # unknown codes still get a string


def test_host_only_calls_reject_bad_arguments():
    import numpy as np
    lib = milo.load_library()
    assert lib.milo_decode_launches(None, 1, 28, 0) == -1
    assert lib.milo_decode_attn_noalloc(None, 1, 2, None, None, None, 0, 0.0, None, None) == 1
    ranks = np.full((8, 4), 16, dtype=np.int32)
    out = np.zeros(1 << 12, dtype=np.int32)
    info = np.zeros(8, dtype=np.int64)
    call = lambda **kw: lib.milo_decode_worklist(
        ranks.ctypes.data, kw.get("H", 4), 4, kw.get("n", 512), 128, kw.get("B", 16), kw.get("Hq", 28),
        kw.get("S", 0), kw.get("ctas", 148), out.ctypes.data, kw.get("cap", out.size), info.ctypes.data)
    assert call() == 0 and info[0] > 0 and info[1] >= 1
    assert call(Hq=27) == 1        # query heads not a multiple of KV heads
    assert call(B=0) == 1
    assert call(ctas=0) == 1
    assert call(S=-1) == 1
    assert call(n=384 + 64) == 2   # block size not a multiple of 128
    assert call(cap=4) == 2        # output too small


def test_python_decode_checks_shapes_before_the_library():
    """The binding rejects a q, out or suffix whose shape or dtype does not match the factors (the C ABI takes
    no q shape or dtype beyond batch and heads) before any library call."""
    import torch

    class FakeFactors(milo.Factors):
        def __init__(self):
            super().__init__(None)
            self._shape = (4, 128, milo.BF16)  # 4 KV heads, d = 128, bf16

        def close(self):
            pass

    f = FakeFactors()
    bf = torch.bfloat16
    good_q = torch.zeros(2, 28, 128, dtype=bf)
    bad = [
        dict(q=torch.zeros(2, 28, 64, dtype=bf)),                       # head dim
        dict(q=torch.zeros(2, 27, 128, dtype=bf)),                      # q heads not a multiple of 4
        dict(q=torch.zeros(2, 28, 128, dtype=torch.float32)),           # dtype
        dict(q=torch.zeros(28, 128, dtype=bf)),                         # rank
        dict(out=torch.zeros(2, 28, 64, dtype=bf)),                     # out shape
        dict(out=torch.zeros(2, 28, 128, dtype=torch.float32)),         # out dtype
        dict(K_suf=torch.zeros(2, 4, 8, 128, dtype=bf)),                # V_suf missing
        dict(K_suf=torch.zeros(2, 4, 8, 128, dtype=bf), V_suf=torch.zeros(2, 4, 9, 128, dtype=bf)),
        dict(K_suf=torch.zeros(3, 4, 8, 128, dtype=bf), V_suf=torch.zeros(3, 4, 8, 128, dtype=bf)),
        dict(K_suf=torch.zeros(2, 4, 8, 64, dtype=bf), V_suf=torch.zeros(2, 4, 8, 64, dtype=bf)),
    ]
    for kw in bad:
        args = dict(q=good_q, K_suf=None, V_suf=None, out=None)
        args.update(kw)
        for fn in (milo.decode_attn, milo.decode_attn_noalloc):
            with pytest.raises(ValueError):
                fn(args["q"], f, args["K_suf"], args["V_suf"], out=args["out"])


def test_quantize_rejects_bad_arguments():
    lib = milo.load_library()
    out = ctypes.c_void_p(123)
    assert lib.milo_factors_quantize(None, None, ctypes.byref(out)) == 1
    assert out.value is None
    assert lib.milo_factors_quantize(None, None, None) == 1


def test_import_checks_array_sizes_for_8bit():
    import numpy as np
    ranks = np.full((2, 2), 5, dtype=np.int32)  # one KV head, two blocks of 512: 20 rows
    with pytest.raises(ValueError):  # bf16-sized codes for an 8-bit object
        milo.import_factors(milo.I8, 1, 1024, 64, 512, 4, ranks, np.zeros((20, 512), np.uint16),
                            np.zeros((20, 64), np.uint16))


def test_rope_decode_rejects_bad_arguments():
    lib = milo.load_library()
    # no factor object, and a rotary base that is not > 1 (checked before anything else runs)
    assert lib.milo_decode_attn_rope(None, 1, 1, None, None, None, 0, 0.0, 1e6, None, None, None) == 1
    assert lib.milo_decode_attn_rope(None, 1, 1, None, None, None, 0, 0.0, 1.0, None, None, None) == 1
    assert lib.milo_decode_attn_rope(None, 1, 1, None, None, None, 0, 0.0, float("nan"), None, None, None) == 1
