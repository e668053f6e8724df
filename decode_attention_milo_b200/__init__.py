"""Python binding of libmilo.so: MILO compressed-KV decode attention on B200.

Argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; PyTorch supplies device memory (tensors) and the current stream.
The library must be built first (python -m decode_attention_milo_b200.build);
importing the binding without it raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

__all__ = ["F32", "BF16", "I8", "MiloError", "Factors", "compress", "decode_attn", "import_factors", "lib_path",
           "load_library", "quantize"]

F32, BF16, I8 = 0, 1, 2  # I8: factor objects only (int8 token factors, bf16 dimension factors)
KEEP_INTERMEDIATES = 1
ALLOC_RULES = {"entropy": 0, "greedy": 1, "uniform": 2, "weights": 3}
POOL_SCOPES = {"pool": 0, "layer": 1}
_HERE = os.path.dirname(os.path.abspath(__file__))


def lib_path() -> str:
    return os.path.join(_HERE, "libmilo.so")


class MiloError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {_status_string(code)} ({code})")


class _Desc(ctypes.Structure):
    _fields_ = [
        ("num_kv_heads", ctypes.c_int32), ("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("context", ctypes.c_int64), ("r_min", ctypes.c_int32),
        ("pool_rows", ctypes.c_int32), ("dtype", ctypes.c_int32), ("alloc_rule", ctypes.c_int32),
        ("pool_scope", ctypes.c_int32), ("reserved", ctypes.c_int32), ("total_rows", ctypes.c_int64),
        ("ranks", ctypes.c_void_p), ("row_offsets", ctypes.c_void_p), ("tok", ctypes.c_void_p),
        ("dim", ctypes.c_void_p), ("eigvals", ctypes.c_void_p), ("eigvecs", ctypes.c_void_p),
        ("entropy", ctypes.c_void_p), ("quotas", ctypes.c_void_p), ("sweeps", ctypes.c_void_p),
    ]


_lib = None


def load_library(path: str | None = None):
    """Loads libmilo.so (once) and declares its C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or lib_path()
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m decode_attention_milo_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, u32, f32, f64 = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                   ctypes.c_float, ctypes.c_double)
    L.milo_abi_version.restype = i32
    L.milo_status_string.restype = ctypes.c_char_p
    L.milo_status_string.argtypes = [i32]
    L.milo_compress.restype = i32
    L.milo_compress.argtypes = [vp, vp, i32, i32, i64, i32, i32, f64, i32, i32, u32, vp, ctypes.POINTER(vp)]
    L.milo_compress_rule.restype = i32
    L.milo_compress_rule.argtypes = [vp, vp, i32, i32, i64, i32, i32, f64, i32, i32, u32, i32, i32, vp, vp,
                                     ctypes.POINTER(vp)]
    L.milo_compress_profiled.restype = i32
    L.milo_compress_profiled.argtypes = [vp, vp, i32, i32, i64, i32, i32, f64, i32, i32, u32, vp,
                                         ctypes.POINTER(vp), ctypes.POINTER(vp)]
    L.milo_decode_attn.restype = i32
    L.milo_decode_attn.argtypes = [vp, i32, i32, vp, vp, vp, i32, f32, vp, vp]
    L.milo_decode_attn_profiled.restype = i32
    L.milo_decode_attn_profiled.argtypes = [vp, i32, i32, vp, vp, vp, i32, f32, vp, vp, vp, vp]
    L.milo_decode_attn_select.restype = i32
    L.milo_decode_attn_select.argtypes = [vp, i32, i32, vp, vp, vp, i32, f32, vp, vp, vp]
    L.milo_decode_attn_rope.restype = i32
    L.milo_decode_attn_rope.argtypes = [vp, i32, i32, vp, vp, vp, i32, f32, f64, vp, vp, vp]
    L.milo_decode_attn_noalloc.restype = i32
    L.milo_decode_attn_noalloc.argtypes = [vp, i32, i32, vp, vp, vp, i32, f32, vp, vp]
    L.milo_decode_launches.restype = i32
    L.milo_decode_launches.argtypes = [vp, i32, i32, i32]
    L.milo_decode_worklist.restype = i32
    L.milo_decode_worklist.argtypes = [vp, i32, i32, i32, i32, i32, i32, i32, i32, vp, i64, vp]
    L.milo_factors_ranks.restype = i32
    L.milo_factors_ranks.argtypes = [vp, vp]
    L.milo_factors_describe.restype = i32
    L.milo_factors_describe.argtypes = [vp, ctypes.POINTER(_Desc)]
    L.milo_factors_status.restype = i32
    L.milo_factors_status.argtypes = [vp, ctypes.POINTER(u32)]
    L.milo_factors_import.restype = i32
    L.milo_factors_import.argtypes = [i32, i32, i64, i32, i32, i32, vp, vp, vp, vp, ctypes.POINTER(vp)]
    L.milo_factors_quantize.restype = i32
    L.milo_factors_quantize.argtypes = [vp, vp, ctypes.POINTER(vp)]
    L.milo_factors_destroy.restype = None
    L.milo_factors_destroy.argtypes = [vp]
    if L.milo_abi_version() != 4:
        raise RuntimeError("libmilo.so ABI version mismatch")
    _lib = L
    return L


def _status_string(code: int) -> str:
    return load_library().milo_status_string(code).decode()


def _check(code: int, what: str):
    if code != 0:
        raise MiloError(code, what)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev_ptr(t, name):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


class Factors:
    """A compressed layer: per-block low-rank factors owned by the library."""

    def __init__(self, handle: ctypes.c_void_p):
        self._h = handle
        self._shape = None

    @property
    def handle(self):
        if not self._h:
            raise ValueError("factor object was destroyed")
        return self._h

    def describe(self) -> dict:
        d = _Desc()
        _check(load_library().milo_factors_describe(self.handle, ctypes.byref(d)), "milo_factors_describe")
        return {name: getattr(d, name) for name, _ in _Desc._fields_}

    def shape(self) -> tuple[int, int, int]:
        """(KV heads, head dim, dtype code) of the factors (cached: they never change)."""
        if self._shape is None:
            d = self.describe()
            self._shape = (d["num_kv_heads"], d["head_dim"], d["dtype"])
        return self._shape

    def ranks(self) -> np.ndarray:
        d = self.describe()
        out = np.zeros((2 * d["num_kv_heads"], d["num_blocks"]), dtype=np.int32)
        _check(load_library().milo_factors_ranks(self.handle, out.ctypes.data_as(ctypes.c_void_p)),
               "milo_factors_ranks")
        return out

    def decode_launches(self, batch: int, num_q_heads: int, suffix_len: int) -> int:
        """Kernels one decode call with this shape launches."""
        n = load_library().milo_decode_launches(self.handle, batch, num_q_heads, suffix_len)
        if n < 0:
            raise MiloError(-n, "milo_decode_launches")
        return n

    def status(self) -> tuple[int, int]:
        bits = ctypes.c_uint32(0)
        code = load_library().milo_factors_status(self.handle, ctypes.byref(bits))
        return code, bits.value

    def close(self):
        if self._h:
            load_library().milo_factors_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def compress(K, V, block_size: int, budget: float, r_min: int = 4, max_sweeps: int = 0,
             keep_intermediates: bool = False, stream=None) -> Factors:
    """Compresses one layer's K, V [H][T][d] (CUDA tensors, float32 or bfloat16). See milo_compress."""
    if K.shape != V.shape or K.dim() != 3 or K.dtype != V.dtype:
        raise ValueError("K and V must both be [H][T][d] with the same dtype")
    H, T, d = K.shape
    h = ctypes.c_void_p()
    flags = KEEP_INTERMEDIATES if keep_intermediates else 0
    _check(load_library().milo_compress(_dev_ptr(K, "K"), _dev_ptr(V, "V"), _dtype_code(K), H, T, d, block_size,
                                        float(budget), r_min, max_sweeps, flags, _stream_ptr(stream),
                                        ctypes.byref(h)), "milo_compress")
    return Factors(h)


def compress_rule(K, V, block_size: int, budget: float, rule: str = "entropy", scope: str = "pool",
                  weights=None, r_min: int = 4, max_sweeps: int = 0, keep_intermediates: bool = False,
                  stream=None) -> Factors:
    """compress() with an allocation rule ("entropy", "greedy", "uniform", "weights") and budget scope
    ("pool" or "layer"); weights: host [2H][nb] array for the "weights" rule. See milo_compress_rule."""
    if K.shape != V.shape or K.dim() != 3 or K.dtype != V.dtype:
        raise ValueError("K and V must both be [H][T][d] with the same dtype")
    H, T, d = K.shape
    w = None
    if weights is not None:
        w = np.ascontiguousarray(weights, dtype=np.float64)
        if w.size != 2 * H * (T // block_size):
            raise ValueError("weights must hold [2H][nb] values")
    h = ctypes.c_void_p()
    flags = KEEP_INTERMEDIATES if keep_intermediates else 0
    _check(load_library().milo_compress_rule(
        _dev_ptr(K, "K"), _dev_ptr(V, "V"), _dtype_code(K), H, T, d, block_size, float(budget), r_min, max_sweeps,
        flags, ALLOC_RULES[rule], POOL_SCOPES[scope], None if w is None else w.ctypes.data_as(ctypes.c_void_p),
        _stream_ptr(stream), ctypes.byref(h)), "milo_compress_rule")
    return Factors(h)


def compress_profiled(K, V, block_size: int, budget: float, events, r_min: int = 4, max_sweeps: int = 0,
                      keep_intermediates: bool = False, stream=None) -> Factors:
    """compress() that records five torch.cuda.Event objects: before the Gram, Jacobi, allocation and
    projection kernels and after the last (milo_compress_profiled)."""
    if K.shape != V.shape or K.dim() != 3 or K.dtype != V.dtype or len(events) != 5:
        raise ValueError("K and V must both be [H][T][d] with the same dtype, and five events are needed")
    H, T, d = K.shape
    h = ctypes.c_void_p()
    flags = KEEP_INTERMEDIATES if keep_intermediates else 0
    evs = (ctypes.c_void_p * 5)(*[e.cuda_event for e in events])
    _check(load_library().milo_compress_profiled(_dev_ptr(K, "K"), _dev_ptr(V, "V"), _dtype_code(K), H, T, d,
                                                 block_size, float(budget), r_min, max_sweeps, flags,
                                                 _stream_ptr(stream), ctypes.byref(h), evs), "milo_compress_profiled")
    return Factors(h)


def _decode_args(q, factors: Factors, K_suf, V_suf, out):
    """Checks the shapes and dtypes of one decode call against the factors (the C ABI takes no q shape or
    dtype beyond batch and heads, so a mismatched tensor would be read or written past its end) and
    returns (batch, q heads, suffix length, out)."""
    import torch
    H, d, dt = factors.shape()
    want = torch.bfloat16 if dt in (BF16, I8) else torch.float32
    if q.dim() != 3 or q.shape[2] != d or q.shape[1] % H != 0 or q.shape[0] < 1:
        raise ValueError(f"q must be [batch][q_heads][{d}] with q_heads a multiple of {H}, got {tuple(q.shape)}")
    if q.dtype != want:
        raise ValueError(f"q must have the factors' dtype {want}, got {q.dtype}")
    B, Hq, _ = q.shape
    S = 0
    if K_suf is not None or V_suf is not None:
        if K_suf is None or V_suf is None:
            raise ValueError("K_suf and V_suf must be given together")
        if K_suf.dim() != 4 or tuple(K_suf.shape) != tuple(V_suf.shape) or tuple(K_suf.shape[:2]) != (B, H) \
                or K_suf.shape[3] != d:
            raise ValueError(f"K_suf and V_suf must both be [{B}][{H}][S][{d}], got {tuple(K_suf.shape)} and "
                             f"{tuple(V_suf.shape)}")
        if K_suf.dtype != want or V_suf.dtype != want:
            raise ValueError(f"K_suf and V_suf must have the factors' dtype {want}")
        S = K_suf.shape[2]
    if out is None:
        out = torch.empty_like(q)
    elif tuple(out.shape) != tuple(q.shape) or out.dtype != want:
        raise ValueError(f"out must be {tuple(q.shape)} of dtype {want}, got {tuple(out.shape)} {out.dtype}")
    return B, Hq, S, out


def decode_attn(q, factors: Factors, K_suf=None, V_suf=None, scale: float = 0.0, out=None, stream=None):
    """One decode step: q [B][Hq][d] → out [B][Hq][d]. Suffix K/V [B][H][S][d] or None. See milo_decode_attn."""
    B, Hq, S, out = _decode_args(q, factors, K_suf, V_suf, out)
    _check(load_library().milo_decode_attn(_dev_ptr(q, "q"), B, Hq, factors.handle,
                                           _dev_ptr(K_suf, "K_suf") if S else None,
                                           _dev_ptr(V_suf, "V_suf") if S else None, S, float(scale),
                                           _dev_ptr(out, "out"), _stream_ptr(stream)), "milo_decode_attn")
    return out


def decode_attn_select(q, factors: Factors, block_mask, K_suf=None, V_suf=None, scale: float = 0.0, out=None,
                       stream=None):
    """decode_attn over the blocks block_mask [H][nb] selects (host array, nonzero = attend).
    See milo_decode_attn_select."""
    B, Hq, S, out = _decode_args(q, factors, K_suf, V_suf, out)
    H = factors.shape()[0]
    nb = factors.describe()["num_blocks"]
    m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    if m.shape != (H, nb):
        raise ValueError(f"block_mask must be [{H}][{nb}], got {m.shape}")
    _check(load_library().milo_decode_attn_select(
        _dev_ptr(q, "q"), B, Hq, factors.handle, _dev_ptr(K_suf, "K_suf") if S else None,
        _dev_ptr(V_suf, "V_suf") if S else None, S, float(scale), m.ctypes.data_as(ctypes.c_void_p),
        _dev_ptr(out, "out"), _stream_ptr(stream)), "milo_decode_attn_select")
    return out


def decode_attn_rope(q, factors: Factors, K_suf=None, V_suf=None, theta: float = 1e6, block_mask=None,
                     scale: float = 0.0, out=None, stream=None):
    """decode_attn over factors of pre-RoPE keys: every key block is rebuilt and rotated at its absolute
    positions (base theta) before the scores; q and the suffix are post-RoPE.  See milo_decode_attn_rope."""
    B, Hq, S, out = _decode_args(q, factors, K_suf, V_suf, out)
    m = None
    if block_mask is not None:
        H = factors.shape()[0]
        nb = factors.describe()["num_blocks"]
        m = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
        if m.shape != (H, nb):
            raise ValueError(f"block_mask must be [{H}][{nb}], got {m.shape}")
    _check(load_library().milo_decode_attn_rope(
        _dev_ptr(q, "q"), B, Hq, factors.handle, _dev_ptr(K_suf, "K_suf") if S else None,
        _dev_ptr(V_suf, "V_suf") if S else None, S, float(scale), float(theta),
        m.ctypes.data_as(ctypes.c_void_p) if m is not None else None, _dev_ptr(out, "out"), _stream_ptr(stream)),
        "milo_decode_attn_rope")
    return out


def decode_attn_profiled(q, factors: Factors, K_suf, V_suf, out, event_before, event_after, scale: float = 0.0,
                         stream=None):
    """decode_attn that records two torch.cuda.Event objects around the main decode kernel."""
    B, Hq, S, out = _decode_args(q, factors, K_suf, V_suf, out)
    _check(load_library().milo_decode_attn_profiled(
        _dev_ptr(q, "q"), B, Hq, factors.handle, _dev_ptr(K_suf, "K_suf") if S else None,
        _dev_ptr(V_suf, "V_suf") if S else None, S, float(scale), _dev_ptr(out, "out"), _stream_ptr(stream),
        ctypes.c_void_p(event_before.cuda_event), ctypes.c_void_p(event_after.cuda_event)),
        "milo_decode_attn_profiled")
    return out


def decode_attn_noalloc(q, factors: Factors, K_suf=None, V_suf=None, scale: float = 0.0, out=None, stream=None):
    """decode_attn through milo_decode_attn_noalloc: the library allocates nothing (bf16 factors only)."""
    B, Hq, S, out = _decode_args(q, factors, K_suf, V_suf, out)
    _check(load_library().milo_decode_attn_noalloc(
        _dev_ptr(q, "q"), B, Hq, factors.handle, _dev_ptr(K_suf, "K_suf") if S else None,
        _dev_ptr(V_suf, "V_suf") if S else None, S, float(scale), _dev_ptr(out, "out"), _stream_ptr(stream)),
        "milo_decode_attn_noalloc")
    return out


def import_factors(dtype: int, num_kv_heads: int, context: int, head_dim: int, block_size: int, r_min: int,
                   ranks: np.ndarray, tok: np.ndarray, dim: np.ndarray, stream=None) -> Factors:
    """Builds a factor object from host arrays in the library's layout (tok [rows][n], dim [rows][d]); with
    dtype I8, tok holds int8 codes and dim bf16 bit patterns (2-byte elements)."""
    ranks = np.ascontiguousarray(ranks, dtype=np.int32)
    tok = np.ascontiguousarray(tok)
    dim = np.ascontiguousarray(dim)
    rows = int(ranks.sum())
    tok_bytes, dim_bytes = {F32: (4, 4), BF16: (2, 2), I8: (1, 2)}.get(dtype, (0, 0))
    if tok.nbytes != rows * block_size * tok_bytes or dim.nbytes != rows * head_dim * dim_bytes:
        raise ValueError(f"tok must hold {rows}x{block_size} and dim {rows}x{head_dim} elements of dtype code {dtype}")
    h = ctypes.c_void_p()
    _check(load_library().milo_factors_import(dtype, num_kv_heads, context, head_dim, block_size, r_min,
                                              ranks.ctypes.data_as(ctypes.c_void_p),
                                              tok.ctypes.data_as(ctypes.c_void_p),
                                              dim.ctypes.data_as(ctypes.c_void_p), _stream_ptr(stream),
                                              ctypes.byref(h)), "milo_factors_import")
    return Factors(h)


def quantize(factors: Factors, stream=None) -> Factors:
    """8-bit copy of a bf16 factor object (int8 token factors per rank channel, scales folded into the bf16
    dimension factors at rank r + 1). See milo_factors_quantize."""
    h = ctypes.c_void_p()
    _check(load_library().milo_factors_quantize(factors.handle, _stream_ptr(stream), ctypes.byref(h)),
           "milo_factors_quantize")
    return Factors(h)


def decode_worklist(ranks, block_size: int, head_dim: int, batch: int, num_q_heads: int, suffix_len: int,
                    num_ctas: int) -> dict:
    """The bf16 decode's work list for host ranks [2H][nb] (milo_decode_worklist; host only, no GPU)."""
    import numpy as np
    r = np.ascontiguousarray(ranks, dtype=np.int32)
    H, nb = r.shape[0] // 2, r.shape[1]
    cap = 1 << 22
    out = np.zeros(cap, dtype=np.int32)
    info = np.zeros(8, dtype=np.int64)
    _check(load_library().milo_decode_worklist(r.ctypes.data, H, nb, block_size, head_dim, batch, num_q_heads,
                                               suffix_len, num_ctas, out.ctypes.data, cap, info.ctypes.data),
           "milo_decode_worklist")
    nwords, nsegs, grid, off_segs, off_pre, off_suf, ipt, nrt = (int(x) for x in info)
    return {"seg_first": out[:grid + 1].copy(),
            "segs": out[off_segs:off_segs + 8 * nsegs].reshape(nsegs, 8).copy(),
            "pre_range": out[off_pre:off_pre + 2 * H * nrt].reshape(H * nrt, 2).copy(),
            "suf_range": out[off_suf:off_suf + 2 * batch * H].reshape(batch * H, 2).copy(),
            "items_per_tile": ipt, "tiles": nrt, "words": nwords}
