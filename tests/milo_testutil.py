"""Shared helpers of the tests: storage casts, oracle-factor packing, error norms.

Packing turns the oracle's per-block factors into the library's documented
layout (ranks [2H][nb], tok [rows][n], dim [rows][d]); it is layout plumbing,
not arithmetic of the method.
"""
import numpy as np

import oracle
from synth import from_storage, to_storage


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def row_rel_max(a, b) -> float:
    """Largest relative L2 error of one output row (one (query, head) vector along the last axis)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return float(np.max(num / np.maximum(den, np.finfo(np.float64).tiny)))


# A whole-tensor relative L2 can hide one bad row (10 % error in one of 448 rows reads as 4.7e-3 over the
# tensor), so every parity check also bounds the worst row, at this multiple of the tensor bound.
ROW_FACTOR = 4.0


def assert_close(got, want, tol, what=""):
    """Whole-tensor relative L2 <= tol and every row's relative L2 <= ROW_FACTOR * tol; prints both."""
    t, r = rel_l2(got, want), row_rel_max(got, want)
    print(f"{what}: relative L2 {t:.2e} (bound {tol:.0e}), worst row {r:.2e} (bound {ROW_FACTOR * tol:.0e})")
    assert t <= tol, (what, t, tol)
    assert r <= ROW_FACTOR * tol, (what, r, ROW_FACTOR * tol)


def cast_fn(dtype):
    return lambda x: from_storage(to_storage(x, dtype), dtype)


def stored_layer(layer: dict, dtype: str) -> dict:
    c = cast_fn(dtype)
    return dict(K=[oracle.stored_factors(p, c) for p in layer["K"]],
                V=[oracle.stored_factors(p, c) for p in layer["V"]])


SLAB = 128  # tokens per slab of the token-side factor


def tok_slabs(u: np.ndarray) -> np.ndarray:
    """U_b (n × r) → the library's slab order: [n/128][r][128] flattened to (n/128·r, 128)."""
    n, r = u.shape
    return u.T.reshape(r, n // SLAB, SLAB).transpose(1, 0, 2).reshape(-1, SLAB)


def untok_slabs(flat: np.ndarray, n: int, r: int) -> np.ndarray:
    """Inverse of tok_slabs: r·n elements → U_b (n × r)."""
    return flat.reshape(n // SLAB, r, SLAB).transpose(1, 0, 2).reshape(r, n).T


def pack_factors(layer: dict, dtype: str):
    """Oracle layer → (ranks [2H][nb] int32, tok (Σr·n/128, 128), dim [rows][d]) in storage dtype."""
    H = len(layer["K"])
    pools = []
    for h in range(H):
        pools += [layer["K"][h], layer["V"][h]]
    ranks = np.array([p["ranks"] for p in pools], dtype=np.int32)
    tok = np.concatenate([tok_slabs(u) for p in pools for u in p["U"]], axis=0)
    dim = np.concatenate([b.T for p in pools for b in p["B"]], axis=0)
    return ranks, to_storage(tok, dtype), to_storage(dim, dtype)


def to_torch(arr, dtype: str, device="cuda"):
    import torch
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32)).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).to(device).view(torch.bfloat16)


def from_torch(t) -> np.ndarray:
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return from_storage(t.view(torch.int16).numpy().view(np.uint16), "bf16")
    return t.double().numpy()


class _CudaArray:
    def __init__(self, ptr, shape, typestr):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (int(ptr), False),
                                         "version": 3, "strides": None}


def device_view(ptr, shape, typestr):
    """Zero-copy torch view of library-owned device memory (read it before the owner is destroyed)."""
    import torch
    return torch.as_tensor(_CudaArray(ptr, shape, typestr), device="cuda")


def factor_arrays(f) -> dict:
    """Host copies of a factor object's arrays, as fp64 / int numpy arrays."""
    import torch
    d = f.describe()
    H2, nb, n, dd, total = 2 * d["num_kv_heads"], d["num_blocks"], d["block_size"], d["head_dim"], d["total_rows"]
    bf = d["dtype"] == 1
    out = dict(desc=d)
    out["ranks"] = device_view(d["ranks"], (H2, nb), "<i4").cpu().numpy()
    out["row_offsets"] = device_view(d["row_offsets"], (H2, nb + 1), "<i8").cpu().numpy()
    if d["dtype"] == 2:  # 8-bit object: int8 codes, bf16 dimension factors
        out["codes"] = device_view(d["tok"], (total * n,), "|i1").cpu().numpy()
        out["tok"] = out["codes"].astype(np.float64)
        dim = device_view(d["dim"], (total, dd), "<i2").cpu().numpy().view(np.uint16)
        out["dim"] = from_storage(dim, "bf16")
    elif bf:
        tok = device_view(d["tok"], (total * n,), "<i2").cpu().numpy().view(np.uint16)
        dim = device_view(d["dim"], (total, dd), "<i2").cpu().numpy().view(np.uint16)
        out["tok"], out["dim"] = from_storage(tok, "bf16"), from_storage(dim, "bf16")
    else:
        out["tok"] = device_view(d["tok"], (total * n,), "<f4").cpu().numpy().astype(np.float64)
        out["dim"] = device_view(d["dim"], (total, dd), "<f4").cpu().numpy().astype(np.float64)
    if d["eigvals"]:
        out["eigvals"] = device_view(d["eigvals"], (H2, nb, dd), "<f4").cpu().numpy().astype(np.float64)
        out["entropy"] = device_view(d["entropy"], (H2, nb), "<f8").cpu().numpy()
        out["quotas"] = device_view(d["quotas"], (H2, nb), "<f8").cpu().numpy()
    if d["eigvecs"]:
        out["eigvecs"] = device_view(d["eigvecs"], (H2, nb, dd, dd), "<f4").cpu().numpy().astype(np.float64)
    torch.cuda.synchronize()
    return out


def layer_from_arrays(got: dict) -> dict:
    """Oracle layer (pools of U, B per block) from a factor object's host arrays (factor_arrays)."""
    d = got["desc"]
    H, nb, n = d["num_kv_heads"], d["num_blocks"], d["block_size"]
    pools = []
    for p in range(2 * H):
        U, B = [], []
        for b in range(nb):
            r0, r1 = int(got["row_offsets"][p, b]), int(got["row_offsets"][p, b + 1])
            U.append(untok_slabs(got["tok"][r0 * n:r1 * n], n, r1 - r0))
            B.append(got["dim"][r0:r1].T)
        pools.append(dict(U=U, B=B, ranks=got["ranks"][p]))
    return dict(K=pools[0::2], V=pools[1::2])


def pack_factors_8bit(qlayer: dict):
    """Oracle 8-bit layer (oracle.quantize_layer) → (ranks, int8 codes in slab order, bf16 dim) for import."""
    H = len(qlayer["K"])
    pools = []
    for h in range(H):
        pools += [qlayer["K"][h], qlayer["V"][h]]
    ranks = np.array([p["ranks"] for p in pools], dtype=np.int32)
    tok = np.concatenate([tok_slabs(u) for p in pools for u in p["U"]], axis=0)
    assert np.array_equal(tok, np.rint(tok)) and tok.min() >= -128 and tok.max() <= 127
    dim = np.concatenate([b.T for p in pools for b in p["B"]], axis=0)
    return ranks, tok.astype(np.int8), to_storage(dim, "bf16")


def stored_layer_8bit(qlayer: dict) -> dict:
    """The 8-bit layer as stored: codes exact, the folded dimension factors rounded to bf16."""
    c = cast_fn("bf16")
    out = dict(qlayer)
    for t in ("K", "V"):
        out[t] = [dict(p, B=[c(b) for b in p["B"]]) for p in qlayer[t]]
    return out
