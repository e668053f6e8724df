"""Workload shapes and the seeded generator of synthetic KV caches.

The five workloads mirror the shapes of Qwen2.5 attention layers
(MILO: Efficient Many-shot ICL with Block-wise Low-rank Compression, §5.1:
Qwen2.5 models, many-shot contexts).  The pages' own datasets are not used;
the caches below stand in for their shapes only.

Every block of keys or values is a low-rank signal plus noise:

    X_b = Gq_b · diag(sigma) · Hq_bᵀ + noise_std · N_b,   sigma_i = exp(-i / tau_b), i = 1..k

with Gq_b (n×k) and Hq_b (d×k) the Q factors of Gaussian matrices (orthonormal
columns), so that with noise_std = 0 the singular values of X_b are exactly
sigma.  Keys additionally get per-channel outlier scales on a few dimensions.

Every random draw comes from a PCG64 stream seeded by
SeedSequence([seed, workload_id, layer, head, tensor, block]) (or a tag in the
block slot), so any block regenerates on its own and the same block is
identical for every caller.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

# Tags for the streams that are not per-block.
_TAG_TAU = 1_000_001
_TAG_OUTLIER = 1_000_002
_TAG_QUERY = 1_000_003
_TAG_SUFFIX = 1_000_004
_TAG_RANGE = 1_000_005
_TAG_MODE = 1_000_006

KEY, VALUE = 0, 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: a stack of attention layers sharing one shape."""

    name: str
    wid: int  # workload id, part of every seed
    layers: int
    kv_heads: int
    q_heads: int
    head_dim: int
    dtype: str  # "f32" or "bf16": the storage dtype of K, V, q, suffix, factors
    context: int  # T, compressed shared-prefix length
    block_size: int  # n, tokens per block
    signal_rank: int  # k
    tau: tuple  # ("fixed", values) | ("loguniform", lo, hi) | ("layer_range", lo, hi) | ("bimodal", lo1, hi1, lo2, hi2)
    noise_std: float
    outlier_dims: int  # key channels with outlier scales (0 = none)
    outlier_range: tuple
    budgets: tuple  # storage budgets beta
    r_min: int
    batch: int  # decode queries
    suffix: int  # S, uncompressed per-query suffix length
    seed: int = 0

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def num_blocks(self) -> int:
        return self.context // self.block_size

    @property
    def rows(self) -> int:
        """Query rows that share one KV head's factors: batch × GQA group."""
        return self.batch * self.group


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 0, 1, 1, 2, 64, "f32", 1024, 256, 40, ("fixed", (2.0, 4.0, 8.0, 16.0)),
                 1e-3, 0, (1.0, 1.0), (0.5,), 4, 1, 0),
        Workload("qwen2.5-0.5b-layer", 1, 1, 2, 14, 64, "bf16", 16384, 512, 48, ("loguniform", 2.0, 32.0),
                 1e-3, 0, (1.0, 1.0), (0.5,), 4, 8, 64),
        Workload("qwen2.5-7b-layer", 2, 1, 4, 28, 128, "bf16", 32768, 512, 96, ("loguniform", 2.0, 48.0),
                 1e-3, 4, (1.0, 8.0), (0.5,), 4, 16, 256),
        Workload("qwen2.5-7b-stack", 3, 28, 4, 28, 128, "bf16", 131072, 512, 96, ("layer_range", 2.0, 64.0),
                 1e-3, 4, (1.0, 8.0), (0.5,), 4, 32, 256),
        Workload("qwen2.5-32b-stack", 4, 64, 8, 40, 128, "bf16", 65536, 1024, 96,
                 ("bimodal", 1.0, 4.0, 32.0, 96.0), 1e-3, 4, (1.0, 8.0), (0.25, 0.5, 0.75), 4, 64, 512),
    ]
}


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(k) for k in key])))


def _loguniform(rng: np.random.Generator, lo: float, hi: float, size=None):
    return np.exp(rng.uniform(math.log(lo), math.log(hi), size=size))


def block_taus(wl: Workload, layer: int, head: int) -> np.ndarray:
    """Decay constant tau_b of every block of one (layer, KV head); K and V share it."""
    nb = wl.num_blocks
    kind = wl.tau[0]
    if kind == "fixed":
        vals = np.asarray(wl.tau[1], dtype=np.float64)
        return np.resize(vals, nb)
    rng = _rng(wl.seed, wl.wid, layer, head, _TAG_TAU)
    if kind == "loguniform":
        return _loguniform(rng, wl.tau[1], wl.tau[2], nb)
    if kind == "layer_range":
        lo, hi = np.sort(_loguniform(_rng(wl.seed, wl.wid, layer, _TAG_RANGE), wl.tau[1], wl.tau[2], 2))
        return _loguniform(rng, lo, hi, nb)
    if kind == "bimodal":
        low = np.zeros(nb, dtype=bool)
        low[rng.permutation(nb)[: nb // 2]] = True
        t = np.empty(nb)
        t[low] = _loguniform(rng, wl.tau[1], wl.tau[2], int(low.sum()))
        t[~low] = _loguniform(rng, wl.tau[3], wl.tau[4], int((~low).sum()))
        return t
    raise ValueError(kind)


def outlier_scales(wl: Workload, layer: int, head: int) -> np.ndarray:
    """Per-channel key scales: U[lo, hi] on `outlier_dims` random channels, 1 elsewhere."""
    s = np.ones(wl.head_dim)
    if wl.outlier_dims:
        rng = _rng(wl.seed, wl.wid, layer, head, _TAG_OUTLIER)
        dims = rng.choice(wl.head_dim, size=wl.outlier_dims, replace=False)
        s[dims] = rng.uniform(wl.outlier_range[0], wl.outlier_range[1], size=wl.outlier_dims)
    return s


def _lowrank_plus_noise(rng: np.random.Generator, rows: int, d: int, k: int, tau: float,
                        noise_std: float) -> np.ndarray:
    k = min(k, rows, d)
    g = rng.standard_normal((rows, k))
    h = rng.standard_normal((d, k))
    noise = rng.standard_normal((rows, d))
    gq, _ = np.linalg.qr(g)
    hq, _ = np.linalg.qr(h)
    sigma = np.exp(-np.arange(1, k + 1, dtype=np.float64) / tau)
    return (gq * sigma) @ hq.T + noise_std * noise


def gen_block_f64(wl: Workload, layer: int, head: int, tensor: int, block: int, tau: float,
                  noise_std: float | None = None, signal_rank: int | None = None) -> np.ndarray:
    """One n×d block in fp64, before outlier scaling and the storage cast."""
    rng = _rng(wl.seed, wl.wid, layer, head, tensor, block)
    return _lowrank_plus_noise(rng, wl.block_size, wl.head_dim,
                               wl.signal_rank if signal_rank is None else signal_rank, tau,
                               wl.noise_std if noise_std is None else noise_std)


def gen_pool_f64(wl: Workload, layer: int, head: int, tensor: int, taus=None,
                 noise_std: float | None = None) -> np.ndarray:
    """All blocks of one (layer, head, K|V) stacked to [T][d] fp64, outliers applied to keys."""
    taus = block_taus(wl, layer, head) if taus is None else np.asarray(taus, dtype=np.float64)
    x = np.concatenate([gen_block_f64(wl, layer, head, tensor, b, float(taus[b]), noise_std)
                        for b in range(wl.num_blocks)], axis=0)
    if tensor == KEY:
        x = x * outlier_scales(wl, layer, head)
    return x


def gen_queries(wl: Workload, layer: int) -> np.ndarray:
    """Decode queries q[batch][q_heads][d] ~ N(0, 1) in fp64."""
    rng = _rng(wl.seed, wl.wid, layer, _TAG_QUERY)
    return rng.standard_normal((wl.batch, wl.q_heads, wl.head_dim))


def gen_suffix(wl: Workload, layer: int, tensor: int) -> np.ndarray:
    """Per-query uncompressed suffix [batch][kv_heads][S][d] in fp64 (one extra low-rank block each)."""
    S = wl.suffix
    out = np.zeros((wl.batch, wl.kv_heads, S, wl.head_dim))
    if S == 0:
        return out
    for i in range(wl.batch):
        for h in range(wl.kv_heads):
            rng = _rng(wl.seed, wl.wid, layer, h, tensor, _TAG_SUFFIX, i)
            kind = wl.tau[0]
            if kind == "fixed":
                tau = float(rng.choice(np.asarray(wl.tau[1])))
            elif kind == "bimodal":
                lo, hi = (wl.tau[1], wl.tau[2]) if rng.uniform() < 0.5 else (wl.tau[3], wl.tau[4])
                tau = float(_loguniform(rng, lo, hi))
            else:
                tau = float(_loguniform(rng, wl.tau[1], wl.tau[2]))
            x = _lowrank_plus_noise(rng, S, wl.head_dim, wl.signal_rank, tau, wl.noise_std)
            if tensor == KEY:
                x = x * outlier_scales(wl, layer, h)
            out[i, h] = x
    return out


# ---- storage casts (no method arithmetic: round-to-nearest-even to the storage type) ----

def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp64 → fp32 → bf16 (round to nearest even); returns the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_storage(x: np.ndarray, dtype: str) -> np.ndarray:
    """fp64 → storage array: float32 for "f32", uint16 bf16 bit patterns for "bf16"."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return f64_to_bf16_bits(x)
    raise ValueError(dtype)


def from_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """Storage array → the exact fp64 values it holds."""
    if dtype == "f32":
        return np.asarray(a, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_bits_to_f64(a)
    raise ValueError(dtype)


def gen_layer(wl: Workload, layer: int = 0, taus=None, heads=None) -> dict:
    """One layer's inputs in storage dtype.

    Returns K, V [kv_heads][T][d], q [batch][q_heads][d], K_suf, V_suf [batch][kv_heads][S][d]
    and the per-head taus used.  `taus` may override the per-head decay constants
    (list of arrays, one per head).  `heads` restricts generation to a subset of KV heads
    (the others are left zero) for sampled checks.
    """
    H, T, d = wl.kv_heads, wl.context, wl.head_dim
    heads = range(H) if heads is None else heads
    K = np.zeros((H, T, d))
    V = np.zeros((H, T, d))
    used = []
    for h in range(H):
        t = block_taus(wl, layer, h) if taus is None else np.asarray(taus[h], dtype=np.float64)
        used.append(t)
        if h in heads:
            K[h] = gen_pool_f64(wl, layer, h, KEY, t)
            V[h] = gen_pool_f64(wl, layer, h, VALUE, t)
    return dict(
        K=to_storage(K, wl.dtype), V=to_storage(V, wl.dtype),
        q=to_storage(gen_queries(wl, layer), wl.dtype),
        K_suf=to_storage(gen_suffix(wl, layer, KEY), wl.dtype),
        V_suf=to_storage(gen_suffix(wl, layer, VALUE), wl.dtype),
        taus=used,
    )
