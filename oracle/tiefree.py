"""Choose generator decay constants whose rank allocation has no near-tie.

TEST INFRASTRUCTURE ONLY.  Integer ranks are compared bit for bit between the
CUDA path (fp32 eigen-decomposition) and this oracle (fp64 SVD).  Largest-
remainder rounding is a step function of the real quotas: it only changes
where the fractional part of the last block that receives the extra unit
meets the fractional part of the first block that does not.  (A quota that
crosses an integer does not change the result: its floor moves by one and the
number of extra units moves the other way.)  So the allocation is stable under
a quota error e when that cut gap exceeds 2e.  This module nudges the decay
constant of a block at the cut until the gap of every pool is at least delta.
"""
from __future__ import annotations

import numpy as np

from synth import workloads as wlmod

from .milo import allocate_ranks, block_svd, rank_total, spectral_entropy


def cut_gap(quotas: np.ndarray, R: int) -> tuple[float, int]:
    """Gap between the rem-th and (rem+1)-th largest fractional parts, and the block after the cut."""
    q = np.asarray(quotas, dtype=np.float64)
    fl = np.floor(q)
    frac = q - fl
    rem = R - int(fl.sum())
    nb = q.size
    if rem <= 0 or rem >= nb:
        return (np.inf if np.all(frac == 0.0) else 0.0), -1
    order = np.lexsort((np.arange(nb), -frac))
    return float(frac[order[rem - 1]] - frac[order[rem]]), int(order[rem])


def greedy_cut_gap(sigma, R: int, r_min: int, d: int) -> float:
    """Margin of the greedy marginal-gain allocation (allocate_ranks_greedy).

    The greedy hands the R − nb·r_min free units to the largest next-component shares; its
    result only changes where the smallest share it took meets the largest share it left
    (across blocks, with blocks already at d excluded).  Returns that difference (inf when
    no unit is free or none is left), so a GPU whose shares are off by less than half of it
    makes the same choices."""
    sigma = np.asarray(sigma, dtype=np.float64)
    nb = sigma.shape[0]
    if R <= nb * r_min or R >= nb * d:
        return float("inf")
    e = sigma[:, :d] ** 2
    t = e.sum(axis=1, keepdims=True)
    share = np.divide(e, t, out=np.zeros_like(e), where=t > 0)
    free = share[:, r_min:d]  # candidate units i = r_min+1 .. d of every block (0-based columns r_min..d-1)
    vals = np.sort(free.ravel())[::-1]
    k = R - nb * r_min
    return float(vals[k - 1] - vals[k])


def _block_entropy(wl, layer, head, tensor, b, tau):
    x = wlmod.gen_block_f64(wl, layer, head, tensor, b, tau)
    if tensor == wlmod.KEY:
        x = x * wlmod.outlier_scales(wl, layer, head)
    stored = wlmod.from_storage(wlmod.to_storage(x, wl.dtype), wl.dtype)
    return spectral_entropy(block_svd(stored)[0])


def tiefree_taus(wl, layer: int, beta: float, delta: float, heads=None, max_iter: int = 400):
    """Per-head decay constants (list of arrays) whose K and V pools both have cut gap >= delta."""
    T, n, d = wl.context, wl.block_size, wl.head_dim
    R = rank_total(beta, T, n, d)
    heads = range(wl.kv_heads) if heads is None else heads
    result = [wlmod.block_taus(wl, layer, h) for h in range(wl.kv_heads)]
    for h in heads:
        taus = result[h].copy()
        ent = {t: np.array([_block_entropy(wl, layer, h, t, b, taus[b]) for b in range(wl.num_blocks)])
               for t in (wlmod.KEY, wlmod.VALUE)}
        for it in range(1, max_iter + 1):
            worst = None
            for t in (wlmod.KEY, wlmod.VALUE):
                if R >= wl.num_blocks * d:
                    continue
                _, q, _ = allocate_ranks(np.exp(ent[t]), R, wl.r_min, d)
                gap, blk = cut_gap(q, R)
                if gap < delta:
                    worst = blk
                    break
            if worst is None:
                break
            taus[worst] *= 1.0 + 1e-3 * it
            for t in (wlmod.KEY, wlmod.VALUE):
                ent[t][worst] = _block_entropy(wl, layer, h, t, worst, taus[worst])
        else:
            raise RuntimeError(f"no tie-free taus for head {h} after {max_iter} nudges")
        result[h] = taus
    return result
