"""fp64 oracle of the decode over pre-RoPE key factors: reconstruct each block's keys, rotate them, attend.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: page "MILO: Efficient Many-shot In-Context Learning with Block-wise
Low-rank Compression": pre-RoPE keys are more low-rank than the rotated ones
and suit low-rank compression better (§3, Figure 1), and at inference the
selected blocks are reconstructed before attention (§4.4, §4.5).  The page
gives no RoPE formula.  Readings taken here:

* The compressed keys are the keys before the rotary embedding; the factor
  pair of block b reconstructs them as K̂_b = U_b·B_bᵀ (n×d).
* Rotary embedding in the half-split form: dimension i < d/2 pairs with
  i + d/2 and the pair turns by the angle pos·θ^(−2i/d):
      y_i       = x_i·cos φ_i − x_{i+d/2}·sin φ_i
      y_{i+d/2} = x_{i+d/2}·cos φ_i + x_i·sin φ_i,    φ_i = pos·θ^(−2i/d).
  θ (the rotary base) is an argument; the Qwen2.5 models use 10^6.
* Positions: token t of the compressed prefix sits at position t (block b
  covers b·n .. b·n + n − 1).  The queries and the uncompressed suffix keys
  are given already rotated at their own positions, as a serving cache holds
  them, so only the reconstructed prefix keys are rotated here.
* Values are untouched by RoPE and keep the rank-space form (p·P_b)·Q_bᵀ.
"""
from __future__ import annotations

import math

import numpy as np


def inv_freq(d: int, theta: float) -> np.ndarray:
    """θ^(−2i/d) for i = 0 .. d/2 − 1, fp64."""
    return np.power(float(theta), -2.0 * np.arange(d // 2, dtype=np.float64) / d)


def apply_rope(x, positions, theta: float) -> np.ndarray:
    """Rotate rows of x [m][d] at the given positions [m] (half-split pairs), fp64."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[1]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * inv_freq(d, theta)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[:, :d // 2], x[:, d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def rotated_prefix_keys(pool: dict, n: int, theta: float) -> np.ndarray:
    """One key pool's reconstructed and rotated prefix keys [T][d] (block b at positions b·n ..)."""
    keys = [u @ b.T for u, b in zip(pool["U"], pool["B"])]
    T = n * len(keys)
    return apply_rope(np.concatenate(keys, axis=0), np.arange(T), theta)


def decode_attention_rope(q: np.ndarray, layer: dict, K_suf: np.ndarray, V_suf: np.ndarray, theta: float,
                          scale: float | None = None, block_mask=None) -> np.ndarray:
    """Softmax decode attention with pre-RoPE key factors: keys reconstructed per block, rotated at their
    positions, scored densely; values in rank space; one softmax over prefix ∪ the query's suffix.

    q [Bq][Hq][d] and the suffix [Bq][H][S][d] are post-RoPE; block_mask [H][nb] (True = attended) or None.
    Returns [Bq][Hq][d].
    """
    q = np.asarray(q, dtype=np.float64)
    Bq, Hq, d = q.shape
    H = len(layer["K"])
    G = Hq // H
    scale = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else scale
    out = np.zeros((Bq, Hq, d))
    for h in range(H):
        kp, vp = layer["K"][h], layer["V"][h]
        n = kp["U"][0].shape[0]
        nb = len(kp["U"])
        keep = [b for b in range(nb) if block_mask is None or block_mask[h][b]]
        krot = rotated_prefix_keys(kp, n, theta)
        keys = np.concatenate([krot[b * n:(b + 1) * n] for b in keep], axis=0) if keep else np.zeros((0, d))
        for i in range(Bq):
            for g in range(G):
                qv = q[i, h * G + g]
                s = scale * np.concatenate([keys @ qv, K_suf[i, h] @ qv])
                e = np.exp(s - s.max())
                acc = np.zeros(d)
                for k, b in enumerate(keep):
                    acc += (e[k * n:(k + 1) * n] @ vp["U"][b]) @ vp["B"][b].T
                acc += e[len(keep) * n:] @ V_suf[i, h]
                out[i, h * G + g] = acc / e.sum()
    return out
