"""fp64 oracle of 8-bit factor storage: asymmetric INT8 codes for the token-side factors.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: page "MILO: Efficient Many-shot In-Context Learning with Block-wise
Low-rank Compression", §5.3 (the compressed caches compose with asymmetric
INT8 and KIVI quantisation for further memory savings).  The page gives no
scheme beyond those names.  Readings taken here:

* What is quantised: the token-side factors U_b (keys) and P_b (values), n×r
  per block, which hold n/(n+d) of a block's factor bytes; the small
  dimension-side factors B_b, Q_b stay in the storage dtype (bf16).
* How: asymmetric 8-bit, one (scale, minimum) pair per rank component of
  each block over the block's n tokens, that is per channel as KIVI does for
  keys; the same rule for the values' factor.  With lo = min_t x_t,
  hi = max_t x_t of one channel, a = (hi − lo)/255 and
  c_t = round((x_t − lo)/a) − 128 in [−128, 127] (round half to even), the
  channel is stored as x̂_t = a·(c_t + 128) + lo.  A constant channel (a = 0)
  gets c_t = −128 and x̂_t = lo.
* Precision of the integer decisions: the codes are taken in fp32 (the
  subtraction, the division by 255 and the division by a each rounded to
  nearest), the precision the kernel works in, so that both sides take the
  same decisions.
* Storage of the scales: folded into the dimension-side factor, with one extra
  component whose token codes are all 1:
      B̂[:, j] = a_j·B[:, j]                     (j < r)
      B̂[:, r] = Σ_j (lo_j + 128·a_j)·B[:, j]
  so that codes_aug · B̂ᵀ = Σ_j x̂_j B_jᵀ exactly, and the decode of
  decode_attention runs unchanged on (codes_aug, B̂) at rank r + 1.
* Blocks stored at full rank r = d, where one more component would exceed the
  head dimension, use the symmetric form instead (zero point 0, no extra
  component): a = max_t |x_t| / 127, c_t = round(x_t / a) in [−127, 127], x̂_t =
  a·c_t (a = 0 gives c_t = 0), and B̂[:, j] = a_j·B[:, j] at rank d.
"""
from __future__ import annotations

import numpy as np

CODE_MIN, CODE_MAX = -128, 127


def quantize_channel(x) -> tuple[np.ndarray, np.float32, np.float32]:
    """One channel (a rank component over a block's tokens) → (int8 codes, scale a, minimum lo), fp32 decisions."""
    x = np.asarray(x, dtype=np.float32)
    lo = x.min()
    hi = x.max()
    a = np.float32(np.float32(hi - lo) / np.float32(255.0))
    if a > 0:
        t = (x - lo) / a  # fp32 subtraction, then fp32 division
        c = np.clip(np.rint(t), 0, 255).astype(np.int32) - 128
    else:
        c = np.full(x.shape, CODE_MIN, dtype=np.int32)
    return c.astype(np.int8), a, lo


def dequantize_channel(codes, a, lo) -> np.ndarray:
    """x̂_t = a·(c_t + 128) + lo, in fp64."""
    return float(a) * (np.asarray(codes, dtype=np.float64) + 128.0) + float(lo)


def quantize_channel_symmetric(x) -> tuple[np.ndarray, np.float32]:
    """One channel in the symmetric form (full-rank blocks) → (int8 codes in [−127, 127], scale a), fp32 decisions."""
    x = np.asarray(x, dtype=np.float32)
    a = np.float32(np.abs(x).max() / np.float32(127.0))
    if a > 0:
        c = np.clip(np.rint(x / a), -127, 127).astype(np.int32)
    else:
        c = np.zeros(x.shape, dtype=np.int32)
    return c.astype(np.int8), a


def quantize_block(u, b) -> dict:
    """One block's pair (U n×r, B d×r, stored values) → the 8-bit form at rank r + 1 (r < d) or r (r = d).

    Returns codes (n×r int8), scale and lo (r each, fp32; lo = 0 in the
    symmetric form), the dequantized token factor u_hat (n×r), and the stored
    pair U_aug (the codes as numbers, plus a last column of 1 when r < d) and
    B_aug (fp64) with U_aug·B_augᵀ = u_hat·Bᵀ.
    """
    u = np.asarray(u, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    n, r = u.shape
    if r >= b.shape[0]:  # full rank: symmetric, no extra component
        codes = np.empty((n, r), dtype=np.int8)
        scale = np.empty(r, dtype=np.float32)
        for j in range(r):
            codes[:, j], scale[j] = quantize_channel_symmetric(u[:, j])
        u_hat = codes.astype(np.float64) * scale.astype(np.float64)[None, :]
        return dict(codes=codes, scale=scale, lo=np.zeros(r, dtype=np.float32), u_hat=u_hat,
                    U_aug=codes.astype(np.float64), B_aug=b * scale.astype(np.float64)[None, :])
    codes = np.empty((n, r), dtype=np.int8)
    scale = np.empty(r, dtype=np.float32)
    lo = np.empty(r, dtype=np.float32)
    u_hat = np.empty((n, r))
    for j in range(r):
        codes[:, j], scale[j], lo[j] = quantize_channel(u[:, j])
        u_hat[:, j] = dequantize_channel(codes[:, j], scale[j], lo[j])
    offset = lo.astype(np.float64) + 128.0 * scale.astype(np.float64)
    b_aug = np.concatenate([b * scale.astype(np.float64)[None, :], (b @ offset)[:, None]], axis=1)
    u_aug = np.concatenate([codes.astype(np.float64), np.ones((n, 1))], axis=1)
    return dict(codes=codes, scale=scale, lo=lo, u_hat=u_hat, U_aug=u_aug, B_aug=b_aug)


def quantize_pool(pool: dict) -> dict:
    """A pool (compress_pool output, factors in stored values) → the same pool in 8-bit form at ranks r_b + 1
    (r_b at full rank).

    The returned pool has U = the stored codes, B = the folded dimension
    factors and ranks = r_b + 1 (r_b at full rank), so decode_attention and
    reconstruct_pool take it as they are; it also keeps codes, scales,
    minima and the dequantized token factors per block.
    """
    blocks = [quantize_block(u, b) for u, b in zip(pool["U"], pool["B"])]
    out = dict(pool)
    out["U"] = [q["U_aug"] for q in blocks]
    out["B"] = [q["B_aug"] for q in blocks]
    out["ranks"] = np.array([q["U_aug"].shape[1] for q in blocks])
    out["codes"] = [q["codes"] for q in blocks]
    out["scale"] = [q["scale"] for q in blocks]
    out["lo"] = [q["lo"] for q in blocks]
    out["u_hat"] = [q["u_hat"] for q in blocks]
    return out


def quantize_layer(layer: dict) -> dict:
    """Every K and V pool of a layer in 8-bit form (quantize_pool)."""
    out = dict(layer)
    out["K"] = [quantize_pool(p) for p in layer["K"]]
    out["V"] = [quantize_pool(p) for p in layer["V"]]
    return out
