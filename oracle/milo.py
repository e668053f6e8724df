"""fp64 oracle: truncated SVD per block, spectral entropy, rank allocation, attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Plain NumPy, fp64, no
blocking or fusion: each function is the definition it cites.

Notation (page "MILO: Efficient Many-shot In-Context Learning with Block-wise
Low-rank Compression"): a pool is the cache of one tensor (K or V) of one KV
head of one layer, [T][d]; it is split into nb = T / n blocks X_b of n tokens
(§4.2).  Each block is stored as a rank-r_b pair: a token-side factor
U_b = X_b · B_b (n×r_b) and a dimension-side factor B_b (d×r_b, orthonormal
columns), so that X_b ≈ U_b · B_bᵀ.  For values the same pair is written
P_b, Q_b.
"""
from __future__ import annotations

import math

import numpy as np


class BudgetError(ValueError):
    """The storage budget cannot give every block the minimum rank."""


# ---------------------------------------------------------------- compression

def block_svd(x: np.ndarray):
    """Singular values (descending) and right singular vectors of one block.

    §4.2: each block's keys and values get their own low-rank approximation.
    By the Eckart–Young theorem the best rank-r approximation in Frobenius
    norm keeps the r leading singular triplets, so the oracle computes the SVD
    x = A · diag(sigma) · Bᵀ with LAPACK and returns (sigma, B) with B's
    columns the right singular vectors, sigma_1 >= sigma_2 >= ...
    """
    x = np.asarray(x, dtype=np.float64)
    _, sigma, bt = np.linalg.svd(x, full_matrices=False)
    return sigma, bt.T


def spectral_entropy(sigma: np.ndarray) -> float:
    """Entropy of the normalised energy spectrum of a block.

    §1 and §4.3 assign rank by each block's entropy, favouring slowly decaying
    spectra.  Reading (the page gives no formula): p_i = sigma_i² / Σ_j sigma_j²
    over all min(n, d) singular values, H = −Σ p_i ln p_i (natural log,
    0·ln 0 = 0).  An all-zero block has H = 0.
    """
    e = np.asarray(sigma, dtype=np.float64) ** 2
    tot = e.sum()
    if tot <= 0.0:
        return 0.0
    p = e / tot
    p = p[p > 0.0]
    return float(-(p * np.log(p)).sum())


def rank_total(beta: float, T: int, n: int, d: int) -> int:
    """Total rank R of one pool under a storage budget beta.

    Reading of "50% rank budget" (§5.2) as "50% KV memory" (the summary's
    result line): a rank-r block stores r·(n + d) numbers against n·d raw,
    so the largest total rank whose factors fit in beta of the raw pool is
    R = floor(beta · T · d / (n + d)).
    """
    return int(math.floor(beta * float(T * d) / float(n + d)))


def allocate_ranks(w, R: int, r_min: int, d: int):
    """Integer ranks proportional to the weights w_b = exp(H_b), summing to R.

    §4.3 allocates a fixed total rank budget over blocks by entropy.  Reading:
    real quotas q_b = clamp(lam · w_b, r_min, d) with the scalar lam chosen so
    that Σ_b q_b = R, then largest-remainder rounding: r_b = floor(q_b), and
    the R − Σ floor(q_b) blocks with the largest fractional parts get one more
    (ties to the lower block index).

    Σ_b clamp(lam·w_b, r_min, d) is continuous, piecewise linear and
    non-decreasing in lam, with kinks at r_min / w_b and d / w_b; lam is found
    exactly by evaluating the sum at the kinks and solving the linear piece
    that crosses R.

    Returns (ranks int64[nb], quotas float64[nb], lam).
    Raises BudgetError if R < nb · r_min.  If R >= nb · d every rank is d.
    """
    w = np.asarray(w, dtype=np.float64)
    nb = w.size
    if R < nb * r_min:
        raise BudgetError(f"total rank {R} < {nb} blocks x r_min {r_min}")
    if R >= nb * d:
        return np.full(nb, d, dtype=np.int64), np.full(nb, float(d)), math.inf

    def total(lam):
        return float(np.clip(lam * w, r_min, d).sum())

    kinks = np.unique(np.concatenate([r_min / w, d / w]))
    vals = np.array([total(k) for k in kinks])
    j = int(np.argmax(vals >= R))  # vals[-1] = nb·d > R, so some kink qualifies
    if vals[j] == R:
        lam = float(kinks[j])
    else:
        lo, hi = kinks[j - 1], kinks[j]
        mid = 0.5 * (lo + hi)
        low = mid * w <= r_min
        high = mid * w >= d
        free = ~(low | high)
        fixed = r_min * int(low.sum()) + d * int(high.sum())
        lam = (R - fixed) / float(w[free].sum())
    q = np.clip(lam * w, r_min, d)
    ranks = np.floor(q).astype(np.int64)
    rem = R - int(ranks.sum())
    frac = q - ranks
    order = np.lexsort((np.arange(nb), -frac))  # frac descending, then index ascending
    ranks[order[:rem]] += 1
    return ranks, q, lam


def allocate_ranks_greedy(sigma, R: int, r_min: int, d: int) -> np.ndarray:
    """Greedy marginal-gain allocation, the form §4.3 describes in words.

    The allocation starts every block at the minimum rank and then hands out the
    remaining rank units one at a time, each to the block with the largest marginal
    gain.  Reading of "marginal information gain": the share of the block's spectral
    energy carried by its next component, g_b(i) = σ_{b,i}² / Σ_j σ_{b,j}² for
    i = r_b + 1 (the distribution whose entropy H_b is), so blocks whose spectrum decays
    slowly keep receiving units; ties go to the lower block index; a block at rank d
    takes no more.  sigma: [nb][d] singular values per block, descending.

    Returns ranks int64[nb].  Raises BudgetError if R < nb · r_min; R >= nb · d gives d
    everywhere.
    """
    sigma = np.asarray(sigma, dtype=np.float64)
    nb = sigma.shape[0]
    if R < nb * r_min:
        raise BudgetError(f"total rank {R} < {nb} blocks x r_min {r_min}")
    if R >= nb * d:
        return np.full(nb, d, dtype=np.int64)
    energy = sigma[:, :d] ** 2
    tot = energy.sum(axis=1)
    share = np.divide(energy, tot[:, None], out=np.zeros_like(energy), where=tot[:, None] > 0)
    ranks = np.full(nb, r_min, dtype=np.int64)
    for _ in range(R - nb * r_min):
        gain = np.where(ranks < d, share[np.arange(nb), np.minimum(ranks, d - 1)], -np.inf)
        b = int(np.argmax(gain))  # first maximum: ties to the lower block index
        ranks[b] += 1
    return ranks


def allocate_ranks_uniform(nb: int, R: int, r_min: int, d: int) -> np.ndarray:
    """Uniform baseline of §5.3's allocation comparison: every block floor(R / nb), the
    R mod nb leftover units to the lowest block indices, within [r_min, d]."""
    if R < nb * r_min:
        raise BudgetError(f"total rank {R} < {nb} blocks x r_min {r_min}")
    if R >= nb * d:
        return np.full(nb, d, dtype=np.int64)
    ranks = np.full(nb, R // nb, dtype=np.int64)
    ranks[: R % nb] += 1
    return ranks


def allocate_ranks_random(nb: int, R: int, r_min: int, d: int, rng) -> np.ndarray:
    """Random baseline of §5.3's allocation comparison: ranks proportional to weights drawn
    uniformly from [1, d] (the range of e^{H_b}), with the same water-filling and rounding
    as the entropy rule.  rng: a numpy Generator (the caller seeds it)."""
    w = rng.uniform(1.0, float(d), size=nb)
    return allocate_ranks(w, R, r_min, d)[0]


def compress_pool(x: np.ndarray, n: int, beta: float, r_min: int) -> dict:
    """Compress one pool [T][d]: partition, per-block SVD, entropy, ranks, factors.

    §4.4 encoding: partition the context into blocks, analyse block entropy,
    store low-rank caches.  Reading: the budget is per pool (one tensor of
    one KV head of one layer), K and V allocated separately (§4.4 notes key
    and value ranks may differ); T must be a multiple of n.

    Returns dict with sigma [nb][d], entropy [nb], weights [nb], R, quotas,
    ranks, U (list of n×r_b), B (list of d×r_b).  U_b = X_b · B_b (singular
    values folded into the token-side factor).
    """
    x = np.asarray(x, dtype=np.float64)
    T, d = x.shape
    if T % n:
        raise ValueError("context length must be a multiple of the block size")
    nb = T // n
    sig, vecs, ent = [], [], []
    for b in range(nb):
        s, bv = block_svd(x[b * n:(b + 1) * n])
        sig.append(s)
        vecs.append(bv)
        ent.append(spectral_entropy(s))
    ent = np.array(ent)
    weights = np.exp(ent)
    R = rank_total(beta, T, n, d)
    ranks, quotas, lam = allocate_ranks(weights, R, r_min, d)
    U, B = [], []
    for b in range(nb):
        r = int(ranks[b])
        br = vecs[b][:, :r]
        U.append(x[b * n:(b + 1) * n] @ br)
        B.append(br)
    return dict(sigma=np.array(sig), entropy=ent, weights=weights, R=R, quotas=quotas, lam=lam,
                ranks=ranks, U=U, B=B, n=n, d=d)


def compress_layer(K: np.ndarray, V: np.ndarray, n: int, beta: float, r_min: int) -> dict:
    """Compress every (KV head, K|V) pool of one layer. K, V: [H][T][d]."""
    H = K.shape[0]
    return dict(K=[compress_pool(K[h], n, beta, r_min) for h in range(H)],
                V=[compress_pool(V[h], n, beta, r_min) for h in range(H)])


ALLOC_RULES = ("entropy", "greedy", "uniform", "weights")
POOL_SCOPES = ("pool", "layer")


def allocate_blocks(rule: str, sigma, R: int, r_min: int, d: int, weights=None):
    """Ranks of a set of blocks under one allocation rule, summing to R.

    The rules are the entropy rule of §4.3 (ranks ∝ exp(H_b), water-filling and largest
    remainder), the greedy marginal-gain form §4.3 describes in words, and the two baselines
    §5.3 compares against: uniform, and random (ranks ∝ weights drawn by the caller, passed
    in as `weights`, with the entropy rule's water-filling).  sigma: [nb][d] singular values.

    Returns (ranks int64[nb], quotas float64[nb] or None for the rules without quotas).
    """
    sigma = np.asarray(sigma, dtype=np.float64)
    nb = sigma.shape[0]
    if rule == "entropy":
        w = np.exp([spectral_entropy(s) for s in sigma])
        r, q, _ = allocate_ranks(w, R, r_min, d)
        return r, q
    if rule == "weights":
        r, q, _ = allocate_ranks(np.asarray(weights, dtype=np.float64), R, r_min, d)
        return r, q
    if rule == "greedy":
        return allocate_ranks_greedy(sigma, R, r_min, d), None
    if rule == "uniform":
        return allocate_ranks_uniform(nb, R, r_min, d), None
    raise ValueError(rule)


def compress_layer_rule(K: np.ndarray, V: np.ndarray, n: int, beta: float, r_min: int, rule: str = "entropy",
                        scope: str = "pool", weights=None, ranks=None) -> dict:
    """Compress one layer with a chosen allocation rule and budget scope.

    scope "pool": each (KV head, K|V) pool gets R = floor(beta·T·d/(n+d)) rank units
    (compress_layer with the entropy rule).  scope "layer": the layer's pools share one
    budget, P·R units over all P·nb blocks (the "global rank budget" of §4.3 taken over the
    layer), with the blocks in the order pool p = 2h + t (t = 0 keys, 1 values), then block.
    weights: [P][nb] for rule "weights".  Factors are computed as in compress_pool.
    ranks: optional [P][nb] integers that replace the allocation (factors at given ranks, to
    compare outputs once the integer decisions have been compared on their own).
    Returns compress_layer's structure; each pool also carries its own rank sum as "R", and
    the layer dict carries "R_total".
    """
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    H, T, d = K.shape
    if T % n:
        raise ValueError("context length must be a multiple of the block size")
    nb = T // n
    P = 2 * H
    xs = [(K if p % 2 == 0 else V)[p // 2] for p in range(P)]
    svd = [[block_svd(x[b * n:(b + 1) * n]) for b in range(nb)] for x in xs]
    sig = np.array([[s for s, _ in pool] for pool in svd])  # [P][nb][d]
    R = rank_total(beta, T, n, d)
    w = None if weights is None else np.asarray(weights, dtype=np.float64).reshape(P, nb)
    given = ranks
    ranks = np.zeros((P, nb), dtype=np.int64)
    quotas = np.full((P, nb), np.nan)
    if given is not None:
        ranks[:] = np.asarray(given, dtype=np.int64).reshape(P, nb)
    elif scope == "pool":
        for p in range(P):
            r, q = allocate_blocks(rule, sig[p], R, r_min, d, None if w is None else w[p])
            ranks[p] = r
            if q is not None:
                quotas[p] = q
    elif scope == "layer":
        r, q = allocate_blocks(rule, sig.reshape(P * nb, -1), P * R, r_min, d, None if w is None else w.ravel())
        ranks[:] = r.reshape(P, nb)
        if q is not None:
            quotas[:] = q.reshape(P, nb)
    else:
        raise ValueError(scope)
    pools = []
    for p in range(P):
        U, B = [], []
        for b in range(nb):
            br = svd[p][b][1][:, :int(ranks[p, b])]
            U.append(xs[p][b * n:(b + 1) * n] @ br)
            B.append(br)
        ent = np.array([spectral_entropy(s) for s in sig[p]])
        pools.append(dict(sigma=sig[p], entropy=ent, weights=np.exp(ent), R=int(ranks[p].sum()), quotas=quotas[p],
                          ranks=ranks[p], U=U, B=B, n=n, d=d))
    return dict(K=pools[0::2], V=pools[1::2], R_total=int(ranks.sum()))


def reconstruct_pool(pool: dict) -> np.ndarray:
    """Dense [T][d] reconstruction Σ_b U_b · B_bᵀ stacked over blocks."""
    return np.concatenate([u @ b.T for u, b in zip(pool["U"], pool["B"])], axis=0)


def stored_factors(pool: dict, cast) -> dict:
    """The pool with its factors passed through the storage cast `cast` (fp64 → stored fp64)."""
    out = dict(pool)
    out["U"] = [cast(u) for u in pool["U"]]
    out["B"] = [cast(b) for b in pool["B"]]
    return out


# ---------------------------------------------------------------- decode

def decode_attention(q: np.ndarray, layer: dict, K_suf: np.ndarray, V_suf: np.ndarray,
                     scale: float | None = None, block_mask=None) -> np.ndarray:
    """Softmax decode attention over the compressed prefix and the per-query suffix, in rank space.

    §4.4 inference attends over the low-rank caches.  With K_b ≈ U_b·B_bᵀ the
    scores of block b are (q · B_b) · U_bᵀ and with V_b ≈ P_b·Q_bᵀ the block's
    value sum is (p · P_b) · Q_bᵀ, so no block is expanded to n×d.
    Readings: every block is attended unless block_mask says otherwise;
    scale = 1/sqrt(d); no RoPE; query head hq reads KV head hq // (Hq / H); the
    prefix is shared by every query and one softmax runs over prefix ∪ that
    query's suffix.

    Block selection (§4.4: decoding retrieves the selected blocks and attends
    sparsely): block_mask [H][nb] of booleans, True = attended; the blocks of a
    KV head that are not selected take no part in that head's softmax, for
    every query.  None selects every block.

    q [Bq][Hq][d]; layer = compress_layer(...) output (possibly with stored
    factors); K_suf, V_suf [Bq][H][S][d] (S may be 0).  Returns [Bq][Hq][d].
    """
    q = np.asarray(q, dtype=np.float64)
    Bq, Hq, d = q.shape
    H = len(layer["K"])
    G = Hq // H
    scale = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else scale
    out = np.zeros((Bq, Hq, d))
    for h in range(H):
        kp, vp = layer["K"][h], layer["V"][h]
        if block_mask is not None:
            keep = [b for b in range(len(kp["U"])) if block_mask[h][b]]
            kp = dict(U=[kp["U"][b] for b in keep], B=[kp["B"][b] for b in keep])
            vp = dict(U=[vp["U"][b] for b in keep], B=[vp["B"][b] for b in keep])
        for i in range(Bq):
            for g in range(G):
                hq = h * G + g
                qv = q[i, hq]
                scores = [(qv @ bk) @ uk.T for uk, bk in zip(kp["U"], kp["B"])]
                scores.append(K_suf[i, h] @ qv)
                s = scale * np.concatenate(scores)
                m = s.max()
                e = np.exp(s - m)
                acc = np.zeros(d)
                pos = 0
                for pv, qb in zip(vp["U"], vp["B"]):
                    nblk = pv.shape[0]
                    acc += (e[pos:pos + nblk] @ pv) @ qb.T
                    pos += nblk
                acc += e[pos:] @ V_suf[i, h]
                out[i, hq] = acc / e.sum()
    return out


def decode_attention_dense(q: np.ndarray, K: np.ndarray, V: np.ndarray, K_suf: np.ndarray,
                           V_suf: np.ndarray, scale: float | None = None) -> np.ndarray:
    """Plain softmax attention over explicit keys and values (prefix [H][T][d] ∪ suffix)."""
    q = np.asarray(q, dtype=np.float64)
    Bq, Hq, d = q.shape
    H = K.shape[0]
    G = Hq // H
    scale = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else scale
    out = np.zeros((Bq, Hq, d))
    for i in range(Bq):
        for hq in range(Hq):
            h = hq // G
            keys = np.concatenate([K[h], K_suf[i, h]], axis=0)
            vals = np.concatenate([V[h], V_suf[i, h]], axis=0)
            s = scale * (keys @ q[i, hq])
            e = np.exp(s - s.max())
            out[i, hq] = (e @ vals) / e.sum()
    return out
