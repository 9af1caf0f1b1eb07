"""fp64 oracle of the QSA compressed lightweight indexer (numpy, plain loops where it helps).

TEST INFRASTRUCTURE ONLY, like the rest of oracle/: imported by tests/ and nothing in the
library. It shares no code with the CUDA path.

What it computes (joezjh.github.io notes page "Qwen3.8-Flash-Next", section on Qwen Sparse
Attention, "压缩轻量级 Indexer": the query/key projections, the key compression equation,
Partial RoPE, the block-causal importance equation, the Top-K block selection and the final
token set; pwwt.cn translation, section on QSA implementation details: four indexer query
heads, one shared key head, token budget K = 2048 and compression ratio r = 4). The
projections W x are inputs. For one sequence of n tokens:

    q^_i^h = RMSNorm(qx_i^h)                         per query head h, over d
    k^_b   = RMSNorm(mean_{j<r} kx_{b r + j})        b < floor(n / r): non-overlapping blocks
    q_i^h  = PRoPE(q^_i^h, i),   k_b = PRoPE(k^_b, b r)   (compress first, then rotate)
    I_ib   = sum_h ReLU(<q_i^h, k_b>)   if b r + r - 1 <= i,  else -inf
    B_i    = the K_B = ceil(K / r) blocks of largest I_ib (only finite ones)
    S_i    = tokens of the blocks in B_i, plus the tail r floor((i+1)/r) .. i

Readings where the pages are silent (each a parameter here):
- RMSNorm is the zero-centred form used throughout the model: x / sqrt(mean(x^2) + eps) *
  (1 + w), eps = 1e-6.
- PRoPE rotates the first `rot` = 64 of the d = 128 dimensions, pairing dimension j with
  j + rot/2 (the half-split convention), with angle pos * base^(-2j/rot), base = 10000;
  the other dimensions pass through.
- Ties in the top-K are broken by the lower block index, so the selected set is unique.
"""
from __future__ import annotations

import math

import numpy as np


def rmsnorm(x, w, eps=1e-6):
    """x / sqrt(mean(x^2) + eps) * (1 + w) over the last axis (zero-centred weight w)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * (1.0 + np.asarray(w, np.float64))


def prope(x, pos, rot=64, base=10000.0):
    """Rotate the first `rot` dimensions of x (last axis) by position `pos` (scalar or an array
    broadcasting over x's leading axes): pairs (j, j + rot/2), angle pos * base^(-2j/rot)."""
    x = np.array(x, dtype=np.float64, copy=True)
    half = rot // 2
    j = np.arange(half, dtype=np.float64)
    ang = np.asarray(pos, dtype=np.float64)[..., None] * base ** (-2.0 * j / rot)
    c, s = np.cos(ang), np.sin(ang)
    a, b = x[..., :half].copy(), x[..., half:rot].copy()
    x[..., :half] = a * c - b * s
    x[..., half:rot] = b * c + a * s
    return x


def compress_keys(kx, r, wk, eps=1e-6, rot=64, base=10000.0):
    """k_b = PRoPE(RMSNorm(AvgPool_r(kx)), b r) for b < floor(n / r). kx: [n, d]."""
    kx = np.asarray(kx, dtype=np.float64)
    nb = kx.shape[0] // r
    kb = np.zeros((nb, kx.shape[1]))
    for b in range(nb):
        kb[b] = kx[b * r:(b + 1) * r].mean(axis=0)
    kb = rmsnorm(kb, wk, eps)
    return prope(kb, np.arange(nb) * r, rot, base)


def scores(qx, kx, r, wq, wk, eps=1e-6, rot=64, base=10000.0):
    """I [n, floor(n / r)]: block-causal sum over heads of ReLU(<q_i^h, k_b>), -inf where the
    block is not complete at or before token i. qx: [n, Hq, d]; kx: [n, d]."""
    qx = np.asarray(qx, dtype=np.float64)
    n, Hq, d = qx.shape
    q = prope(rmsnorm(qx, wq, eps), np.arange(n)[:, None] * np.ones((1, Hq)), rot, base)
    kb = compress_keys(kx, r, wk, eps, rot, base)
    nb = kb.shape[0]
    I = np.full((n, nb), -np.inf)
    for i in range(n):
        for b in range(nb):
            if b * r + r - 1 <= i:
                I[i, b] = sum(max(0.0, float(np.dot(q[i, h], kb[b]))) for h in range(Hq))
    return I


def select_blocks(I, K, r):
    """B_i: indices of the K_B = ceil(K / r) largest finite scores of row i, ordered by score
    (descending) then block index; rows with fewer finite scores are padded with -1."""
    I = np.asarray(I, dtype=np.float64)
    kb = int(math.ceil(K / r))
    n, nb = I.shape
    out = np.full((n, kb), -1, dtype=np.int64)
    for i in range(n):
        cand = [(-I[i, b], b) for b in range(nb) if np.isfinite(I[i, b])]
        cand.sort()
        for j, (_, b) in enumerate(cand[:kb]):
            out[i, j] = b
    return out


def token_set(blocks_i, i, r):
    """S_i: the tokens of the selected blocks plus the tail r floor((i+1)/r) .. i, sorted."""
    toks = set()
    for b in blocks_i:
        if b >= 0:
            toks.update(range(b * r, b * r + r))
    toks.update(range(r * ((i + 1) // r), i + 1))
    return sorted(toks)


def indexer(qx, kx, wq, wk, K=2048, r=4, eps=1e-6, rot=64, base=10000.0):
    """Scores and selected blocks of one sequence: (I [n, nb], B [n, ceil(K / r)])."""
    I = scores(qx, kx, r, wq, wk, eps, rot, base)
    return I, select_blocks(I, K, r)
