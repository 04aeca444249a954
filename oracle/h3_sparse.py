"""fp64 CPU oracle of block-sparse attention (the optional sparse backend).

TEST INFRASTRUCTURE ONLY (same rules as oracle/h3_block.py): only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg may use it.

What the pages fix: "HyperFlow for MiniMax-H3" (model card), summary table and
Performance: an optional sparse attention backend (NVIDIA Sol-Attn), off by
default, an approximation of dense attention (PSNR about 23 dB against the
dense run). The pages do not describe its method.

Reading taken (listed in the design notes): block-sparse attention with a
selection by pooled scores.
s1. The sequence is cut into key tiles of 128 rows and query blocks of 256
    rows (two query tiles). Pooled vectors are means over a tile's / block's
    valid (non-padding) rows, per head.
s2. Score(block B, tile J, head h) = mean q_B,h . mean k_J,h. Candidate tiles
    are those with at least one valid row.
s3. Each (block, head) keeps k = max(1, ceil(n x m / 1024)) of its n
    candidate tiles, m = round(1024 x density) (density in 1/1024 steps): the
    highest scores, ties broken toward the lower tile index. A block without
    valid rows keeps nothing (its rows are padding, whose attention output the
    block's zero gates discard).
s4. Valid query rows attend, with the usual softmax and 1/sqrt(D) scale, to
    the valid keys of their block's kept tiles only. Padding query rows are
    not defined by this approximation.
Density 1 keeps every candidate, which is dense attention exactly.
"""
from __future__ import annotations

import math

import numpy as np

from .h3_block import TAG_PAD, f64, softmax

TILE = 128
BLOCK = 256


def tile_means(x, valid, rows):
    """Means over valid rows of consecutive `rows`-row groups.
    x: [N, H, D]; valid: bool [N] -> (means [G, H, D], counts [G])."""
    x = f64(x)
    N = x.shape[0]
    G = (N + rows - 1) // rows
    means = np.zeros((G,) + x.shape[1:])
    counts = np.zeros(G, dtype=np.int64)
    for g in range(G):
        sl = slice(g * rows, min(N, (g + 1) * rows))
        m = valid[sl]
        counts[g] = int(m.sum())
        if counts[g]:
            means[g] = x[sl][m].mean(axis=0)
    return means, counts


def block_scores(q, k, tag):
    """Scores [n_blocks, H, n_tiles] and the candidate mask [n_tiles]."""
    valid = np.asarray(tag) != TAG_PAD
    qm, qc = tile_means(q, valid, BLOCK)
    km, kc = tile_means(k, valid, TILE)
    scores = np.einsum("bhd,jhd->bhj", qm, km)
    return scores, kc > 0, qc > 0


def keep_count(density, n_cand):
    """k = max(1, ceil(n m / 1024)), m = round(1024 density), in integers."""
    if not n_cand:
        return 0
    m = min(1024, max(1, int(round(1024.0 * density))))
    return max(1, (n_cand * m + 1023) // 1024)


def select(scores, cand, block_valid, density):
    """bool [n_blocks, H, n_tiles]: the kept tiles of every (block, head)."""
    nb, H, nt = scores.shape
    keep = np.zeros((nb, H, nt), dtype=bool)
    idx = np.nonzero(cand)[0]
    kk = keep_count(density, idx.size)
    for b in range(nb):
        if not block_valid[b]:
            continue
        for h in range(H):
            s = scores[b, h, idx]
            order = sorted(range(idx.size), key=lambda i: (-s[i], idx[i]))
            keep[b, h, idx[order[:kk]]] = True
    return keep


def sparse_attention(q, k, v, tag, keep, rows=None):
    """Attention of every valid query row (or of the given rows only)
    restricted to the valid keys of its block's kept tiles. q, k, v:
    [N, H, D]; returns [N, H, D] (rows not computed, and padding rows, 0)."""
    q, k, v = f64(q), f64(k), f64(v)
    N, H, D = q.shape
    valid = np.asarray(tag) != TAG_PAD
    want = np.ones(N, dtype=bool) if rows is None else np.isin(np.arange(N), rows)
    out = np.zeros((N, H, D))
    scale = 1.0 / math.sqrt(D)
    tile_of = np.arange(N) // TILE
    for b in range(keep.shape[0]):
        rows_b = np.arange(b * BLOCK, min(N, (b + 1) * BLOCK))
        rows = rows_b[valid[rows_b] & want[rows_b]]
        if rows.size == 0:
            continue
        for h in range(H):
            cols = np.nonzero(keep[b, h][tile_of] & valid)[0]
            s = q[rows, h] @ k[cols, h].T * scale
            out[rows, h] = softmax(s, axis=-1) @ v[cols, h]
    return out


def sparse_block_attention(q, k, v, tag, density):
    """Selection and attention together: (o [N, H, D], keep)."""
    scores, cand, bvalid = block_scores(q, k, tag)
    keep = select(scores, cand, bvalid, density)
    return sparse_attention(q, k, v, tag, keep), keep
