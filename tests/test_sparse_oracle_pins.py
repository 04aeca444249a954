"""Pins of the block-sparse attention oracle (oracle/h3_sparse.py): density 1
is dense attention, a hand-built selection, isolation from dropped tiles,
nesting of selections, and pooling over valid rows only."""
import numpy as np
import pytest

from oracle.h3_block import attention, documents
from oracle.h3_sparse import (BLOCK, TILE, block_scores, keep_count, select, sparse_attention,
                              sparse_block_attention, tile_means)


def _qkv(N=640, H=2, D=8, seed=0, pad=()):
    rng = np.random.default_rng(seed)
    q, k, v = (rng.standard_normal((N, H, D)) for _ in range(3))
    tag = np.zeros(N, dtype=np.int32)
    tag[list(pad)] = -1
    return q, k, v, tag


def test_keep_count():
    assert keep_count(0.25, 10) == 3 and keep_count(0.01, 10) == 1 and keep_count(1.0, 7) == 7
    assert keep_count(0.5, 0) == 0


def test_density_one_is_dense_attention():
    q, k, v, tag = _qkv(pad=range(600, 640))
    o, keep = sparse_block_attention(q, k, v, tag, 1.0)
    doc = documents(tag)
    ref = attention(q, k, v, doc, doc)
    valid = tag != -1
    np.testing.assert_allclose(o[valid], ref[valid], rtol=1e-12, atol=1e-12)


def test_hand_built_selection():
    """4 key tiles whose keys all equal (j, 0) in tile j, one block of queries
    all equal to (1, 0): scores rank the tiles 3 > 2 > 1 > 0; keeping half
    keeps tiles 3 and 2. With every tile equal, the lower indices win."""
    N, D = 4 * TILE, 2
    k = np.zeros((N, 1, D))
    for j in range(4):
        k[j * TILE:(j + 1) * TILE, 0, 0] = j
    q = np.zeros((N, 1, D))
    q[:, 0, 0] = 1.0
    tag = np.zeros(N, dtype=np.int32)
    scores, cand, bvalid = block_scores(q, k, tag)
    np.testing.assert_allclose(scores[0, 0], [0, 1, 2, 3])
    keep = select(scores, cand, bvalid, 0.5)
    assert keep[0, 0].tolist() == [False, False, True, True]
    flat = select(np.zeros_like(scores), cand, bvalid, 0.5)
    assert flat[0, 0].tolist() == [True, True, False, False]


def test_dropped_tiles_do_not_influence_the_output():
    q, k, v, tag = _qkv(N=768, H=1)
    o, keep = sparse_block_attention(q, k, v, tag, 0.5)
    b = 0
    dropped = [j for j in range(6) if not keep[b, 0, j]]
    kept = [j for j in range(6) if keep[b, 0, j]]
    assert dropped and kept
    rows = slice(0, BLOCK)
    k2, v2 = k.copy(), v.copy()
    j = dropped[0]
    v2[j * TILE:(j + 1) * TILE] += 5.0
    o2 = sparse_attention(q, k2, v2, tag, keep)
    np.testing.assert_array_equal(o2[rows], o[rows])
    j = kept[0]
    v2 = v.copy()
    v2[j * TILE:(j + 1) * TILE] += 5.0
    o3 = sparse_attention(q, k, v2, tag, keep)
    assert np.abs(o3[rows] - o[rows]).max() > 1e-3


def test_selections_nest_as_density_grows():
    q, k, v, tag = _qkv(N=1280, H=3, seed=2)
    scores, cand, bvalid = block_scores(q, k, tag)
    a = select(scores, cand, bvalid, 0.3)
    b = select(scores, cand, bvalid, 0.6)
    assert np.all(b[a]) and b.sum() > a.sum()


def test_pooling_ignores_padding_rows():
    q, k, v, tag = _qkv(N=512, H=1, pad=range(100, 128))
    means, counts = tile_means(k, tag != -1, TILE)
    assert counts[0] == 100
    np.testing.assert_allclose(means[0], k[:100].mean(axis=0))
    k2 = k.copy()
    k2[100:128] = 1e6          # padding keys never enter a pooled score
    s1, _, _ = block_scores(q, k, tag)
    s2, _, _ = block_scores(q, k2, tag)
    np.testing.assert_array_equal(s1, s2)


@pytest.mark.parametrize("density", [0.25, 0.5])
def test_sparse_output_is_a_convex_combination_of_kept_values(density):
    """Every output row lies within the per-channel range of the values it was
    allowed to see (softmax weights are a convex combination)."""
    q, k, v, tag = _qkv(N=768, H=2, seed=5)
    o, keep = sparse_block_attention(q, k, v, tag, density)
    tiles = np.arange(768) // TILE
    for b in range(keep.shape[0]):
        for h in range(2):
            cols = keep[b, h][tiles]
            lo, hi = v[cols, h].min(axis=0), v[cols, h].max(axis=0)
            rows = o[b * BLOCK:(b + 1) * BLOCK, h]
            assert np.all(rows >= lo - 1e-12) and np.all(rows <= hi + 1e-12)
