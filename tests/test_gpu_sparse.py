"""GPU parity of block-sparse attention (h3blk_set_attention_density) against
the fp64 oracle (oracle/h3_sparse.py). The tile selection is an integer
decision taken from fp32 pooled scores on the GPU: every kept tile must be
among the oracle's best within a small score margin (ties may go either way),
and the attention and block outputs are then compared with the GPU's own
selection."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import h3_inputs as hi
from oracle.h3_block import BlockOracle
from oracle.h3_sparse import block_scores, keep_count, sparse_attention
from tests._parity import GpuCase, assert_intermediate, assert_stage

pytestmark = pytest.mark.gpu


def _gpu_keep(case, n):
    lists = case.stage("KV_LIST").cpu().numpy()
    nb, H, _ = lists.shape
    n_tiles = (n + 127) // 128
    keep = np.zeros((nb, H, n_tiles), dtype=bool)
    for b in range(nb):
        for h in range(H):
            c = lists[b, h, 0]
            tiles = lists[b, h, 1:1 + c]
            assert np.all(np.diff(tiles) > 0), "kept tiles ascending and distinct"
            keep[b, h, tiles] = True
    return keep


def _check_selection(keep, q, k, tag, density):
    scores, cand, bvalid = block_scores(q, k, tag)
    kk = keep_count(density, int(cand.sum()))
    tol = 1e-3 * np.abs(scores).max()
    for b in range(scores.shape[0]):
        for h in range(scores.shape[1]):
            got = keep[b, h]
            if not bvalid[b]:
                continue
            assert got.sum() == kk and not np.any(got & ~cand)
            s = scores[b, h][cand]
            kth = np.sort(s)[::-1][kk - 1]
            assert np.all(scores[b, h][got] >= kth - tol)
            assert np.all(scores[b, h][cand & ~got] <= kth + tol)


def _qkv64(case, d):
    q, k, v = case.qkv()
    return q.double().numpy(), k.double().numpy(), v.double().numpy()


@pytest.mark.parametrize("density,quant", [(0.34, 0), (0.5, 0), (0.34, 1)])
def test_tiny_sparse_block(density, quant):
    dims, lay = hi.workload("tiny_320")
    inp = hi.make_inputs(replace(dims, quant=quant), lay)
    case = GpuCase(inp)
    case.block.set_attention_density(density)
    case.ws = case.block.workspace(case.n)
    case.run()
    assert case.block.check(case.ws, case.n) == 0
    lay = inp.layout
    q, k, v = _qkv64(case, inp.dims)
    keep = _gpu_keep(case, lay.n)
    _check_selection(keep, q, k, lay.tag, density)
    assert keep.sum() < keep.size          # something was dropped
    valid = lay.tag != -1
    o_ref = sparse_attention(q, k, v, lay.tag, keep)
    o_gpu = case.stage("O").float().cpu().numpy().reshape(lay.n, inp.dims.heads, inp.dims.head_dim)
    assert_intermediate("o", o_gpu[valid], o_ref[valid])
    ref = BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table, keep=keep)
    assert_stage("out", case.out, ref["out"])
    pad = torch.from_numpy(~valid).cuda()
    assert torch.equal(case.out[pad], case.x[pad])   # padding rows pass through


def test_full_keep_equals_dense_bit_for_bit():
    """A density that keeps every candidate (1023/1024) visits the same tiles
    in the same order as dense attention on a layout without padding."""
    inp = hi.make_inputs("real_8k")
    case = GpuCase(inp)
    dense = case.run().clone()
    o_dense = case.stage("O").clone()
    case.block.set_attention_density(0.999)
    case.ws = case.block.workspace(case.n)
    case.run()
    assert torch.equal(case.stage("O"), o_dense)
    assert torch.equal(case.out, dense)


def test_real_dims_sparse_sampled_rows():
    inp = hi.make_inputs("real_8k")
    case = GpuCase(inp)
    case.block.set_attention_density(0.25)
    case.ws = case.block.workspace(case.n)
    case.run()
    lay, d = inp.layout, inp.dims
    q, k, v = _qkv64(case, d)
    keep = _gpu_keep(case, lay.n)
    _check_selection(keep, q, k, lay.tag, 0.25)
    rows = hi.sample_rows(lay, k=48, k_pad=0, seed=3)
    o_ref = sparse_attention(q, k, v, lay.tag, keep, rows=rows)[rows]
    o_gpu = case.stage("O")[torch.from_numpy(rows).cuda()].float().cpu().numpy().reshape(len(rows), d.heads, d.head_dim)
    assert_intermediate("o", o_gpu, o_ref)


def test_padded_32k_sparse_sampled_rows():
    """The 32k layout with 168 padding rows at the tail: padding tiles are
    never candidates, mixed tiles are masked per key, padding rows pass the
    block through unchanged."""
    inp = hi.make_inputs("t2va_32k_pad168")
    case = GpuCase(inp)
    case.block.set_attention_density(0.3)
    case.ws = case.block.workspace(case.n)
    case.run()
    assert case.block.check(case.ws, case.n) == 0
    lay, d = inp.layout, inp.dims
    q, k, v = _qkv64(case, d)
    keep = _gpu_keep(case, lay.n)
    _check_selection(keep, q, k, lay.tag, 0.3)
    rows = hi.sample_rows(lay, k=32, k_pad=0, seed=4)
    o_ref = sparse_attention(q, k, v, lay.tag, keep, rows=rows)[rows]
    o_gpu = case.stage("O")[torch.from_numpy(rows).cuda()].float().cpu().numpy().reshape(len(rows), d.heads, d.head_dim)
    assert_intermediate("o", o_gpu, o_ref)
    pad = torch.from_numpy(lay.tag == -1).cuda()
    assert torch.equal(case.out[pad], case.x[pad])
