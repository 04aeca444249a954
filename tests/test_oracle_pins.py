"""Pins of the fp64 oracle to things other than itself: hand-worked cases,
closed forms, library routines, brute force and invariants of the block.

Sources: "MiniMaxH3Transformer3DModel" (diffusers API page: introduction,
constructor and forward parameters) and "HyperFlow H3 Flash Brings MiniMax H3
Video to One GPU" ("How it got smaller and faster").
"""
import json
import math
import os
from dataclasses import replace
from types import SimpleNamespace

import numpy as np
import pytest
import scipy.linalg
import torch

import h3_inputs as hi
from oracle import h3_block as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# Page constants
# ---------------------------------------------------------------------------

def test_real_dims_match_constructor_defaults():
    with open(os.path.join(GOLDEN, "h3_constructor_defaults.json")) as f:
        g = json.load(f)
    d = hi.REAL
    assert d.hidden == g["hidden_size"]
    assert d.heads == g["num_attention_heads"]
    assert d.head_dim == g["attention_head_dim"]
    assert d.ffn == g["ffn_dim"]
    assert d.rope_theta == g["rope_theta"]
    assert d.norm_eps == g["norm_eps"] and d.qk_norm_eps == g["qk_norm_eps"]
    assert d.heads * d.head_dim > d.hidden  # stated on the page


# ---------------------------------------------------------------------------
# Hand-worked 2-row cases (C = 4, H = 1, D = 6, one rotary pair per axis)
# ---------------------------------------------------------------------------

def _hand_case(pad_second_row):
    dims = SimpleNamespace(hidden=4, heads=1, head_dim=6, ffn=2, hd=6, n_tags=1, n_t=1,
                           rope_pairs=(1, 1, 1), rope_theta=10000.0, norm_eps=0.0,
                           qk_norm_eps=0.0, quant=0)
    wq = np.zeros((6, 4)); wq[0, 0] = 1.0          # q = [h0, 0, 0, 0, 0, 0]
    wk = wq.copy()                                  # k = q
    wv = np.zeros((6, 4)); wv[:4, :4] = np.eye(4)   # v = [h0, h1, h2, h3, 0, 0]
    wo = np.zeros((4, 6)); wo[:4, :4] = np.eye(4)   # y = o[:4]
    w13 = np.zeros((4, 4)); w13[0, 0] = 1.0; w13[2, 0] = 1.0   # gate0 = up0 = h2[0]
    w2 = np.zeros((4, 2)); w2[0, 0] = 1.0           # ffn out = [a0, 0, 0, 0]
    w = SimpleNamespace(wqkv=np.concatenate([wq, wk, wv]), q_gain=np.ones(6), k_gain=np.ones(6),
                        wo=wo, w13=w13, w2=w2)
    table = np.zeros((1, 1, 6, 4))
    table[0, 0, orc.MOD_GATE1] = 1.0
    table[0, 0, orc.MOD_GATE2] = 1.0
    x = np.array([[1.0, 1.0, 1.0, 1.0], [2.0, 0.0, 0.0, 0.0]])
    tag = np.array([0, -1 if pad_second_row else 0])
    tidx = np.array([0, 0])
    pos = np.array([[0, 0, 0], [1, 0, 0]])
    return orc.BlockOracle(dims, w).forward(x, tag, tidx, pos, table)


def test_hand_worked_two_valid_rows():
    # h1 = rmsnorm(x): row0 [1,1,1,1], row1 [2,0,0,0]. q = k = [h0,0,...]:
    # row0 [1,0..] -> qk-norm [sqrt6, 0..]; row1 [2,0..] -> [sqrt6, 0..], then
    # RoPE with t = 1 on pair 0: [sqrt6 cos1, sqrt6 sin1, 0..].
    # logits / sqrt6: self = sqrt6, cross = sqrt6 cos1, so each row keeps
    # weight p = sigmoid(sqrt6 (1 - cos1)) on itself.
    p = 1.0 / (1.0 + math.exp(math.sqrt(6.0) * (math.cos(1.0) - 1.0)))
    s6 = math.sqrt(6.0)
    r = _hand_case(False)
    np.testing.assert_allclose(r["q"][0, 0], [s6, 0, 0, 0, 0, 0], atol=1e-12)
    np.testing.assert_allclose(r["q"][1, 0], [s6 * math.cos(1), s6 * math.sin(1), 0, 0, 0, 0], atol=1e-12)
    # v0 = [1,1,1,1,0,0], v1 = [2,0,0,0,0,0]
    np.testing.assert_allclose(r["o"][0], [2 - p, p, p, p, 0, 0], atol=1e-12)
    np.testing.assert_allclose(r["o"][1], [1 + p, 1 - p, 1 - p, 1 - p, 0, 0], atol=1e-12)
    x1_0 = np.array([3 - p, 1 + p, 1 + p, 1 + p])
    x1_1 = np.array([3 + p, 1 - p, 1 - p, 1 - p])
    np.testing.assert_allclose(r["x1"], [x1_0, x1_1], atol=1e-12)
    for i, x1 in enumerate((x1_0, x1_1)):
        h20 = x1[0] / math.sqrt(np.mean(x1 ** 2))
        a0 = h20 * h20 / (1.0 + math.exp(-h20))   # silu(g) * u with g = u = h2[0]
        np.testing.assert_allclose(r["a"][i], [a0, 0.0], atol=1e-12)
        np.testing.assert_allclose(r["out"][i], x1 + np.array([a0, 0, 0, 0]), atol=1e-12)


def test_hand_worked_valid_plus_padding_row():
    # row1 is padding: its own document, zero modulation -> out = x exactly.
    # row0 attends only to itself: o = v0 = [1,1,1,1,0,0], x1 = [2,2,2,2],
    # h2 = [1,1,1,1], a0 = silu(1) * 1, out = [2 + silu(1), 2, 2, 2].
    r = _hand_case(True)
    silu1 = 1.0 / (1.0 + math.exp(-1.0))
    np.testing.assert_allclose(r["o"][0], [1, 1, 1, 1, 0, 0], atol=1e-12)
    np.testing.assert_allclose(r["out"][0], [2 + silu1, 2, 2, 2], atol=1e-12)
    assert np.array_equal(r["out"][1], [2.0, 0, 0, 0])


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def _brute_attention(q, k, v, doc):
    """Pure-Python loops: for each query and head, softmax over same-doc keys."""
    R, H, D = q.shape
    out = np.zeros_like(q)
    for i in range(R):
        for h in range(H):
            keys = [j for j in range(R) if doc[j] == doc[i]]
            logits = [sum(q[i, h, c] * k[j, h, c] for c in range(D)) / math.sqrt(D) for j in keys]
            mx = max(logits)
            ws = [math.exp(l - mx) for l in logits]
            tot = sum(ws)
            for w_, j in zip(ws, keys):
                for c in range(D):
                    out[i, h, c] += w_ / tot * v[j, h, c]
    return out


def test_attention_brute_force():
    rng = np.random.default_rng(3)
    R, H, D = 9, 2, 4
    q, k, v = (rng.standard_normal((R, H, D)) for _ in range(3))
    tag = np.array([0, 1, 2, -1, 3, 3, -1, 0, 2])
    doc = orc.documents(tag)
    np.testing.assert_allclose(orc.attention(q, k, v, doc, doc), _brute_attention(q, k, v, doc), atol=1e-12)


def test_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(4)
    R, H, D = 33, 3, 16
    q, k, v = (rng.standard_normal((R, H, D)) for _ in range(3))
    tag = np.where(np.arange(R) >= 27, -1, 0)
    doc = orc.documents(tag)
    mask = torch.from_numpy(doc[:, None] == doc[None, :])
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask)
    np.testing.assert_allclose(orc.attention(q, k, v, doc, doc), ref.permute(1, 0, 2).numpy(), atol=1e-12)


def test_attention_single_key_document_returns_v():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((5, 2, 8)) for _ in range(3))
    doc = orc.documents(np.array([0, 0, 0, 0, -1]))
    o = orc.attention(q, k, v, doc, doc)
    np.testing.assert_allclose(o[4], v[4], atol=1e-14)


def test_attention_equal_keys_average_values():
    rng = np.random.default_rng(6)
    q = rng.standard_normal((6, 2, 8))
    k = np.broadcast_to(rng.standard_normal((1, 2, 8)), (6, 2, 8)).copy()
    v = rng.standard_normal((6, 2, 8))
    doc = np.zeros(6, dtype=np.int64)
    np.testing.assert_allclose(orc.attention(q, k, v, doc, doc), np.broadcast_to(v.mean(0), v.shape), atol=1e-13)


def test_softmax_matches_scipy():
    rng = np.random.default_rng(7)
    s = rng.standard_normal((4, 50)) * 10
    import scipy.special
    np.testing.assert_allclose(orc.softmax(s), scipy.special.softmax(s, axis=-1), atol=1e-15)


# ---------------------------------------------------------------------------
# RoPE and norms
# ---------------------------------------------------------------------------

def test_rope_frequencies_match_classical_form():
    # theta^(-i/n) equals the classical 1 / theta^(2i / (2n)) of an axis with 2n channels
    for n in (8, 12, 16, 24):
        classical = 1.0 / 10000.0 ** (np.arange(0, 2 * n, 2) / (2 * n))
        np.testing.assert_allclose(orc.rope_frequencies(n, 10000.0), classical, rtol=1e-15)


def test_rope_is_complex_rotation():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((7, 3, 128))
    pos = rng.integers(0, 500, size=(7, 3))
    pairs = (16, 24, 24)
    y = orc.apply_rope(x, pos, pairs, 1e4)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    ang = orc.rope_angles(pos, pairs, 1e4, 128)[:, None, :]
    zr = z * np.exp(1j * ang)
    np.testing.assert_allclose(y[..., 0::2], zr.real, atol=1e-12)
    np.testing.assert_allclose(y[..., 1::2], zr.imag, atol=1e-12)


def test_rope_preserves_pair_norms_and_identity_at_zero():
    rng = np.random.default_rng(9)
    x = rng.standard_normal((5, 2, 64))
    pos = rng.integers(0, 100, size=(5, 3))
    y = orc.apply_rope(x, pos, (8, 12, 12), 1e4)
    np.testing.assert_allclose(np.hypot(y[..., 0::2], y[..., 1::2]), np.hypot(x[..., 0::2], x[..., 1::2]), rtol=1e-13)
    np.testing.assert_array_equal(orc.apply_rope(x, np.zeros((5, 3), int), (8, 12, 12), 1e4), x)


def test_rope_unrotated_tail_passes_through():
    # the page's own split rotates 2*3*16 = 96 of 128 channels; the rest pass through
    rng = np.random.default_rng(10)
    x = rng.standard_normal((4, 1, 128))
    y = orc.apply_rope(x, rng.integers(1, 50, size=(4, 3)), (16, 16, 16), 1e4)
    np.testing.assert_array_equal(y[..., 96:], x[..., 96:])
    assert not np.allclose(y[..., :96], x[..., :96])


def test_rope_relative_position_invariance():
    rng = np.random.default_rng(11)
    q, k = rng.standard_normal((2, 1, 1, 128))
    pairs = (16, 24, 24)
    p1, p2 = np.array([[3, 5, 7]]), np.array([[10, 2, 30]])
    base = np.sum(orc.apply_rope(q, p1, pairs, 1e4) * orc.apply_rope(k, p2, pairs, 1e4))
    for shift in ([5, 0, 0], [0, 9, 0], [0, 0, 13], [2, 3, 4]):
        s = np.array([shift])
        moved = np.sum(orc.apply_rope(q, p1 + s, pairs, 1e4) * orc.apply_rope(k, p2 + s, pairs, 1e4))
        assert abs(moved - base) < 1e-11


def test_rmsnorm_matches_torch():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((6, 40)) * 3
    ref = torch.nn.functional.rms_norm(torch.from_numpy(x), (40,), eps=1e-5).numpy()
    np.testing.assert_allclose(orc.rmsnorm(x, 1e-5), ref, rtol=1e-14)


def test_qk_norm_scale_invariance_and_unit_rms():
    rng = np.random.default_rng(13)
    xh = rng.standard_normal((3, 4, 64))
    g = np.ones(64)
    y = orc.qk_rmsnorm(xh, g, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(orc.qk_rmsnorm(7.5 * xh, g, 0.0), y, rtol=1e-13)
    g2 = rng.standard_normal(64)
    np.testing.assert_allclose(orc.qk_rmsnorm(xh, g2, 0.0), y * g2, rtol=1e-13)


def test_adaln_special_cases():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((3, 16))
    shift = rng.standard_normal((3, 16))
    np.testing.assert_allclose(orc.adaln(x, shift, -np.ones((3, 16)), 1e-5), shift, atol=0)
    np.testing.assert_allclose(orc.adaln(x, 0 * shift, 0 * shift, 1e-5), orc.rmsnorm(x, 1e-5), atol=0)


def test_silu_matches_torch():
    g = np.linspace(-20, 20, 101)
    np.testing.assert_allclose(orc.silu(g), torch.nn.functional.silu(torch.from_numpy(g)).numpy(), rtol=1e-14, atol=1e-300)


def test_modulation_gather_and_padding():
    table = np.arange(2 * 3 * 6 * 4, dtype=np.float64).reshape(2, 3, 6, 4)
    m = orc.modulation(table, np.array([1, -1, 0]), np.array([2, 1, 0]))
    np.testing.assert_array_equal(m[0], table[1, 2])
    np.testing.assert_array_equal(m[1], 0)
    np.testing.assert_array_equal(m[2], table[0, 0])


# ---------------------------------------------------------------------------
# Rotated W8A8
# ---------------------------------------------------------------------------

def test_hadamard_matches_scipy_and_is_orthogonal():
    h = orc.sylvester_hadamard(128)
    np.testing.assert_array_equal(h, scipy.linalg.hadamard(128))
    np.testing.assert_array_equal(h @ h.T, 128 * np.eye(128, dtype=np.int64))


def test_rotation_preserves_norm_and_is_an_involution():
    rng = np.random.default_rng(15)
    a = rng.standard_normal((5, 384))
    r = orc.rotate_blocks(a)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1), np.linalg.norm(a, axis=1), rtol=1e-13)
    np.testing.assert_allclose(orc.rotate_blocks(r), a, atol=1e-13)
    # rotating both operands leaves the product unchanged
    w = rng.standard_normal((7, 384))
    np.testing.assert_allclose(r @ orc.rotate_blocks(w).T, a @ w.T, atol=1e-11)


def test_quantize_rows_hand_values():
    v = np.array([[127.0, -63.5, 0.5, 1.5, -127.0, 2.5],
                  [0.0, 0.0, 0.0, 0.0, 0.0, 0.0],
                  [-2.0, 1.0, 0.0, 0.0, 0.0, 0.0]])
    q, s = orc.quantize_rows(v)
    # row 0: s = 1, round half to even: -63.5 -> -64, 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    np.testing.assert_array_equal(q[0], [127, -64, 0, 2, -127, 2])
    assert s[0] == 1.0
    np.testing.assert_array_equal(q[1], 0)
    assert s[1] == 0.0
    # row 2: s = 2/127; -2 -> -127, 1 -> 63.5 -> 64 (half to even), zeros stay 0
    np.testing.assert_array_equal(q[2], [-127, 64, 0, 0, 0, 0])
    assert q.dtype == np.int8


def test_int8_matmul_exact_against_python_ints():
    rng = np.random.default_rng(16)
    a = rng.integers(-127, 128, size=(5, 37)).astype(np.int8)
    w = rng.integers(-127, 128, size=(4, 37)).astype(np.int8)
    acc = orc.int8_matmul_exact(a, w)
    for i in range(5):
        for j in range(4):
            assert acc[i, j] == sum(int(a[i, t]) * int(w[j, t]) for t in range(37))


def test_int8_accumulator_extreme_fits_int32():
    K = 14336
    a = np.full((1, K), 127, dtype=np.int8)
    acc = orc.int8_matmul_exact(a, a)
    assert acc[0, 0] == 231225344 and acc[0, 0] < 2 ** 31 - 1


def test_w8a8_linear_close_to_float_linear():
    rng = np.random.default_rng(17)
    a = rng.standard_normal((16, 512))
    w = rng.standard_normal((64, 512)) / np.sqrt(512)
    wq, sw = orc.prepare_int8_weight(w)
    y = orc.w8a8_linear(a, wq, sw)
    ref = a @ w.T
    rel = np.sqrt(np.mean((y - ref) ** 2) / np.mean(ref ** 2))
    assert rel < 2e-2
    # without rounding the rotated product reproduces the float product exactly
    np.testing.assert_allclose(orc.rotate_blocks(a) @ orc.rotate_blocks(w).T, ref, atol=1e-11)


# ---------------------------------------------------------------------------
# Whole-block invariants (tiny dims)
# ---------------------------------------------------------------------------

@pytest.fixture(scope="module")
def tiny():
    inp = hi.make_inputs("tiny_320")
    return inp, orc.BlockOracle(inp.dims, inp.weights)


def _fwd(ob, inp, x=None, tag=None, tidx=None, pos=None, table=None, rows=None):
    lay = inp.layout
    return ob.forward(inp.x if x is None else x, lay.tag if tag is None else tag,
                      lay.tidx if tidx is None else tidx, lay.pos if pos is None else pos,
                      inp.table if table is None else table, rows=rows)


def test_zero_gate_is_identity(tiny):
    inp, ob = tiny
    table = inp.table.clone()
    table[:, :, orc.MOD_GATE1] = 0
    table[:, :, orc.MOD_GATE2] = 0
    r = _fwd(ob, inp, table=table)
    np.testing.assert_array_equal(r["out"], orc.f64(inp.x))


def test_padding_rows_pass_through_and_never_influence(tiny):
    inp, ob = tiny
    r = _fwd(ob, inp)
    pad = inp.layout.tag == -1
    np.testing.assert_array_equal(r["out"][pad], orc.f64(inp.x)[pad])
    x2 = inp.x.clone()
    x2[torch.from_numpy(pad)] = torch.randn(int(pad.sum()), inp.dims.hidden).to(torch.bfloat16) * 5
    r2 = _fwd(ob, inp, x=x2)
    np.testing.assert_array_equal(r2["out"][~pad], r["out"][~pad])


def test_padded_and_padless_layouts_agree(tiny):
    inp, ob = tiny
    valid = inp.layout.tag != -1
    r = _fwd(ob, inp)
    lay = inp.layout
    r2 = ob.forward(inp.x[torch.from_numpy(valid)], lay.tag[valid], lay.tidx[valid], lay.pos[valid], inp.table)
    np.testing.assert_allclose(r2["out"], r["out"][valid], atol=1e-12)


def test_row_permutation_equivariance(tiny):
    inp, ob = tiny
    lay = inp.layout
    perm = np.random.default_rng(18).permutation(lay.n)
    r = _fwd(ob, inp)
    r2 = ob.forward(inp.x[torch.from_numpy(perm)], lay.tag[perm], lay.tidx[perm], lay.pos[perm], inp.table)
    np.testing.assert_allclose(r2["out"], r["out"][perm], atol=1e-12)


def test_global_position_shift_invariance(tiny):
    inp, ob = tiny
    r = _fwd(ob, inp)
    r2 = _fwd(ob, inp, pos=inp.layout.pos + np.array([[7, 3, 11]], dtype=np.int32))
    np.testing.assert_allclose(r2["out"], r["out"], atol=1e-10)


def test_subset_mode_equals_full(tiny):
    inp, ob = tiny
    rows = hi.sample_rows(inp.layout, k=40, k_pad=4)
    r = _fwd(ob, inp)
    rs = _fwd(ob, inp, rows=rows)
    for key in ("h1", "q", "k", "v", "o", "x1", "h2", "a", "out"):
        np.testing.assert_allclose(rs[key], r[key][rows], atol=1e-12, err_msg=key)


def test_w8a8_block_close_to_bf16_block(tiny):
    inp, ob = tiny
    obq = orc.BlockOracle(replace(inp.dims, quant=1), inp.weights)
    r = _fwd(ob, inp)
    rq = _fwd(obq, inp)
    d = rq["out"] - r["out"]
    ref = r["out"] - orc.f64(inp.x)
    assert np.sqrt(np.mean(d ** 2) / np.mean(ref ** 2)) < 0.05


def test_oracle_snapshot_unchanged(tiny):
    """Regression pin: the tiny workload's oracle outputs on a few rows, as
    written by tests/golden/make_oracle_snapshot.py (which calls only the
    oracle). A change here must come with a reason from the pages."""
    inp, ob = tiny
    snap = np.load(os.path.join(GOLDEN, "tiny_320_oracle_snapshot.npz"))
    rows = snap["rows"]
    r = _fwd(ob, inp, rows=rows)
    for key in ("h1", "q", "o", "x1", "a", "out"):
        np.testing.assert_allclose(r[key], snap[key], rtol=1e-12, atol=1e-12, err_msg=key)


def test_gate1_gates_attention_and_gate2_gates_ffn(tiny):
    # reading of the modulation order: [shift1, scale1, gate1, shift2, scale2, gate2]
    inp, ob = tiny
    x = orc.f64(inp.x)
    t1 = inp.table.clone()
    t1[:, :, orc.MOD_GATE1] = 0
    r1 = _fwd(ob, inp, table=t1)
    np.testing.assert_array_equal(r1["x1"], x)          # no attention branch
    assert not np.allclose(r1["out"], x)                 # ffn branch still there
    t2 = inp.table.clone()
    t2[:, :, orc.MOD_GATE2] = 0
    r2 = _fwd(ob, inp, table=t2)
    np.testing.assert_array_equal(r2["out"], r2["x1"])  # no ffn branch
    assert not np.allclose(r2["x1"], x)
    # shift2/scale2 act only on the ffn input
    t3 = inp.table.clone()
    t3[:, :, orc.MOD_SHIFT2] += 1.0
    r3 = _fwd(ob, inp, table=t3)
    np.testing.assert_array_equal(r3["x1"], _fwd(ob, inp)["x1"])
    assert not np.allclose(r3["out"], _fwd(ob, inp)["out"])


# ---------------------------------------------------------------------------
# Readings pinned by hand values: which coordinate drives which rotary pair
# block, and which half of the SwiGLU weight goes through silu. Each pin is a
# function so that the planted-mistake tests below can show that it catches a
# swapped copy of the oracle.
# ---------------------------------------------------------------------------

def _rope_axis_pin():
    # rope_pairs (1, 2, 1), head_dim 8: pair 0 follows t, pairs 1-2 follow h,
    # pair 3 follows w. Frequencies: t [1], h [1, 1e4^(-1/2) = 0.01], w [1].
    # Input pairs (1,2) (3,4) (5,6) (7,8); a pair (a, b) turned by phi becomes
    # (a cos phi - b sin phi, a sin phi + b cos phi).
    x = np.arange(1.0, 9.0).reshape(1, 1, 8)
    c, s = math.cos, math.sin
    cases = {
        (0, 1, 0): [1, 2, 3 * c(1) - 4 * s(1), 3 * s(1) + 4 * c(1),
                    5 * c(0.01) - 6 * s(0.01), 5 * s(0.01) + 6 * c(0.01), 7, 8],
        (0, 3, 0): [1, 2, 3 * c(3) - 4 * s(3), 3 * s(3) + 4 * c(3),
                    5 * c(0.03) - 6 * s(0.03), 5 * s(0.03) + 6 * c(0.03), 7, 8],
        (0, 0, 1): [1, 2, 3, 4, 5, 6, 7 * c(1) - 8 * s(1), 7 * s(1) + 8 * c(1)],
        (1, 0, 0): [1 * c(1) - 2 * s(1), 1 * s(1) + 2 * c(1), 3, 4, 5, 6, 7, 8],
        (2, 0, 5): [1 * c(2) - 2 * s(2), 1 * s(2) + 2 * c(2), 3, 4, 5, 6,
                    7 * c(5) - 8 * s(5), 7 * s(5) + 8 * c(5)],
    }
    for p, want in cases.items():
        got = orc.apply_rope(x, np.array([p]), (1, 2, 1), 1e4)
        np.testing.assert_allclose(got[0, 0], want, atol=1e-12, err_msg=f"position {p}")


def test_rope_axis_to_pair_block_mapping_hand_values():
    _rope_axis_pin()


def _swiglu_half_pin():
    # C = 4, F = 1, H = 1, D = 6. gate1 = 0 so x1 = x; gate2 = 1. x = [1, 2, 0, 0]
    # with eps 0 gives h2 = x / sqrt(5/4) = [2/sqrt5, 4/sqrt5, 0, 0].
    # w13 row 0 (the W1 half, through silu) reads h2[0]; row 1 (the W3 half,
    # the linear "up" branch) reads h2[1]: a = silu(2/sqrt5) * 4/sqrt5.
    dims = SimpleNamespace(hidden=4, heads=1, head_dim=6, ffn=1, hd=6, n_tags=1, n_t=1,
                           rope_pairs=(1, 1, 1), rope_theta=10000.0, norm_eps=0.0,
                           qk_norm_eps=1e-6, quant=0)   # q = k = 0 here; eps keeps their norm finite
    w13 = np.zeros((2, 4)); w13[0, 0] = 1.0; w13[1, 1] = 1.0
    w2 = np.zeros((4, 1)); w2[0, 0] = 1.0
    w = SimpleNamespace(wqkv=np.zeros((18, 4)), q_gain=np.ones(6), k_gain=np.ones(6),
                        wo=np.zeros((4, 6)), w13=w13, w2=w2)
    table = np.zeros((1, 1, 6, 4))
    table[0, 0, orc.MOD_GATE2] = 1.0
    x = np.array([[1.0, 2.0, 0.0, 0.0]])
    r = orc.BlockOracle(dims, w).forward(x, np.array([0]), np.array([0]), np.array([[0, 0, 0]]), table)
    g, u = 2 / math.sqrt(5), 4 / math.sqrt(5)
    a = g / (1 + math.exp(-g)) * u          # 1.1357...; the swapped reading gives 1.3709...
    np.testing.assert_allclose(r["a"][0], [a], atol=1e-12)
    np.testing.assert_allclose(r["out"][0], [1 + a, 2, 0, 0], atol=1e-12)


def test_swiglu_w1_half_goes_through_silu_hand_values():
    _swiglu_half_pin()


def test_swiglu_hand_value_with_distinct_gate_and_up():
    # silu(2) * 3 = 3 * 2 / (1 + e^-2); silu(3) * 2 would be 5.7155...
    np.testing.assert_allclose(orc.swiglu(np.array([2.0]), np.array([3.0])), [6 / (1 + math.exp(-2))], rtol=1e-15)


# Planted mistakes (in the oracle, on the CPU): each pin above must fail on a
# plausibly wrong copy of the function it guards.

def _rope_angles_axes_swapped(pos, rope_pairs, theta, head_dim):
    pos = np.asarray(pos, dtype=np.float64)[:, [0, 2, 1]]       # h and w exchanged
    return _ORIG_ROPE_ANGLES(pos, rope_pairs, theta, head_dim)


def _rope_angles_axes_reversed(pos, rope_pairs, theta, head_dim):
    pos = np.asarray(pos, dtype=np.float64)[:, ::-1]             # pos[:, 2 - axis]
    return _ORIG_ROPE_ANGLES(pos, rope_pairs, theta, head_dim)


def _rope_angles_doubled_exponent(pos, rope_pairs, theta, head_dim):
    pos = np.asarray(pos, dtype=np.float64)
    ang = np.zeros((pos.shape[0], head_dim // 2))
    j = 0
    for axis, n in enumerate(rope_pairs):
        ang[:, j:j + n] = pos[:, axis:axis + 1] * theta ** (-2.0 * np.arange(n) / n)
        j += n
    return ang


_ORIG_ROPE_ANGLES = orc.rope_angles


@pytest.mark.parametrize("mutant", [_rope_angles_axes_swapped, _rope_angles_axes_reversed,
                                    _rope_angles_doubled_exponent])
def test_rope_axis_pin_catches_planted_mistakes(monkeypatch, mutant):
    monkeypatch.setattr(orc, "rope_angles", mutant)
    with pytest.raises(AssertionError):
        _rope_axis_pin()


def test_rope_axis_pin_catches_a_flipped_rotation_sign(monkeypatch):
    orig = orc.rope_angles
    monkeypatch.setattr(orc, "rope_angles", lambda *a: -orig(*a))
    with pytest.raises(AssertionError):
        _rope_axis_pin()


def test_swiglu_pin_catches_swapped_halves(monkeypatch):
    monkeypatch.setattr(orc, "swiglu", lambda g, u: orc.silu(u) * g)
    with pytest.raises(AssertionError):
        _swiglu_half_pin()


# ---------------------------------------------------------------------------
# Faithful (bf16-store) diagnostic mode and the exact int8 product
# ---------------------------------------------------------------------------

def test_bf16_round_hand_values():
    # bf16 keeps 8 significant bits: the spacing just above 1 is 2^-7
    cases = [(1 + 2 ** -8, 1.0),                          # tie -> even (1.0)
             (1 + 3 * 2 ** -8, 1 + 2 ** -6),              # tie -> even (mantissa 2)
             (1 + 2 ** -8 + 2 ** -20, 1 + 2 ** -7),       # just above the tie
             (-3.0, -3.0), (0.0, 0.0), (2 ** -130, 2 ** -130),
             (65280.0 + 127.0, 65280.0), (255.0, 255.0), (257.0, 256.0), (259.0, 260.0)]
    for v, want in cases:
        assert orc.bf16_round(np.array([v]))[0] == want, v


def test_faithful_mode_rounds_exactly_the_stored_stages(tiny):
    inp, _ = tiny
    lay = inp.layout
    exact = orc.BlockOracle(inp.dims, inp.weights)
    faith = orc.BlockOracle(inp.dims, inp.weights, faithful=True)
    re_ = _fwd(exact, inp)
    rf = _fwd(faith, inp)
    for key in ("h1", "q", "k", "v", "o", "x1", "h2", "a", "out"):
        np.testing.assert_array_equal(orc.bf16_round(rf[key]), rf[key], err_msg=key)
    # the roundings move the output by a few bf16 ulps at most, never more
    d = np.abs(rf["out"] - re_["out"])
    assert d.max() < 4 * 2.0 ** -7 * max(1.0, np.abs(re_["out"]).max())
    assert d.max() > 0
    # zero gates: the identity survives the roundings (x is bf16 already)
    table = inp.table.clone()
    table[:, :, orc.MOD_GATE1] = 0
    table[:, :, orc.MOD_GATE2] = 0
    r0 = faith.forward(inp.x, lay.tag, lay.tidx, lay.pos, table)
    np.testing.assert_array_equal(r0["out"], orc.f64(inp.x))


def test_faithful_w8a8_leaves_the_quantised_inputs_unrounded(tiny):
    inp, _ = tiny
    faith = orc.BlockOracle(replace(inp.dims, quant=1), inp.weights, faithful=True)
    r = _fwd(faith, inp, rows=np.arange(8))
    # h1 feeds the rotation + quantisation straight from fp32 on this path
    assert not np.array_equal(orc.bf16_round(r["h1"]), r["h1"])
    np.testing.assert_array_equal(orc.bf16_round(r["o"]), r["o"])


def test_int8_product_exact_at_extremes_and_random():
    rng = np.random.default_rng(40)
    a = rng.integers(-127, 128, size=(5, 14336)).astype(np.int8)
    w = rng.integers(-127, 128, size=(3, 14336)).astype(np.int8)
    got = orc.int8_matmul_exact(a, w)
    for i in range(5):
        for j in range(3):
            assert got[i, j] == sum(int(p) * int(q) for p, q in zip(a[i].tolist(), w[j].tolist()))
    full = np.full((1, 14336), 127, np.int8)
    assert orc.int8_matmul_exact(full, full)[0, 0] == 127 * 127 * 14336
    assert orc.int8_matmul_exact(full, -full)[0, 0] == -127 * 127 * 14336


def test_qkv_parts_equal_the_full_projection(tiny):
    inp, ob = tiny
    lay = inp.layout
    rng = np.random.default_rng(41)
    h = rng.standard_normal((6, inp.dims.hidden))
    pos = lay.pos[:6]
    full = ob.qkv(h, pos)
    kv = ob.qkv(h, pos, part=("k", "v"))
    q = ob.qkv(h, pos, part=("q",))
    np.testing.assert_array_equal(kv["k"], full["k"])
    np.testing.assert_array_equal(kv["v"], full["v"])
    np.testing.assert_array_equal(q["q"], full["q"])
    obq = orc.BlockOracle(replace(inp.dims, quant=1), inp.weights)
    fq = obq.qkv(h, pos)
    np.testing.assert_array_equal(obq.qkv(h, pos, part=("k", "v"))["v"], fq["v"])
