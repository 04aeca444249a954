"""Pins of the model-shell oracle (oracle/h3_model.py) against closed forms,
library routines and invariants of the model ("MiniMaxH3Transformer3DModel",
diffusers API page: introduction, constructor and forward parameters)."""
from dataclasses import replace

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import h3_inputs as hi
from oracle.h3_model import ModelOracle, affine, scatter_rows


def _tiny(seed=0, two_time=False, n_layers=2, n_refiner=1):
    d, lay = hi.workload("tiny_320", seed)
    if two_time:
        d = replace(d, n_t=4)
        lay = hi.layout_two_time(lay, seed)
    sd = replace(hi.TINY_SHELL, n_layers=n_layers, n_refiner=n_refiner)
    p = hi.make_model_params(d, hi.TINY_MOD, sd, seed, two_time)
    mi = hi.make_model_inputs(d, sd, lay, seed, two_time)
    return d, p, mi


def _zero_gates(layer):
    """Copy of a layer whose AdaLN projection gives gate1 = gate2 = 0."""
    C = layer.w.wo.shape[0]
    aw, ab = layer.adaln_w.clone(), layer.adaln_b.clone()
    for g in (2, 5):
        aw[:, g * C:(g + 1) * C] = 0
        ab[:, g * C:(g + 1) * C] = 0
    return replace(layer, adaln_w=aw, adaln_b=ab)


def test_affine_is_torch_linear():
    rng = np.random.default_rng(1)
    x, w, b = rng.standard_normal((5, 7)), rng.standard_normal((3, 7)), rng.standard_normal(3)
    ref = F.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(affine(x, w, b), ref, rtol=1e-14, atol=1e-14)


def test_scatter_rows_hand_values():
    x = scatter_rows(5, 2, [(np.array([3, 0]), np.array([[1.0, 2.0], [3.0, 4.0]])),
                            (np.array([4]), np.array([[5.0, 6.0]]))])
    np.testing.assert_array_equal(x, [[3, 4], [0, 0], [0, 0], [1, 2], [5, 6]])


def test_hand_worked_two_channel_model():
    """C = 2, one video row, no text, no audio, no layers. proj_in W = [1, 2]^T,
    b = [0, 1]: x = [3, 7]. norm_out: shift = [0.5, -0.5], scale = [1, 0] (the
    time MLP and projection weights are zero, so the table is the bias).
    proj_out W = [1, -1], b = 0.25:
    y = 2*3/r + 0.5 - (7/r - 0.5) + 0.25 with r = sqrt(29 + eps)."""
    eps = 1e-5
    z = lambda *s: torch.zeros(*s)  # noqa: E731
    md = hi.ModDims(freq_dim=4, time_hidden=2, time_dim=2)
    time = hi.ModParams(md, z(2, 4), z(2), z(2, 2), z(2), None, None, None, None,
                        z(1, 12, 2).bfloat16(), z(1, 12))
    sd = hi.ShellDims(video_in=1, audio_in=1, text_dim=2, n_layers=0, n_refiner=0, final_norm_eps=eps)
    p = hi.ModelParams(sd, time, [], [], refiner_gain=torch.ones(2).bfloat16(),
                       out_adaln_w=z(1, 4, 2).bfloat16(),
                       out_adaln_b=torch.tensor([[0.5, -0.5, 1.0, 0.0]]),
                       proj_in_w=torch.tensor([[1.0], [2.0]]), proj_in_b=torch.tensor([0.0, 1.0]),
                       audio_in_w=z(2, 1), audio_in_b=z(2), ctx_w=z(2, 2).bfloat16(), ctx_b=z(2),
                       proj_out_w=torch.tensor([[1.0, -1.0]]), proj_out_b=torch.tensor([0.25]),
                       audio_out_w=z(1, 2), audio_out_b=z(1))
    lay = hi.Layout("hand", np.array([0], np.int32), np.array([0], np.int32), np.zeros((1, 3), np.int32))
    d = replace(hi.TINY, hidden=2, n_tags=1, n_t=1)
    mi = hi.ModelInputs(lay, np.array([0], np.int32), np.zeros(0, np.int32), np.zeros(0, np.int32),
                        torch.tensor([[3.0]]), z(0, 1), z(0, 2).bfloat16(),
                        np.array([0.3], np.float32), np.array([0.3], np.float32), 0.0)
    out = ModelOracle(d, p).forward(mi)
    r = np.sqrt(29.0 + eps)
    np.testing.assert_allclose(out["x0"], [[3.0, 7.0]], rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["video"], [[6 / r + 0.5 - (7 / r - 0.5) + 0.25]], rtol=1e-14)
    assert out["audio"].shape == (0, 1)


def test_shell_only_reduces_to_rms_norm_and_linear():
    """No layers, zero norm_out projection: each video output row is
    linear(rms_norm(proj_in(v))) of its own input row, via torch routines."""
    d, p, mi = _tiny(n_layers=0)
    p = replace(p, out_adaln_w=torch.zeros_like(p.out_adaln_w), out_adaln_b=torch.zeros_like(p.out_adaln_b))
    out = ModelOracle(d, p).forward(mi)
    t64 = lambda a: a.to(torch.float64)  # noqa: E731
    x = F.linear(t64(mi.video), t64(p.proj_in_w), t64(p.proj_in_b))
    h = F.rms_norm(x, (d.hidden,), eps=p.sd.final_norm_eps)
    ref = F.linear(h, t64(p.proj_out_w), t64(p.proj_out_b)).numpy()
    np.testing.assert_allclose(out["video"], ref, rtol=1e-11, atol=1e-12)


def test_refiner_with_zero_gates_is_the_output_norm():
    """Refiner layers whose gates are zero pass the text rows through, so the
    packed text rows are rms_norm(ctx(text)) * gain."""
    d, p, mi = _tiny(n_layers=0, n_refiner=2)
    p = replace(p, refiner=[_zero_gates(L) for L in p.refiner])
    out = ModelOracle(d, p).forward(mi)
    t64 = lambda a: a.to(torch.float64)  # noqa: E731
    r = F.linear(t64(mi.text), t64(p.ctx_w), t64(p.ctx_b))
    ref = F.rms_norm(r, (d.hidden,), weight=t64(p.refiner_gain), eps=p.sd.final_norm_eps).numpy()
    np.testing.assert_allclose(out["x0"][mi.text_idx], ref, rtol=1e-11, atol=1e-12)


def test_stack_with_zero_gates_is_identity():
    d, p, mi = _tiny(n_layers=2)
    shell = ModelOracle(d, replace(p, layers=[])).forward(mi)
    gated = ModelOracle(d, replace(p, layers=[_zero_gates(L) for L in p.layers])).forward(mi)
    np.testing.assert_allclose(gated["x"], shell["x0"], rtol=0, atol=0)
    np.testing.assert_allclose(gated["video"], shell["video"], rtol=0, atol=0)
    full = ModelOracle(d, p).forward(mi)
    assert np.abs(full["video"] - shell["video"]).max() > 1e-3   # the layers do act


def test_padding_rows_start_at_zero_and_stay_unaddressed():
    d, p, mi = _tiny()
    out = ModelOracle(d, p).forward(mi)
    pad = mi.layout.tag == hi.TAG_PAD
    assert pad.any()
    np.testing.assert_array_equal(out["x0"][pad], 0.0)
    np.testing.assert_array_equal(out["x"][pad], 0.0)   # zero modulation: padding rows pass through


def test_refiner_sees_only_text_rows():
    """With no stack layers, the text rows of x0 do not depend on the video or
    audio inputs, and the video outputs do not depend on the text."""
    d, p, mi = _tiny(n_layers=0)
    a = ModelOracle(d, p).forward(mi)
    mi2 = replace(mi, video=mi.video * 2 + 1, audio=-mi.audio)
    b = ModelOracle(d, p).forward(mi2)
    np.testing.assert_array_equal(a["x0"][mi.text_idx], b["x0"][mi.text_idx])
    mi3 = replace(mi, text=(mi.text.float() * -1.5).bfloat16())
    c = ModelOracle(d, p).forward(mi3)
    np.testing.assert_array_equal(a["video"], c["video"])
    assert np.abs(a["x0"][mi.text_idx] - c["x0"][mi.text_idx]).max() > 1e-3


def test_row_permutation_equivariance():
    """Reordering the packed sequence (tags, timestep indices and positions
    move with their rows, the index tensors are remapped) leaves both heads'
    outputs unchanged: the stack only sees rows through their tags and
    positions."""
    d, p, mi = _tiny(two_time=True)
    lay = mi.layout
    perm = np.random.default_rng(5).permutation(lay.n)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(lay.n)
    lay2 = hi.Layout(lay.name, lay.tag[perm], lay.tidx[perm], lay.pos[perm])
    mi2 = replace(mi, layout=lay2, video_idx=inv[mi.video_idx].astype(np.int32),
                  audio_idx=inv[mi.audio_idx].astype(np.int32), text_idx=inv[mi.text_idx].astype(np.int32))
    a = ModelOracle(d, p).forward(mi)
    b = ModelOracle(d, p).forward(mi2)
    np.testing.assert_allclose(b["video"], a["video"], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(b["audio"], a["audio"], rtol=1e-10, atol=1e-10)


def test_head_rows_follow_index_order():
    """Swapping two audio rows together with their index entries swaps the
    two audio outputs."""
    d, p, mi = _tiny()
    a = ModelOracle(d, p).forward(mi)
    ai = mi.audio_idx.copy()
    ai[[0, 5]] = ai[[5, 0]]
    au = mi.audio.clone()
    au[[0, 5]] = au[[5, 0]]
    b = ModelOracle(d, p).forward(replace(mi, audio_idx=ai, audio=au))
    sw = a["audio"].copy()
    sw[[0, 5]] = sw[[5, 0]]
    np.testing.assert_allclose(b["audio"], sw, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("two_time", [False, True])
def test_layer_tables_use_each_layers_projection(two_time):
    """Layer k's table is affine in its own projection: doubling layer 1's
    projection weights and bias doubles its table and leaves layer 0's."""
    d, p, mi = _tiny(two_time=two_time)
    o = ModelOracle(d, p)
    t1 = o.tables(mi.t_now, mi.t_end, mi.gate)
    L1 = p.layers[1]
    p2 = replace(p, layers=[p.layers[0], replace(L1, adaln_w=(L1.adaln_w.float() * 2).bfloat16(),
                                                     adaln_b=L1.adaln_b * 2)])
    t2 = ModelOracle(d, p2).tables(mi.t_now, mi.t_end, mi.gate)
    np.testing.assert_array_equal(t2["layers"][0], t1["layers"][0])
    np.testing.assert_allclose(t2["layers"][1], 2 * t1["layers"][1], rtol=1e-14, atol=1e-15)
    assert t1["layers"][0].shape == (d.n_tags, d.n_t, 6, d.hidden)
    assert t1["out"].shape == (d.n_tags, d.n_t, 2, d.hidden)


def test_subset_rows_match_the_full_forward():
    d, p, mi = _tiny(n_layers=2)
    full = ModelOracle(d, p).forward(mi)
    rows = hi.sample_rows(mi.layout, k=40, k_pad=4, seed=3)
    sub = ModelOracle(d, p).forward(mi, rows=rows)
    np.testing.assert_allclose(sub["video"], full["video"][sub["video_sel"]], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(sub["audio"], full["audio"][sub["audio_sel"]], rtol=1e-12, atol=1e-12)
    assert sub["video_sel"].size > 10
