"""Pins of the modulation-table producer oracle (oracle/h3_modulation.py):
closed forms of the sinusoidal embedding, a hand-worked time MLP, the
two-time blend's end points and linearity, and per-tag selection."""
import math

import numpy as np
import pytest

import h3_inputs as hi
from oracle import h3_modulation as om
from oracle.h3_block import silu


def test_embedding_at_zero_and_unit_pairs():
    e = om.sinusoidal_embedding([0.0], 256)
    np.testing.assert_array_equal(e[0, :128], 1.0)
    np.testing.assert_array_equal(e[0, 128:], 0.0)
    t = np.array([0.0, 0.25, 0.5, 1.0])
    e = om.sinusoidal_embedding(t, 256)
    np.testing.assert_allclose(e[:, :128] ** 2 + e[:, 128:] ** 2, 1.0, rtol=1e-14)
    # the first frequency is 1: channel 0 is cos(t), channel 128 is sin(t)
    np.testing.assert_allclose(e[:, 0], np.cos(t), rtol=1e-15)
    np.testing.assert_allclose(e[:, 128], np.sin(t), rtol=1e-15)


def test_frequencies_closed_form():
    w = om.timestep_frequencies(256)
    np.testing.assert_allclose(w, np.exp(-math.log(10000.0) * np.arange(128) / 128), rtol=1e-13)
    assert w[0] == 1.0


def test_hand_worked_time_mlp():
    # freq_dim 2: e(t) = [cos t, sin t]; W1 = I, b1 = 0, W2 = [[1, 1]], b2 = 0.5
    # E(t) = silu(cos t) + silu(sin t) + 0.5
    w1, b1 = np.eye(2), np.zeros(2)
    w2, b2 = np.array([[1.0, 1.0]]), np.array([0.5])
    for t in (0.0, 0.3, 1.0):
        e = om.sinusoidal_embedding([t], 2)
        got = om.time_mlp(e, w1, b1, w2, b2)[0, 0]
        c, s = math.cos(t), math.sin(t)
        want = c / (1 + math.exp(-c)) + s / (1 + math.exp(-s)) + 0.5
        assert abs(got - want) < 1e-14


def test_two_time_blend_end_points_and_linearity():
    rng = np.random.default_rng(1)
    mlp = (rng.standard_normal((8, 16)), rng.standard_normal(8), rng.standard_normal((4, 8)), rng.standard_normal(4))
    mlp_r = (rng.standard_normal((8, 16)), rng.standard_normal(8), rng.standard_normal((4, 8)), rng.standard_normal(4))
    t, r = np.array([0.7]), np.array([0.2])
    e0 = om.two_time_embedding(t, r, 0.0, mlp, mlp_r, 16)
    e1 = om.two_time_embedding(t, r, 1.0, mlp, mlp_r, 16)
    np.testing.assert_allclose(e0, om.time_mlp(om.sinusoidal_embedding(t, 16), *mlp), rtol=1e-14)
    np.testing.assert_allclose(e1, om.time_mlp(om.sinusoidal_embedding(r, 16), *mlp_r), rtol=1e-14)
    eg = om.two_time_embedding(t, r, 0.25, mlp, mlp_r, 16)
    np.testing.assert_allclose(eg, 0.75 * e0 + 0.25 * e1, rtol=1e-13)


def test_modulation_table_per_tag_selection():
    rng = np.random.default_rng(2)
    E = rng.standard_normal((3, 5))
    A = rng.standard_normal((2, 12, 5))
    b = rng.standard_normal((2, 12))
    tab = om.modulation_table(E, A, b)
    for tag in range(2):
        np.testing.assert_allclose(tab[tag], silu(E) @ A[tag].T + b[tag], rtol=1e-13)
    # swapping the tags' weights swaps their tables
    tab2 = om.modulation_table(E, A[::-1], b[::-1])
    np.testing.assert_allclose(tab2[0], tab[1], rtol=1e-14)
    # zero projection leaves the bias
    np.testing.assert_array_equal(om.modulation_table(E, 0 * A, b), np.broadcast_to(b[:, None, :], tab.shape))


def test_produce_layout_is_six_blocks_of_hidden():
    dims, md = hi.TINY, hi.TINY_MOD
    p = hi.make_modulation_params(dims, md)
    params = {"freq_dim": md.freq_dim, "mlp": (p.w1, p.b1, p.w2, p.b2), "adaln_w": p.adaln_w, "adaln_b": p.adaln_b}
    t = np.array([0.1, 0.9], dtype=np.float32)
    out = om.produce(params, t, None, 0.0)
    assert out.shape == (dims.n_tags, 2, 6, dims.hidden)
    flat = om.modulation_table(om.two_time_embedding(t, None, 0.0, params["mlp"], None, md.freq_dim),
                               p.adaln_w, p.adaln_b)
    np.testing.assert_array_equal(out[2, 1, 3], flat[2, 1, 3 * dims.hidden:4 * dims.hidden])


def test_two_time_sets_order():
    tn, te = hi.two_time_sets([0.9, 0.5], [0.6, 0.1])
    # table index 2 * i + j pairs t_now[i] with t_end[j]
    np.testing.assert_array_equal(tn, np.float32([0.9, 0.9, 0.5, 0.5]))
    np.testing.assert_array_equal(te, np.float32([0.6, 0.1, 0.6, 0.1]))
