"""The seeded synthetic workloads have the shapes their recipe states (row
counts per modality, padding, tags, timestep indices, positions, dimensions),
so every parity case and the bench run on the stated inputs."""
import numpy as np
import pytest

import h3_inputs as hi


def _count(lay, tag):
    return int((lay.tag == tag).sum())


@pytest.mark.parametrize("name,n,v,text,audio,video,cond", [
    ("tiny_320", 320, 288, 64, 32, 192, 0),
    ("real_8k", 8192, 8192, 512, 256, 7424, 0),
    ("t2va_32k", 32768, 32768, 512, 1008, 31248, 0),
    ("t2va_32k_pad168", 32768, 32600, 512, 1008, 31248 - 168, 0),
    ("ref2va_54k", 54528, 54320, 512, 1008 + 3 * 128, 31248, 9 * 24 * 42 + 3 * 4 * 24 * 42),
    ("w8a8_t2va_32k", 32768, 32768, 512, 1008, 31248, 0),
])
def test_row_counts(name, n, v, text, audio, video, cond):
    _, lay = hi.workload(name)
    assert lay.n == n and lay.n_valid == v and lay.n_pad == n - v
    assert _count(lay, hi.TAG_TEXT) == text
    assert _count(lay, hi.TAG_AUDIO) == audio
    assert _count(lay, hi.TAG_VIDEO) == video
    assert _count(lay, hi.TAG_COND) == cond
    # padding, where there is any, is a tail of the sequence
    pad = np.nonzero(lay.tag == hi.TAG_PAD)[0]
    assert pad.size == n - v and (pad.size == 0 or pad[0] == n - pad.size)


def test_dimensions():
    d, _ = hi.workload("real_8k")
    assert (d.hidden, d.heads, d.head_dim, d.ffn) == (5376, 56, 128, 14336)
    assert sum(d.rope_pairs) == d.head_dim // 2
    t, _ = hi.workload("tiny_320")
    assert (t.hidden, t.heads, t.head_dim, t.ffn) == (256, 6, 64, 768)
    assert sum(t.rope_pairs) == t.head_dim // 2
    assert hi.workload("ref2va_54k")[0].n_t == 3
    w8 = hi.workload("w8a8_t2va_32k")[0]
    assert w8.n_t == 4 and w8.quant == 1


def test_timestep_indices():
    _, lay = hi.workload("t2va_32k")
    assert set(lay.tidx[lay.tag == hi.TAG_VIDEO]) == {0}
    assert set(lay.tidx[lay.tag == hi.TAG_TEXT]) == {0}
    assert set(lay.tidx[lay.tag == hi.TAG_AUDIO]) == {1}
    _, ref = hi.workload("ref2va_54k")
    assert set(ref.tidx[ref.tag == hi.TAG_COND]) == {2}
    # reference audio at index 2, target audio at index 1
    assert sorted(set(ref.tidx[ref.tag == hi.TAG_AUDIO])) == [1, 2]
    _, two = hi.workload("w8a8_t2va_32k")
    assert set(two.tidx) == {0, 1, 2, 3}
    _, tiny = hi.workload("tiny_320")
    assert set(tiny.tidx) == {0, 1}


def test_positions():
    _, lay = hi.workload("t2va_32k")
    text = lay.pos[lay.tag == hi.TAG_TEXT]
    assert np.array_equal(text[:, 0], np.arange(512)) and np.array_equal(text[:, 0], text[:, 1])
    audio = lay.pos[lay.tag == hi.TAG_AUDIO]
    assert np.array_equal(audio[:, 0], np.arange(1008)) and not audio[:, 1:].any()
    video = lay.pos[lay.tag == hi.TAG_VIDEO]
    assert video.max(axis=0).tolist() == [30, 23, 41] and len({tuple(p) for p in video}) == 31248
    _, pad = hi.workload("t2va_32k_pad168")
    assert not pad.pos[pad.tag == hi.TAG_PAD].any()
    # references advance one shared time axis: 9 images, then 3 x 4 video frames
    _, ref = hi.workload("ref2va_54k")
    cond_t = ref.pos[ref.tag == hi.TAG_COND][:, 0]
    assert cond_t.min() == 0 and cond_t.max() == 9 + 3 * 4 - 1
