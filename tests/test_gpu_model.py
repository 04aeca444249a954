"""GPU parity of the model shell (h3blk_model_forward, h3blk_model_graph_create)
against the fp64 model oracle (oracle/h3_model.py): input projections, token
refiner, the block stack with per-layer tables, norm_out and both heads."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import h3_inputs as hi
from oracle.h3_model import ModelOracle
from tests._parity import REL_RMS, assert_intermediate, errors

pytestmark = pytest.mark.gpu


def _case(two_time=False, quant=0, n_layers=2, n_refiner=1, layout=None, seed=0):
    d, lay = hi.workload("tiny_320", seed)
    if two_time:
        d = replace(d, n_t=4)
        lay = hi.layout_two_time(lay, seed)
    if layout is not None:
        lay = layout
    d = replace(d, quant=quant)
    sd = replace(hi.TINY_SHELL, n_layers=n_layers, n_refiner=n_refiner)
    p = hi.make_model_params(d, hi.TINY_MOD, sd, seed, two_time)
    mi = hi.make_model_inputs(d, sd, lay, seed, two_time)
    return d, sd, p, mi


def _run(d, sd, p, mi):
    import joint_video_audio_b200 as j
    m = j.Model(d, sd)
    dm = m.load(p)
    di = j.DeviceInputs.from_model_inputs(mi)
    vo, ao, ws = m.buffers(dm, di)
    m.forward(dm, di, vo, ao, ws)
    assert m.check(ws) == 0
    return m, dm, di, vo, ao, ws


def _compare(vo, ao, ref, tag=""):
    out = {}
    for name, g, r in (("video", vo, ref["video"]), ("audio", ao, ref["audio"])):
        if r.size:
            out[name] = assert_intermediate(f"{tag}{name}", g, r)
        else:
            assert g.numel() == 0
    return out


@pytest.mark.parametrize("two_time,quant", [(False, 0), (True, 0), (True, 1)])
def test_tiny_model_matches_oracle(two_time, quant):
    d, sd, p, mi = _case(two_time=two_time, quant=quant)
    _, _, _, vo, ao, _ = _run(d, sd, p, mi)
    torch.cuda.synchronize()
    ref = ModelOracle(d, p).forward(mi)
    _compare(vo, ao, ref)


def test_shell_only_matches_oracle():
    """No stack layers: projections, refiner, norm_out and heads alone. Only
    the packed rows' bf16 rounding separates the two."""
    d, sd, p, mi = _case(n_layers=0, n_refiner=1)
    _, _, _, vo, ao, _ = _run(d, sd, p, mi)
    torch.cuda.synchronize()
    ref = ModelOracle(d, p).forward(mi)
    e = _compare(vo, ao, ref)
    assert e["video"][1] < 3e-3   # one bf16 rounding of the projected rows


def test_layout_without_text_and_audio():
    """Only video and padding rows: the refiner and the audio head are skipped
    and the padding rows stay zero through the stack."""
    b = hi._Builder("video_only")
    b.add("video", hi.TAG_VIDEO, 0, hi.grid_positions(3, 8, 8))
    b.add("pad", hi.TAG_PAD, 0, hi.pad_positions(64))
    lay = b.build()
    lay.tidx = np.random.default_rng(4).integers(0, 2, size=lay.n).astype(np.int32)
    d, sd, p, mi = _case(layout=lay)
    assert mi.text_idx.size == 0 and mi.audio_idx.size == 0
    _, _, _, vo, ao, ws = _run(d, sd, p, mi)
    torch.cuda.synchronize()
    ref = ModelOracle(d, p).forward(mi)
    _compare(vo, ao, ref)
    assert ao.shape == (0, sd.audio_in)


def test_graph_replay_matches_eager_and_follows_new_inputs():
    import joint_video_audio_b200 as j
    d, sd, p, mi = _case(two_time=True)
    m, dm, di, vo, ao, ws = _run(d, sd, p, mi)
    eager_v, eager_a = vo.clone(), ao.clone()
    g = m.graph(dm, di, vo, ao, ws)
    vo.zero_()
    ao.zero_()
    g.launch()
    torch.cuda.synchronize()
    assert torch.equal(vo, eager_v) and torch.equal(ao, eager_a)   # same launches, same order
    # a new step: new timesteps and latents written into the same device buffers
    tn, te = hi.two_time_sets(np.float32([0.31, 0.9]), np.float32([0.05, 0.6]))
    mi2 = replace(mi, t_now=tn, t_end=te, video=mi.video * 0.5 - 0.25)
    di.t["t_now"].copy_(torch.from_numpy(tn))
    di.t["t_end"].copy_(torch.from_numpy(te))
    di.t["video"].copy_(mi2.video)
    g.launch()
    assert j.Model.check(ws) == 0
    ref = ModelOracle(d, p).forward(mi2)
    _compare(vo, ao, ref, "graph ")
    del g


def test_bad_row_index_is_reported():
    import joint_video_audio_b200 as j
    d, sd, p, mi = _case(n_layers=1)
    vi = mi.video_idx.copy()
    vi[7] = mi.layout.n + 5        # outside the packed sequence
    mi = replace(mi, video_idx=vi)
    m = j.Model(d, sd)
    dm = m.load(p)
    di = j.DeviceInputs.from_model_inputs(mi)
    vo, ao, ws = m.buffers(dm, di)
    m.forward(dm, di, vo, ao, ws)
    assert m.check(ws) == j.capi.H3BLK_ERR_BAD_INDEX


@pytest.mark.slow
def test_real_dims_model_sampled_rows():
    """Real dimensions on the 8k layout: 2 refiner layers over the 512 text rows
    and one stack layer; sampled rows against the oracle's subset mode."""
    d, lay = hi.workload("real_8k")
    sd = replace(hi.REAL_SHELL, n_layers=1, n_refiner=2)
    p = hi.make_model_params(d, hi.REAL_MOD, sd)
    mi = hi.make_model_inputs(d, sd, lay)
    _, _, _, vo, ao, _ = _run(d, sd, p, mi)
    torch.cuda.synchronize()
    rows = hi.sample_rows(lay, k=96, k_pad=0, seed=1)
    ref = ModelOracle(d, p).forward(mi, rows=rows)
    assert ref["video_sel"].size > 40 and ref["audio_sel"].size > 0
    assert_intermediate("video", vo[torch.from_numpy(ref["video_sel"]).cuda()], ref["video"])
    assert_intermediate("audio", ao[torch.from_numpy(ref["audio_sel"]).cuda()], ref["audio"])
    ma, rr = errors(vo[torch.from_numpy(ref["video_sel"]).cuda()], ref["video"])
    assert rr <= REL_RMS
