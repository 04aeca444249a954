"""GPU parity of the modulation-table producer (h3blk_modulation_table)
against the fp64 oracle (oracle/h3_modulation.py), and the producer feeding
h3blk_forward."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import h3_inputs as hi
from oracle import h3_modulation as om
from tests._parity import assert_stage, errors

pytestmark = pytest.mark.gpu


def _oracle_table(p, t_now, t_end, gate):
    params = {"freq_dim": p.md.freq_dim, "mlp": (p.w1, p.b1, p.w2, p.b2), "adaln_w": p.adaln_w, "adaln_b": p.adaln_b}
    if p.w1_r is not None:
        params["mlp_r"] = (p.w1_r, p.b1_r, p.w2_r, p.b2_r)
    return om.produce(params, t_now, t_end, gate)


@pytest.mark.parametrize("dims,md,two_time", [
    (hi.TINY, hi.TINY_MOD, False),
    (replace(hi.TINY, n_t=4), hi.TINY_MOD, True),
    (replace(hi.REAL, n_t=3), hi.REAL_MOD, False),
    (replace(hi.REAL, n_t=4), hi.REAL_MOD, True),
])
def test_modulation_table_matches_oracle(dims, md, two_time):
    import joint_video_audio_b200 as j
    p = hi.make_modulation_params(dims, md, two_time=two_time)
    if two_time:
        t_now, t_end = hi.two_time_sets([0.83, 0.41], [0.55, 0.12])
        gate = 0.35
    else:
        t_now = np.linspace(0.05, 0.95, dims.n_t).astype(np.float32)
        t_end, gate = None, 0.0
    blk = j.H3Block(dims)
    w = j.ModulationWeights(p)
    got = j.modulation_table(blk, w, t_now, t_end, gate)
    torch.cuda.synchronize()
    ref = _oracle_table(p, t_now, t_end, gate)
    assert_stage("table", got, ref)
    ma, rr = errors(got, ref)
    assert rr < 1e-5, rr  # fp32 arithmetic throughout: far inside the block tolerance


def test_produced_table_drives_the_block():
    import joint_video_audio_b200 as j
    from oracle.h3_block import BlockOracle
    inp = hi.make_inputs("tiny_320")
    p = hi.make_modulation_params(inp.dims, hi.TINY_MOD)
    t_now = np.float32([0.7, 0.2])
    blk = j.H3Block(inp.dims)
    table = j.modulation_table(blk, j.ModulationWeights(p), t_now)
    w = j.DeviceWeights.from_host(inp.weights)
    lay = inp.layout
    out = blk.forward(inp.x.cuda(), inp.tag.cuda(), inp.tidx.cuda(), inp.pos.cuda().contiguous(), table, w)
    torch.cuda.synchronize()
    ref_table = _oracle_table(p, t_now, None, 0.0)
    ref = BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, ref_table)["out"]
    assert_stage("out", out, ref)
