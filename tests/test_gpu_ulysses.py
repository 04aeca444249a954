"""GPU parity of the sequence-parallel (Ulysses) block: every rank of a
group emulated on this one device (per-rank buffers, phases ordered by the
stream), the fused exchange storing into the other ranks' buffers from the
QKV and attention epilogues. Each output row is computed by the same
arithmetic as the single-device forward, so the two must agree bit for bit;
the single-device forward is itself checked against the fp64 oracle."""
from dataclasses import replace

import pytest
import torch

import h3_inputs as hi
from tests._parity import GpuCase, assert_stage

pytestmark = pytest.mark.gpu


def _run_group(case: GpuCase, world: int):
    from joint_video_audio_b200.ulysses import EmulatedGroup
    grp = EmulatedGroup(case.block, case.n, world)
    out = grp.forward(case.x, case.tag, case.tidx, case.pos, case.table, case.w)
    torch.cuda.synchronize()
    assert grp.check() == [0] * world
    return out


@pytest.mark.parametrize("world", [2])
@pytest.mark.parametrize("name,quant", [("tiny_320", 0), ("tiny_320_twotime_w8a8", 1)])
def test_tiny_group_is_bit_identical_to_one_device(name, quant, world):
    if quant:
        d, lay = hi.workload("tiny_320")
        d = replace(d, n_t=4, quant=1)
        lay = hi.layout_two_time(lay)
        inp = hi.make_inputs(d, lay)
    else:
        inp = hi.make_inputs(name)
    case = GpuCase(inp)
    single = case.run().clone()
    grouped = _run_group(case, world)
    assert torch.equal(grouped, single)
    if not quant:
        from oracle.h3_block import BlockOracle
        lay = inp.layout
        ref = BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)["out"]
        assert_stage("out", grouped, ref)


@pytest.mark.parametrize("world", [4, 8])
def test_real_dims_group_is_bit_identical_to_one_device(world):
    """Real dimensions (56 heads of 128) on the 8k layout: 14 or 7 heads and
    2048 or 1024 rows per rank."""
    case = GpuCase(hi.make_inputs("real_8k"))
    single = case.run().clone()
    grouped = _run_group(case, world)
    assert torch.equal(grouped, single)


def test_padded_layout_group():
    """168 padding rows at the tail (t2va geometry) split across 4 ranks: the
    last rank holds every padding row, and padding rows still pass through."""
    inp = hi.make_inputs("t2va_32k_pad168")
    case = GpuCase(inp)
    single = case.run().clone()
    grouped = _run_group(case, 4)
    assert torch.equal(grouped, single)
    pad = torch.from_numpy(inp.layout.tag == hi.TAG_PAD).cuda()
    assert torch.equal(grouped[pad], case.x[pad])
