"""h3blk_attention_noalloc: the attention step for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library). Checked through the C-ABI against the attention output of the
regular h3blk_forward on the same inputs, on consecutive calls that reuse the
shared scratch, at tiny and real dimensions; errors found on the device are
read back with h3blk_attention_noalloc_check. Collected last on purpose: if
it fails, every other test has already run."""
import numpy as np
import pytest
import torch

import h3_inputs as hi
from tests._parity import assert_intermediate

pytestmark = pytest.mark.gpu


def _forward_case(layout, dims=hi.TINY):
    import joint_video_audio_b200 as j
    inp = hi.make_inputs(dims, layout)
    dev = torch.device("cuda")
    blk = j.H3Block(inp.dims)
    w = j.DeviceWeights.from_host(inp.weights, dev)
    ws = blk.workspace(layout.n, dev)
    tag, tidx = inp.tag.to(dev), inp.tidx.to(dev)
    blk.forward(inp.x.to(dev), tag, tidx, inp.pos.to(dev).contiguous(), inp.table.to(dev), w, workspace=ws)
    torch.cuda.synchronize()
    qkv = blk.stage(ws, layout.n, "QKV").clone()
    o_ref = blk.stage(ws, layout.n, "O").clone()
    return inp.dims, qkv, tag, tidx, o_ref


def _noalloc(dims, qkv, tag, tidx, expect=None):
    """One call through the C-ABI, then its device-side status read back with
    h3blk_attention_noalloc_check (H3BLK_OK unless `expect` says otherwise)."""
    from joint_video_audio_b200 import _binding as B
    n = qkv.shape[0]
    o = torch.full((n, dims.heads * dims.head_dim), float("nan"), dtype=torch.bfloat16, device=qkv.device)
    stream = torch.cuda.current_stream().cuda_stream
    st = B.h3blk_attention_noalloc(n, dims.heads, dims.head_dim, dims.n_tags, dims.n_t, qkv.data_ptr(),
                                   tag.data_ptr(), tidx.data_ptr(), o.data_ptr(), stream)
    assert st == B.H3BLK_OK, B.error_string(st)
    dev_status = B.h3blk_attention_noalloc_check(stream)
    want = B.H3BLK_OK if expect is None else expect
    assert dev_status == want, f"device status {B.error_string(dev_status)}, expected {B.error_string(want)}"
    return o


def test_noalloc_attention_matches_forward_on_consecutive_calls():
    assert torch.cuda.is_available()
    base = hi.layout_tiny()
    perm = np.random.default_rng(11).permutation(base.n)[:300]  # ragged, padding scattered
    other = hi.Layout("tiny_perm300", base.tag[perm], base.tidx[perm], base.pos[perm])
    cases = [_forward_case(base), _forward_case(other)]
    # two calls in a row on each case, alternating so the shared scratch always
    # holds the previous (different) sequence's tile summary
    for _ in range(2):
        for dims, qkv, tag, tidx, o_ref in cases:
            o = _noalloc(dims, qkv, tag, tidx)
            assert torch.isfinite(o.float()).all()
            assert_intermediate("o (no-alloc vs forward)", o, o_ref)


def test_noalloc_reports_an_out_of_range_tag_then_recovers():
    """A tag outside the table is found on the device and comes back through
    h3blk_attention_noalloc_check as BAD_INDEX (the call itself only covers
    the launch); the next valid call reports OK and matches the forward."""
    from joint_video_audio_b200 import _binding as B
    dims, qkv, tag, tidx, o_ref = _forward_case(hi.layout_tiny())
    bad = tag.clone()
    bad[17] = dims.n_tags
    _noalloc(dims, qkv, bad, tidx, expect=B.H3BLK_ERR_BAD_INDEX)
    bad_t = tidx.clone()
    bad_t[200] = dims.n_t
    _noalloc(dims, qkv, tag, bad_t, expect=B.H3BLK_ERR_BAD_INDEX)
    o = _noalloc(dims, qkv, tag, tidx)
    assert_intermediate("o (no-alloc after an error vs forward)", o, o_ref)


def test_noalloc_attention_at_real_dims_matches_forward():
    """56 heads x 128 over the 8192-row real-dimension sequence, twice."""
    dims, lay = hi.workload("real_8k")
    dims, qkv, tag, tidx, o_ref = _forward_case(lay, dims)
    for _ in range(2):
        o = _noalloc(dims, qkv, tag, tidx)
        assert torch.isfinite(o.float()).all()
        assert_intermediate("o (no-alloc vs forward, real dims)", o, o_ref)


def test_noalloc_rejects_too_long_sequences_and_too_many_heads():
    from joint_video_audio_b200 import _binding as B
    st = B.h3blk_attention_noalloc(524288 + 1, 6, 64, 4, 2, 1 << 40, 1 << 41, 1 << 42, 1 << 43, None)
    assert st == B.H3BLK_ERR_UNSUPPORTED
    st = B.h3blk_attention_noalloc(1024, 16384 // 128 + 1, 128, 4, 2, 1 << 40, 1 << 41, 1 << 42, 1 << 43, None)
    assert st == B.H3BLK_ERR_UNSUPPORTED
    st = B.h3blk_attention_noalloc(1024, 70000, 64, 4, 2, 1 << 40, 1 << 41, 1 << 42, 1 << 43, None)
    assert st == B.H3BLK_ERR_UNSUPPORTED
