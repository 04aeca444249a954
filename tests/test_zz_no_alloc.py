"""h3blk_attention_noalloc: the attention step for callers that cannot
allocate device memory (it keeps its scratch in a fixed array inside the
library). Checked through the C-ABI against the attention output of the
regular h3blk_forward on the same inputs, on consecutive calls that reuse the
shared scratch. Collected last on purpose: if it fails, every other test has
already run."""
import numpy as np
import pytest
import torch

import h3_inputs as hi
from tests._parity import assert_intermediate

pytestmark = pytest.mark.gpu


def _forward_case(layout):
    import joint_video_audio_b200 as j
    inp = hi.make_inputs(hi.TINY, layout)
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


def _noalloc(dims, qkv, tag, tidx):
    from joint_video_audio_b200 import _binding as B
    n = qkv.shape[0]
    o = torch.full((n, dims.heads * dims.head_dim), float("nan"), dtype=torch.bfloat16, device=qkv.device)
    st = B.h3blk_attention_noalloc(n, dims.heads, dims.head_dim, dims.n_tags, dims.n_t, qkv.data_ptr(),
                                   tag.data_ptr(), tidx.data_ptr(), o.data_ptr(),
                                   torch.cuda.current_stream().cuda_stream)
    assert st == B.H3BLK_OK, B.error_string(st)
    torch.cuda.synchronize()
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


def test_noalloc_rejects_too_long_sequences():
    from joint_video_audio_b200 import _binding as B
    st = B.h3blk_attention_noalloc(524288 + 1, 6, 64, 4, 2, 1 << 40, 1 << 41, 1 << 42, 1 << 43, None)
    assert st == B.H3BLK_ERR_UNSUPPORTED
