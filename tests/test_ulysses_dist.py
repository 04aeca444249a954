"""Host-side tests of the sequence-parallel (Ulysses) plan: index algebra,
and a world-size-2 gloo run of the collective form of the exchange on CPU,
with the fp64 oracle computing each rank's share; the result must equal the
oracle's single-process block."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import h3_inputs as hi
from joint_video_audio_b200.ulysses import UlyssesPlan


def test_plan_partitions_rows_and_heads():
    p = UlyssesPlan(320, 6, 64, 2)
    assert (p.n_local, p.hg) == (160, 3)
    assert p.rows(1) == slice(160, 320)
    assert list(p.head_range(1)) == [3, 4, 5]
    cols = torch.cat([p.qkv_columns(d) for d in range(2)])
    assert sorted(cols.tolist()) == list(range(3 * 6 * 64))     # every column exactly once
    # group 1's first columns: q of head 3
    assert p.qkv_columns(1)[:2].tolist() == [3 * 64, 3 * 64 + 1]
    with pytest.raises(ValueError):
        UlyssesPlan(320, 6, 64, 4)       # 4 does not divide 6 heads
    with pytest.raises(ValueError):
        UlyssesPlan(322, 6, 64, 3)       # 3 does not divide 322 rows


def test_pack_merge_round_trip():
    """Packing every rank's rows by head group and merging the received blocks
    gives each group owner the q|k|v of its heads over all rows; packing the
    attention outputs by row owner and merging gives each rank all heads of
    its rows."""
    G, N, H, D = 4, 64, 8, 4
    p = UlyssesPlan(N, H, D, G)
    full = torch.randn(N, 3 * H * D)
    sent = [p.pack_qkv(full[p.rows(r)]) for r in range(G)]        # [G][G, nl, 3 hg D]
    for d in range(G):
        got = p.merge_qkv(torch.stack([sent[r][d] for r in range(G)]))
        assert torch.equal(got, full[:, p.qkv_columns(d)])
    o_full = torch.randn(N, H * D)
    o_sent = [p.pack_o(o_full[:, p.head_range(g)[0] * D:(p.head_range(g)[-1] + 1) * D]) for g in range(G)]
    for r in range(G):
        got = p.merge_o(torch.stack([o_sent[g][r] for g in range(G)]))
        assert torch.equal(got, o_full[p.rows(r)])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    from oracle.h3_block import (BlockOracle, MOD_GATE1, MOD_GATE2, MOD_SCALE1, MOD_SCALE2, MOD_SHIFT1,
                                 MOD_SHIFT2, adaln, attention, documents, modulation, swiglu)
    os.environ["MASTER_ADDR"], os.environ["MASTER_PORT"] = "127.0.0.1", str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = hi.make_inputs("tiny_320")
        d, lay = inp.dims, inp.layout
        orc = BlockOracle(d, inp.weights)
        p = UlyssesPlan(lay.n, d.heads, d.head_dim, world)
        rows = p.rows(rank)
        x = inp.x.double().numpy()[rows]
        m = modulation(inp.table, lay.tag[rows], lay.tidx[rows])
        h1 = adaln(x, m[:, MOD_SHIFT1], m[:, MOD_SCALE1], d.norm_eps)
        parts = orc.qkv(h1, lay.pos[rows])                            # [nl, H, D] each
        qkv = torch.from_numpy(np.concatenate([parts[k].reshape(len(x), -1) for k in ("q", "k", "v")], axis=1))
        send = p.pack_qkv(qkv).contiguous()
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send)
        mine = p.merge_qkv(recv).numpy()                               # [N, 3 hg D]
        hgD = p.hg * d.head_dim
        qh, kh, vh = (mine[:, i * hgD:(i + 1) * hgD].reshape(lay.n, p.hg, d.head_dim) for i in range(3))
        doc = documents(lay.tag)
        o_grp = torch.from_numpy(attention(qh, kh, vh, doc, doc).reshape(lay.n, hgD))
        osend = p.pack_o(o_grp).contiguous()
        orecv = torch.empty_like(osend)
        dist.all_to_all_single(orecv, osend)
        o = p.merge_o(orecv).numpy()                                   # [nl, H D]
        x1 = x + m[:, MOD_GATE1] * orc.linear(o, "o")
        h2 = adaln(x1, m[:, MOD_SHIFT2], m[:, MOD_SCALE2], d.norm_eps)
        g_u = orc.linear(h2, "13")
        out = x1 + m[:, MOD_GATE2] * orc.linear(swiglu(g_u[:, :d.ffn], g_u[:, d.ffn:]), "2")
        gathered = [torch.empty(p.n_local, d.hidden, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, torch.from_numpy(out))
        if rank == 0:
            q.put(torch.cat(gathered).numpy())
    finally:
        dist.destroy_process_group()


def test_collective_exchange_world2_matches_single_process_oracle():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    got = q.get(timeout=300)
    for pr in procs:
        pr.join(timeout=120)
        assert pr.exitcode == 0
    from oracle.h3_block import BlockOracle
    inp = hi.make_inputs("tiny_320")
    lay = inp.layout
    ref = BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)["out"]
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-10)
