"""The phase and barrier ordering of the cross-GPU Ulysses driver
(PeerGroup), checked on CPU: each rank runs in its own thread against a fake
symmetric-memory handle whose barrier is a real group barrier, and fake
library phases that record which rank buffers they write and read. The
record must show, over several forwards, that every buffer is read only
after all of that forward's writes into it and before any write of the next
forward (the exchange is race-free by construction), and that every rank
takes the same collective steps in the same order.

Source of the scheme: "HyperFlow for MiniMax-H3" model card (Usage and
Performance: Ulysses sequence parallelism over 4 GPUs)."""
import threading

import pytest
import torch

import h3_inputs as hi
import joint_video_audio_b200 as j
from joint_video_audio_b200 import _binding as B
from joint_video_audio_b200 import ulysses as U


class _Recorder:
    def __init__(self):
        self.lock = threading.Lock()
        self.events = []  # (seq, rank, kind, forward, writes, reads)

    def add(self, rank, kind, fwd, writes=(), reads=()):
        with self.lock:
            self.events.append((len(self.events), rank, kind, fwd, tuple(writes), tuple(reads)))


class _FakeSymm:
    """Per-rank handle of one symmetric buffer: every rank's pointer, and a
    barrier shared by the group."""

    def __init__(self, name, ptrs, barrier, rec, rank_of):
        self.name, self.buffer_ptrs, self._barrier, self._rec, self._rank_of = name, ptrs, barrier, rec, rank_of

    def barrier(self):
        r = self._rank_of()
        self._rec.add(r, f"barrier_{self.name}:arrive", None)
        self._barrier.wait(timeout=30)
        self._rec.add(r, f"barrier_{self.name}:leave", None)


def _run_group(G, n_forwards, monkeypatch, failing_rank=None):
    import torch.distributed as dist
    import torch.distributed._symmetric_memory as symm_mem

    rec = _Recorder()
    tls = threading.local()
    rank_of = lambda: tls.rank  # noqa: E731
    # fake symmetric allocations: rank r's buffer of kind k has pointer base_k + r
    bases = {"qkv": 1 << 40, "o": 1 << 41}
    barriers = {k: threading.Barrier(G) for k in bases}
    order = []  # allocation order of symm_mem.empty within a rank: qkv, then o

    def fake_empty(nbytes, dtype=None, device=None):
        return torch.empty(8, dtype=torch.uint8)

    calls = threading.local()

    def fake_rendezvous(buf, group):
        i = getattr(calls, "n", 0)
        calls.n = i + 1
        kind = ("qkv", "o")[i]
        order.append(kind)
        return _FakeSymm(kind, [bases[kind] + r for r in range(G)], barriers[kind], rec, rank_of)

    fwd_of = {}

    def owner(kind, ptr):
        return ptr - bases[kind]

    def fake_qkv(h, n, u, x, tag, tidx, pos, table, w, ws, wsb, s):
        r = u.rank
        if r == failing_rank:
            raise RuntimeError(f"rank {r} failed in its QKV phase")
        # the QKV epilogue stores every head group's q / k / v into its owner's buffer
        rec.add(r, "qkv", fwd_of[r], writes=[("qkv", owner("qkv", u.qkv[k])) for k in range(u.world)],
                reads=[])
        return B.H3BLK_OK

    def fake_attn(h, n, u, tag, ws, wsb, s):
        r = u.rank
        rec.add(r, "attention", fwd_of[r], writes=[("o", owner("o", u.o[k])) for k in range(u.world)],
                reads=[("qkv", owner("qkv", u.qkv[r]))])
        return B.H3BLK_OK

    def fake_out(h, n, u, x, tag, tidx, table, w, out, ws, wsb, s):
        r = u.rank
        rec.add(r, "out", fwd_of[r], writes=[], reads=[("o", owner("o", u.o[r]))])
        fwd_of[r] += 1
        return B.H3BLK_OK

    monkeypatch.setattr(symm_mem, "empty", fake_empty)
    monkeypatch.setattr(symm_mem, "rendezvous", fake_rendezvous)
    monkeypatch.setattr(dist, "get_world_size", lambda group=None: G)
    monkeypatch.setattr(dist, "get_rank", lambda group=None: tls.rank)
    monkeypatch.setattr(B, "h3blk_ulysses_qkv", fake_qkv)
    monkeypatch.setattr(B, "h3blk_ulysses_attention", fake_attn)
    monkeypatch.setattr(B, "h3blk_ulysses_out", fake_out)
    monkeypatch.setattr(U, "_stream", lambda: 0)

    from dataclasses import replace
    dims = replace(hi.TINY, heads=8)   # divisible by every group size tested
    n = 64 * G
    errors = []

    def rank_main(r):
        try:
            tls.rank = r
            fwd_of[r] = 0
            blk = j.H3Block(dims)
            pg = U.PeerGroup(blk, n, device="cpu")
            assert pg.rank == r and [pg.u.qkv[k] for k in range(G)] == [bases["qkv"] + k for k in range(G)]
            x = torch.zeros(n // G, dims.hidden, dtype=torch.bfloat16)
            meta = torch.zeros(n, 3, dtype=torch.int32)
            for _ in range(n_forwards):
                pg.forward(x, meta[:, 0], meta[:, 1], meta, meta, w=type("W", (), {"c": None})())
        except Exception as e:  # noqa: BLE001
            errors.append(e)
            for b in barriers.values():
                b.abort()

    threads = [threading.Thread(target=rank_main, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=60)
    assert not errors, errors
    return rec.events


@pytest.mark.parametrize("G", [2, 4])
def test_peer_group_phase_order_is_race_free(G, monkeypatch):
    n_fwd = 3
    ev = _run_group(G, n_fwd, monkeypatch)
    seq = {}
    for s, r, kind, f, w, rd in ev:
        if f is not None:
            seq[(r, kind, f)] = s
    # every rank ran every phase of every forward
    assert len(seq) == G * 3 * n_fwd
    # per rank: the same steps in the same order (phases and barriers)
    per_rank = [[k for _, rr, k, _, _, _ in ev if rr == r] for r in range(G)]
    assert all(p == per_rank[0] for p in per_rank)
    assert per_rank[0][:6] == ["qkv", "barrier_qkv:arrive", "barrier_qkv:leave", "attention", "barrier_o:arrive",
                               "barrier_o:leave"]
    # buffer discipline: each buffer's reads of forward f come after every
    # write of forward f into it and before any write of forward f + 1
    for kind, writer, reader in (("qkv", "qkv", "attention"), ("o", "attention", "out")):
        for b in range(G):
            for f in range(n_fwd):
                writes_f = [s for s, r, k, ff, w, _ in ev if k == writer and ff == f and (kind, b) in w]
                reads_f = [s for s, r, k, ff, _, rd in ev if k == reader and ff == f and (kind, b) in rd]
                writes_next = [s for s, r, k, ff, w, _ in ev if k == writer and ff == f + 1 and (kind, b) in w]
                assert len(writes_f) == G and len(reads_f) == 1
                assert max(writes_f) < min(reads_f), (kind, b, f)
                if writes_next:
                    assert max(reads_f) < min(writes_next), (kind, b, f)


def test_peer_group_barrier_failure_surfaces(monkeypatch):
    """A rank that fails before the first barrier makes the other ranks'
    barrier end with an error instead of waiting for good."""
    with pytest.raises(AssertionError) as e:
        _run_group(2, 1, monkeypatch, failing_rank=1)
    msg = str(e.value)
    assert "rank 1 failed" in msg and "BrokenBarrierError" in msg
