"""Sequence parallelism (Ulysses) for the block: the plan of which rows and
heads each rank holds, and drivers that run the three phases of
h3blk_ulysses_qkv / _attention / _out. Marshalling only; every step of the
block runs in the library's kernels.

``UlyssesPlan`` is pure host logic: rank r holds rows [r * N/G, (r+1) * N/G)
and, for attention, heads [r * H/G, (r+1) * H/G). Its pack / merge helpers give
the layouts of a collective-based exchange (all-to-all of q / k / v by head
group, then of the attention output by row owner); the fused path stores those
same layouts straight into the owners' buffers from the QKV and attention
epilogues.
"""
from __future__ import annotations

import torch

from . import _binding as B
from .block import H3Block, _ptr, _stream


class UlyssesPlan:
    def __init__(self, n_rows: int, heads: int, head_dim: int, world: int):
        if world < 1 or world > B.H3BLK_MAX_RANKS:
            raise ValueError(f"world must be in 1..{B.H3BLK_MAX_RANKS}")
        if heads % world or n_rows % world:
            raise ValueError("the group size must divide both the head count and the row count")
        self.n, self.heads, self.head_dim, self.world = n_rows, heads, head_dim, world
        self.n_local = n_rows // world
        self.hg = heads // world

    def rows(self, rank: int) -> slice:
        return slice(rank * self.n_local, (rank + 1) * self.n_local)

    def head_range(self, rank: int) -> range:
        return range(rank * self.hg, (rank + 1) * self.hg)

    def qkv_columns(self, rank: int) -> torch.Tensor:
        """Columns of a full [*, 3 H D] q|k|v row that belong to head group
        ``rank``, in the order of its [*, 3 Hg D] buffer."""
        H, D = self.heads, self.head_dim
        cols = [part * H * D + h * D + c for part in range(3) for h in self.head_range(rank) for c in range(D)]
        return torch.tensor(cols, dtype=torch.long)

    def pack_qkv(self, qkv_local: torch.Tensor) -> torch.Tensor:
        """[n_local, 3 H D] of this rank's rows -> [world, n_local, 3 Hg D]:
        block d is what head group d's owner receives."""
        return torch.stack([qkv_local[:, self.qkv_columns(d)] for d in range(self.world)])

    def merge_qkv(self, recv: torch.Tensor) -> torch.Tensor:
        """[world (source), n_local, 3 Hg D] -> [N, 3 Hg D] in sequence order."""
        return recv.reshape(self.n, 3 * self.hg * self.head_dim)

    def pack_o(self, o_group: torch.Tensor) -> torch.Tensor:
        """[N, Hg D] (this rank's heads over every row) -> [world, n_local, Hg D]:
        block d holds the rows rank d owns."""
        return o_group.reshape(self.world, self.n_local, self.hg * self.head_dim)

    def merge_o(self, recv: torch.Tensor) -> torch.Tensor:
        """[world (source head group), n_local, Hg D] -> [n_local, H D]."""
        return recv.permute(1, 0, 2).reshape(self.n_local, self.heads * self.head_dim)


def _check(fn, st):
    if st != B.H3BLK_OK:
        raise B.H3BlkError(fn, st)


class EmulatedGroup:
    """Every rank of a group on this one device: per-rank buffers and
    workspaces, the phases run rank by rank on the current stream, which
    orders them as the group barrier would. Exercises the fused exchange (the
    epilogues store into the other ranks' buffers) on a single GPU."""

    def __init__(self, block: H3Block, n_rows: int, world: int, device="cuda"):
        d = block.dims
        self.block, self.plan = block, UlyssesPlan(n_rows, d.heads, d.head_dim, world)
        qb, ob = B.h3blk_ulysses_buffer_bytes(block.handle, n_rows, world)
        wb = B.h3blk_ulysses_workspace_bytes(block.handle, n_rows, world)
        self.qkv = [torch.empty(qb, dtype=torch.uint8, device=device) for _ in range(world)]
        self.o = [torch.empty(ob, dtype=torch.uint8, device=device) for _ in range(world)]
        self.ws = [torch.empty(wb, dtype=torch.uint8, device=device) for _ in range(world)]
        self.u = []
        for r in range(world):
            u = B.h3blk_ulysses(world=world, rank=r)
            for k in range(world):
                u.qkv[k] = self.qkv[k].data_ptr()
                u.o[k] = self.o[k].data_ptr()
            self.u.append(u)

    def forward(self, x, tag, tidx, pos, table, w, out=None):
        """x / out: bf16 [N, C] (rank r's rows are x[plan.rows(r)])."""
        h, n, s = self.block.handle, self.plan.n, _stream()
        out = torch.empty_like(x) if out is None else out
        G = self.plan.world
        for r in range(G):
            _check("h3blk_ulysses_qkv", B.h3blk_ulysses_qkv(
                h, n, self.u[r], x[self.plan.rows(r)].data_ptr(), _ptr(tag), _ptr(tidx), _ptr(pos), _ptr(table),
                w.c, self.ws[r].data_ptr(), self.ws[r].numel(), s))
        for r in range(G):
            _check("h3blk_ulysses_attention", B.h3blk_ulysses_attention(
                h, n, self.u[r], _ptr(tag), self.ws[r].data_ptr(), self.ws[r].numel(), s))
        for r in range(G):
            _check("h3blk_ulysses_out", B.h3blk_ulysses_out(
                h, n, self.u[r], x[self.plan.rows(r)].data_ptr(), _ptr(tag), _ptr(tidx), _ptr(table), w.c,
                out[self.plan.rows(r)].data_ptr(), self.ws[r].data_ptr(), self.ws[r].numel(), s))
        return out

    def check(self) -> list:
        return [B.h3blk_model_check(ws.data_ptr(), _stream()) for ws in self.ws]


class PeerGroup:
    """One rank per process and GPU: the q / k / v and output buffers live in
    symmetric memory, so every rank holds its peers' pointers, and the phases
    are separated by the symmetric-memory group barrier on the compute stream.
    Needs torch.distributed initialised with NCCL and peer access between the
    GPUs."""

    def __init__(self, block: H3Block, n_rows: int, group=None, device="cuda"):
        import torch.distributed as dist
        import torch.distributed._symmetric_memory as symm_mem
        d = block.dims
        world, rank = dist.get_world_size(group), dist.get_rank(group)
        self.block, self.plan, self.rank = block, UlyssesPlan(n_rows, d.heads, d.head_dim, world), rank
        qb, ob = B.h3blk_ulysses_buffer_bytes(block.handle, n_rows, world)
        wb = B.h3blk_ulysses_workspace_bytes(block.handle, n_rows, world)
        self.qkv = symm_mem.empty(qb, dtype=torch.uint8, device=device)
        self.o = symm_mem.empty(ob, dtype=torch.uint8, device=device)
        grp = group if group is not None else dist.group.WORLD
        self.hq = symm_mem.rendezvous(self.qkv, grp)
        self.ho = symm_mem.rendezvous(self.o, grp)
        self.ws = torch.empty(wb, dtype=torch.uint8, device=device)
        self.u = B.h3blk_ulysses(world=world, rank=rank)
        for k in range(world):
            self.u.qkv[k] = int(self.hq.buffer_ptrs[k])
            self.u.o[k] = int(self.ho.buffer_ptrs[k])

    def forward(self, x_local, tag, tidx, pos, table, w, out_local=None):
        h, n, s = self.block.handle, self.plan.n, _stream()
        out_local = torch.empty_like(x_local) if out_local is None else out_local
        _check("h3blk_ulysses_qkv", B.h3blk_ulysses_qkv(
            h, n, self.u, x_local.data_ptr(), _ptr(tag), _ptr(tidx), _ptr(pos), _ptr(table), w.c,
            self.ws.data_ptr(), self.ws.numel(), s))
        self.hq.barrier()
        _check("h3blk_ulysses_attention", B.h3blk_ulysses_attention(
            h, n, self.u, _ptr(tag), self.ws.data_ptr(), self.ws.numel(), s))
        self.ho.barrier()
        _check("h3blk_ulysses_out", B.h3blk_ulysses_out(
            h, n, self.u, x_local.data_ptr(), _ptr(tag), _ptr(tidx), _ptr(table), w.c, out_local.data_ptr(),
            self.ws.data_ptr(), self.ws.numel(), s))
        return out_local
