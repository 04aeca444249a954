"""torch-tensor marshalling around the h3blk C-ABI (no arithmetic here).

``H3Block`` owns one h3blk handle; its methods check tensor devices, dtypes,
shapes and contiguity, pass raw pointers and the current CUDA stream to the
library, and turn non-zero status codes into exceptions.
"""
from __future__ import annotations

import torch

from . import _binding as B

_DT = {"bf16": torch.bfloat16, "i8": torch.int8, "f32": torch.float32, "i32": torch.int32}


def _ptr(t):
    return 0 if t is None else t.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def make_config(dims) -> B.h3blk_config:
    """dims: any object with hidden, heads, head_dim, ffn, n_tags, n_t,
    rope_pairs (t, h, w), rope_theta, norm_eps, qk_norm_eps, quant."""
    pt, ph, pw = dims.rope_pairs
    return B.h3blk_config(hidden=dims.hidden, heads=dims.heads, head_dim=dims.head_dim, ffn=dims.ffn,
                          n_tags=dims.n_tags, n_t=dims.n_t, rope_pairs_t=pt, rope_pairs_h=ph, rope_pairs_w=pw,
                          rope_theta=float(dims.rope_theta), norm_eps=float(dims.norm_eps),
                          qk_norm_eps=float(dims.qk_norm_eps), quant=int(getattr(dims, "quant", 0)))


class DeviceWeights:
    """Block weights resident on the GPU, and the C struct pointing at them."""

    def __init__(self, tensors: dict, keepalive=None):
        self.t = tensors
        self._keep = keepalive
        self.c = B.h3blk_weights(**{k: _ptr(tensors.get(k)) for k, _ in B.h3blk_weights._fields_})

    @classmethod
    def from_host(cls, w, device="cuda"):
        """w: object with bf16 tensors wqkv, q_gain, k_gain, wo, w13, w2."""
        t = {k: getattr(w, k).to(device=device, dtype=torch.bfloat16).contiguous()
             for k in ("wqkv", "q_gain", "k_gain", "wo", "w13", "w2")}
        return cls(t)


class H3Block:
    def __init__(self, dims):
        self.dims = dims
        self.cfg = make_config(dims)
        self.handle = B.h3blk_create(self.cfg)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and B is not None and getattr(B, "h3blk_destroy", None) is not None:
            # at interpreter exit the binding may already be torn down; the
            # process exit then releases the handle
            B.h3blk_destroy(h)
        self.handle = None

    # ------------------------------------------------------------ attention mode
    def set_attention_density(self, density: float) -> None:
        """1.0: dense attention; below: block-sparse (h3blk_set_attention_density).
        The workspace size follows the setting."""
        st = B.h3blk_set_attention_density(self.handle, float(density))
        if st != B.H3BLK_OK:
            raise B.H3BlkError("h3blk_set_attention_density", st)

    # ------------------------------------------------------------ workspace
    def workspace_bytes(self, n_rows: int) -> int:
        return B.h3blk_workspace_bytes(self.handle, n_rows)

    def workspace(self, n_rows: int, device="cuda") -> torch.Tensor:
        return torch.empty(self.workspace_bytes(n_rows), dtype=torch.uint8, device=device)

    def stage(self, workspace: torch.Tensor, n_rows: int, name: str) -> torch.Tensor:
        """View of a stage buffer inside the workspace (see h3blk_stage_view)."""
        off, nb = B.h3blk_stage_view(self.handle, n_rows, name)
        raw = workspace[off:off + nb]
        d = self.dims
        hd = d.heads * d.head_dim
        shapes = {"H1": ("bf16", d.hidden), "H2": ("bf16", d.hidden), "X1": ("bf16", d.hidden),
                  "QKV": ("bf16", 3 * hd), "O": ("bf16", hd), "A": ("bf16", d.ffn),
                  "H1_Q8": ("i8", d.hidden), "H2_Q8": ("i8", d.hidden), "O_Q8": ("i8", hd), "A_Q8": ("i8", d.ffn),
                  "H1_SCALE": ("f32", 1), "H2_SCALE": ("f32", 1), "O_SCALE": ("f32", 1), "A_SCALE": ("f32", 1),
                  "ERROR": ("i32", 1), "KV_LIST": ("i32", 1)}
        dt, cols = shapes[name]
        v = raw.view(_DT[dt])
        if name == "ERROR":
            return v
        if name == "KV_LIST":
            n_tiles = (n_rows + 127) // 128
            return v.view((n_tiles + 1) // 2, d.heads, 1 + n_tiles)
        return v.view(n_rows, cols) if cols > 1 else v.view(n_rows)

    # ------------------------------------------------------------ int8 weights
    def prepare_int8(self, w: DeviceWeights) -> DeviceWeights:
        nb = B.h3blk_int8_weights_bytes(self.handle)
        blob = torch.empty(nb, dtype=torch.uint8, device=w.t["wqkv"].device)
        c = B.h3blk_prepare_int8_weights(self.handle, w.c, blob.data_ptr(), nb, _stream())
        dw = DeviceWeights.__new__(DeviceWeights)
        dw.t, dw._keep, dw.c = {}, blob, c
        dw.blob = blob
        return dw

    # ------------------------------------------------------------ forward
    def forward(self, x, tag, tidx, pos, table, w: DeviceWeights, out=None, workspace=None) -> torch.Tensor:
        n = x.shape[0]
        d = self.dims
        dev = x.device
        assert dev.type == "cuda", "h3blk runs on the GPU only"
        for t, dt, shape in ((x, torch.bfloat16, (n, d.hidden)), (tag, torch.int32, (n,)),
                             (tidx, torch.int32, (n,)), (pos, torch.int32, (n, 3)),
                             (table, torch.float32, (d.n_tags, d.n_t, 6, d.hidden))):
            if t.dtype != dt or tuple(t.shape) != shape or not t.is_contiguous() or t.device != dev:
                raise ValueError(f"expected {dt} {shape} contiguous on {dev}, got {t.dtype} {tuple(t.shape)}")
        if out is None:
            out = torch.empty_like(x)
        if workspace is None:
            workspace = self.workspace(n, dev)
        st = B.h3blk_forward(self.handle, n, x.data_ptr(), tag.data_ptr(), tidx.data_ptr(), pos.data_ptr(),
                             table.data_ptr(), w.c, out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                             _stream())
        if st != B.H3BLK_OK:
            raise B.H3BlkError("h3blk_forward", st)
        return out

    def check(self, workspace: torch.Tensor, n_rows: int) -> int:
        return B.h3blk_check(self.handle, n_rows, workspace.data_ptr(), _stream())


# ---------------------------------------------------------------- kernel-level calls

def rotate_quantize(x: torch.Tensor):
    """bf16 [rows, K] -> (int8 [rows, K], fp32 [rows])."""
    assert x.is_cuda and x.dtype == torch.bfloat16 and x.is_contiguous() and x.dim() == 2
    q = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    s = torch.empty(x.shape[0], dtype=torch.float32, device=x.device)
    st = B.h3blk_rotate_quantize(x.shape[0], x.shape[1], x.data_ptr(), q.data_ptr(), s.data_ptr(), _stream())
    if st != B.H3BLK_OK:
        raise B.H3BlkError("h3blk_rotate_quantize", st)
    return q, s


def gemm_s8_s32(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """int8 A [M, K], B [N, K] -> exact int32 A B^T."""
    assert a.is_cuda and a.dtype == torch.int8 and b.dtype == torch.int8 and a.shape[1] == b.shape[1]
    c = torch.empty(a.shape[0], b.shape[0], dtype=torch.int32, device=a.device)
    st = B.h3blk_gemm_s8_s32(a.shape[0], b.shape[0], a.shape[1], a.data_ptr(), b.data_ptr(), c.data_ptr(), _stream())
    if st != B.H3BLK_OK:
        raise B.H3BlkError("h3blk_gemm_s8_s32", st)
    return c


def gemm_bf16(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """bf16 A [M, K], B [N, K] -> bf16 A B^T (fp32 accumulation)."""
    assert a.is_cuda and a.dtype == torch.bfloat16 and b.dtype == torch.bfloat16 and a.shape[1] == b.shape[1]
    c = torch.empty(a.shape[0], b.shape[0], dtype=torch.bfloat16, device=a.device)
    st = B.h3blk_gemm_bf16(a.shape[0], b.shape[0], a.shape[1], a.data_ptr(), b.data_ptr(), c.data_ptr(), _stream())
    if st != B.H3BLK_OK:
        raise B.H3BlkError("h3blk_gemm_bf16", st)
    return c


# ---------------------------------------------------------------- modulation-table producer

class ModulationWeights:
    """Producer weights resident on the GPU and the C struct pointing at them."""

    def __init__(self, p, device="cuda"):
        """p: object with md (freq_dim, time_hidden, time_dim), fp32 w1, b1, w2,
        b2 (and optional *_r copies), bf16 adaln_w, fp32 adaln_b."""
        f32 = lambda t: None if t is None else t.to(device=device, dtype=torch.float32).contiguous()  # noqa: E731
        self.t = {k: f32(getattr(p, k)) for k in ("w1", "b1", "w2", "b2", "w1_r", "b1_r", "w2_r", "b2_r", "adaln_b")}
        self.t["adaln_w"] = p.adaln_w.to(device=device, dtype=torch.bfloat16).contiguous()
        self.c = B.h3blk_mod_weights(freq_dim=p.md.freq_dim, time_hidden=p.md.time_hidden, time_dim=p.md.time_dim,
                                     **{k: _ptr(v) for k, v in self.t.items()})


def modulation_table(block: H3Block, w: ModulationWeights, t_now, t_end=None, gate=0.0, scratch=None):
    """fp32 table [n_tags, n_t, 6, hidden] for h3blk_forward."""
    d = block.dims
    dev = w.t["w1"].device
    table = torch.empty(d.n_tags, d.n_t, 6, d.hidden, dtype=torch.float32, device=dev)
    nb = B.h3blk_modulation_scratch_bytes(block.handle, w.c)
    if scratch is None:
        scratch = torch.empty(nb, dtype=torch.uint8, device=dev)
    st = B.h3blk_modulation_table(block.handle, w.c, list(t_now), None if t_end is None else list(t_end), gate,
                                  table.data_ptr(), scratch.data_ptr(), scratch.numel(), _stream())
    if st != B.H3BLK_OK:
        raise B.H3BlkError("h3blk_modulation_table", st)
    return table
