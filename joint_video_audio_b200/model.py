"""torch-tensor marshalling around the model-shell entry points of libh3blk
(h3blk_model_forward, h3blk_model_graph_create): device weights, device inputs
and the C structs pointing at them. No arithmetic here; every step runs in the
library's kernels.
"""
from __future__ import annotations

import torch

from . import _binding as B
from .block import DeviceWeights, H3Block, ModulationWeights, _ptr, _stream


class DeviceModel:
    """All weights of a model resident on the GPU, and the h3blk_model_weights
    struct pointing at them. ``p`` carries time (ModulationWeights inputs),
    layers / refiner (each with w, adaln_w, adaln_b), refiner_gain,
    out_adaln_w/b and the fp32 projections; the stack's layers are converted
    to the rotated int8 blob when the block runs W8A8."""

    def __init__(self, block: H3Block, p, device="cuda"):
        f32 = lambda t: t.to(device=device, dtype=torch.float32).contiguous()  # noqa: E731
        bf = lambda t: t.to(device=device, dtype=torch.bfloat16).contiguous()  # noqa: E731
        self.time = ModulationWeights(p.time, device)
        self._keep = []

        def layer(L, quant):
            dw = L.w if isinstance(L.w, DeviceWeights) else DeviceWeights.from_host(L.w, device)
            if quant:
                dw = block.prepare_int8(dw)
            aw, ab = bf(L.adaln_w), f32(L.adaln_b)
            self._keep += [dw, aw, ab]
            return B.h3blk_layer_weights(w=dw.c, adaln_w=aw.data_ptr(), adaln_b=ab.data_ptr())

        q = int(getattr(block.dims, "quant", 0))
        lw = [layer(L, q) for L in p.layers]
        rw = [layer(L, 0) for L in p.refiner]
        self._layers = (B.h3blk_layer_weights * max(1, len(lw)))(*lw)
        self._refiner = (B.h3blk_layer_weights * max(1, len(rw)))(*rw)
        self.t = {"refiner_gain": bf(p.refiner_gain), "out_adaln_w": bf(p.out_adaln_w),
                  "out_adaln_b": f32(p.out_adaln_b), "ctx_w": bf(p.ctx_w), "ctx_b": f32(p.ctx_b)}
        for k in ("proj_in_w", "proj_in_b", "audio_in_w", "audio_in_b", "proj_out_w", "proj_out_b",
                  "audio_out_w", "audio_out_b"):
            self.t[k] = f32(getattr(p, k))
        self.n_layers, self.n_refiner = len(lw), len(rw)
        self.c = B.h3blk_model_weights(time=self.time.c, layers=self._layers, refiner=self._refiner,
                                       **{k: v.data_ptr() for k, v in self.t.items()})

    def nbytes(self) -> int:
        """Device bytes of every weight this model holds."""
        ts = list(self.t.values()) + list(self.time.t.values())
        for k in self._keep:
            if isinstance(k, DeviceWeights):
                ts += list(k.t.values()) + ([k.blob] if getattr(k, "blob", None) is not None else [])
            else:
                ts.append(k)
        return sum(t.numel() * t.element_size() for t in ts if t is not None)


class DeviceInputs:
    """One packed sequence's inputs on the GPU (int32 indices, fp32 latents,
    bf16 text states, fp32 timesteps) and the h3blk_model_inputs struct."""

    def __init__(self, layout_tag, layout_tidx, layout_pos, video_idx, audio_idx, text_idx, video, audio, text,
                 t_now, t_end=None, gate=0.0, device="cuda"):
        i32 = lambda a: torch.as_tensor(a).to(device=device, dtype=torch.int32).contiguous()  # noqa: E731
        f32 = lambda a: torch.as_tensor(a).to(device=device, dtype=torch.float32).contiguous()  # noqa: E731
        self.t = {"tag": i32(layout_tag), "tidx": i32(layout_tidx), "pos": i32(layout_pos).view(-1, 3),
                  "video_idx": i32(video_idx), "audio_idx": i32(audio_idx), "text_idx": i32(text_idx),
                  "video": f32(video), "audio": f32(audio),
                  "text": torch.as_tensor(text).to(device=device, dtype=torch.bfloat16).contiguous(),
                  "t_now": f32(t_now), "t_end": f32(t_now if t_end is None else t_end)}
        self.gate = float(gate)
        self.n_rows = self.t["tag"].numel()
        self.n_video, self.n_audio, self.n_text = (self.t[k].numel() for k in ("video_idx", "audio_idx", "text_idx"))
        self.c = B.h3blk_model_inputs(n_rows=self.n_rows, n_video=self.n_video, n_audio=self.n_audio,
                                      n_text=self.n_text, gate=self.gate,
                                      **{k: (v.data_ptr() if v.numel() else None) for k, v in self.t.items()})

    @classmethod
    def from_model_inputs(cls, mi, device="cuda"):
        """mi: h3_inputs.ModelInputs-like object."""
        lay = mi.layout
        return cls(lay.tag, lay.tidx, lay.pos, mi.video_idx, mi.audio_idx, mi.text_idx, mi.video, mi.audio,
                   mi.text, mi.t_now, mi.t_end, mi.gate, device)


class Model:
    """The transformer forward around the block stack, through the C-ABI."""

    def __init__(self, dims, sd):
        """dims: block dims (see block.make_config); sd: video_in, audio_in,
        text_dim, n_layers, n_refiner, final_norm_eps."""
        self.block = H3Block(dims)
        self.dims, self.sd = dims, sd
        self.mc = B.h3blk_model_config(n_layers=sd.n_layers, n_refiner=sd.n_refiner, video_in=sd.video_in,
                                       audio_in=sd.audio_in, text_dim=sd.text_dim,
                                       final_norm_eps=float(sd.final_norm_eps))

    def load(self, params, device="cuda") -> DeviceModel:
        dm = DeviceModel(self.block, params, device)
        if dm.n_layers != self.sd.n_layers or dm.n_refiner != self.sd.n_refiner:
            raise ValueError("layer counts of the weights and the model config differ")
        return dm

    def workspace_bytes(self, dm: DeviceModel, n_rows: int, n_text: int) -> int:
        return B.h3blk_model_workspace_bytes(self.block.handle, self.mc, dm.time.c, n_rows, n_text)

    def buffers(self, dm: DeviceModel, di: DeviceInputs):
        dev = di.t["tag"].device
        ws = torch.empty(self.workspace_bytes(dm, di.n_rows, di.n_text), dtype=torch.uint8, device=dev)
        vo = torch.empty(di.n_video, self.sd.video_in, dtype=torch.float32, device=dev)
        ao = torch.empty(di.n_audio, self.sd.audio_in, dtype=torch.float32, device=dev)
        return vo, ao, ws

    def forward(self, dm: DeviceModel, di: DeviceInputs, video_out=None, audio_out=None, workspace=None):
        """Returns (video velocity fp32 [Nv, video_in], audio velocity fp32 [Na, audio_in])."""
        if video_out is None or audio_out is None or workspace is None:
            video_out, audio_out, workspace = self.buffers(dm, di)
        st = B.h3blk_model_forward(self.block.handle, self.mc, dm.c, di.c, _ptr(video_out) or None,
                                   _ptr(audio_out) or None, workspace.data_ptr(), workspace.numel(), _stream())
        if st != B.H3BLK_OK:
            raise B.H3BlkError("h3blk_model_forward", st)
        return video_out, audio_out

    @staticmethod
    def check(workspace) -> int:
        return B.h3blk_model_check(workspace.data_ptr(), _stream())

    def graph(self, dm: DeviceModel, di: DeviceInputs, video_out, audio_out, workspace) -> "ModelGraph":
        g = B.h3blk_model_graph_create(self.block.handle, self.mc, dm.c, di.c, _ptr(video_out) or None,
                                       _ptr(audio_out) or None, workspace.data_ptr(), workspace.numel())
        return ModelGraph(g, (dm, di, video_out, audio_out, workspace))


class ModelGraph:
    """An instantiated CUDA graph of one model forward (h3blk_graph)."""

    def __init__(self, handle, keepalive):
        self.handle = handle
        self._keep = keepalive

    @property
    def nodes(self) -> tuple[int, int]:
        """(kernel launches, other nodes) of one replay."""
        return B.h3blk_graph_info(self.handle)

    def launch(self):
        st = B.h3blk_graph_launch(self.handle, _stream())
        if st != B.H3BLK_OK:
            raise B.H3BlkError("h3blk_graph_launch", st)

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and B is not None and getattr(B, "h3blk_graph_destroy", None) is not None:
            B.h3blk_graph_destroy(h)
        self.handle = None


__all__ = ["DeviceInputs", "DeviceModel", "Model", "ModelGraph"]
