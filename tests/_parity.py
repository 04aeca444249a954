"""Shared helpers of the GPU parity tests (host-side only)."""
from __future__ import annotations

import numpy as np
import torch

import h3_inputs as hi

# Float tolerance of the block (bf16 I/O, fp32 accumulation) against the fp64
# oracle: on the block output, max |gpu - ref| <= 3e-2 and
# rms(gpu - ref) / rms(ref) <= 1e-2. Intermediate stages are stored in bf16 at
# their own magnitude (SwiGLU outputs reach ~10, where one bf16 ulp is 0.06),
# so their elementwise bound also scales with the value: |d| <= 3e-2 + 2^-7 |ref|
# (two bf16 ulps), together with the same relative-RMS bound.
MAX_ABS = 3e-2
REL_RMS = 1e-2
STAGE_RTOL = 2.0 ** -7


def to64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().float().cpu().numpy().astype(np.float64)
    return np.asarray(t, dtype=np.float64)


def errors(gpu, ref):
    g, r = to64(gpu), to64(ref)
    d = g - r
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    denom = float(np.mean(r * r)) if r.size else 1.0
    rel = float(np.sqrt(np.mean(d * d) / denom)) if denom > 0 else float(np.sqrt(np.mean(d * d)))
    return max_abs, rel


def assert_stage(name, gpu, ref, max_abs=MAX_ABS, rel_rms=REL_RMS, rtol=None):
    """rtol=None: the block-output bound (max-abs); otherwise max-abs + rtol |ref|."""
    g, r = to64(gpu), to64(ref)
    ma, rr = errors(g, r)
    assert np.all(np.isfinite(g)), f"{name}: non-finite values"
    if rtol is None:
        ok_abs = ma <= max_abs
    else:
        excess = np.abs(g - r) - (max_abs + rtol * np.abs(r))
        ok_abs = bool(np.all(excess <= 0))
    assert ok_abs and rr <= rel_rms, (f"{name}: max_abs {ma:.3e} (bound {max_abs}" +
                                      (f" + {rtol:.4f}|ref|" if rtol else "") + f"), rel_rms {rr:.3e} (<= {rel_rms})")
    return ma, rr


def assert_intermediate(name, gpu, ref, rel_rms=REL_RMS):
    return assert_stage(name, gpu, ref, rel_rms=rel_rms, rtol=STAGE_RTOL)


class GpuCase:
    """Inputs of one workload resident on the GPU, run through libh3blk."""

    def __init__(self, inp: hi.Inputs, device="cuda"):
        import joint_video_audio_b200 as j
        self.inp = inp
        self.dims = inp.dims
        self.n = inp.layout.n
        self.x = inp.x.to(device)
        self.tag = inp.tag.to(device)
        self.tidx = inp.tidx.to(device)
        self.pos = inp.pos.to(device).contiguous()
        self.table = inp.table.to(device)
        self.block = j.H3Block(inp.dims)
        w = j.DeviceWeights.from_host(inp.weights, device)
        self.w_bf16 = w
        self.w = self.block.prepare_int8(w) if inp.dims.quant else w
        self.ws = self.block.workspace(self.n, device)
        self.out = torch.empty_like(self.x)

    def run(self, x=None, table=None):
        self.block.forward(self.x if x is None else x, self.tag, self.tidx, self.pos,
                           self.table if table is None else table, self.w, out=self.out, workspace=self.ws)
        torch.cuda.synchronize()
        return self.out

    def stage(self, name):
        return self.block.stage(self.ws, self.n, name)

    def qkv(self, rows=None):
        d = self.dims
        hd = d.heads * d.head_dim
        t = self.stage("QKV")
        if rows is not None:
            t = t[torch.as_tensor(rows, device=t.device)]
        t = t.float().cpu()
        r = t.shape[0]
        return (t[:, :hd].reshape(r, d.heads, d.head_dim), t[:, hd:2 * hd].reshape(r, d.heads, d.head_dim),
                t[:, 2 * hd:].reshape(r, d.heads, d.head_dim))


def rows_of(t, rows):
    if rows is None:
        return t
    return t[torch.as_tensor(rows, device=t.device)]


def blob_tensor(dw, ptr, numel, dtype):
    """View of one array inside the int8 weight blob written by the library."""
    off = ptr - dw.blob.data_ptr()
    nbytes = numel * torch.tensor([], dtype=dtype).element_size()
    return dw.blob[off:off + nbytes].view(dtype)
