#!/usr/bin/env python
"""Throughput of one MiniMax-H3 block forward on B200: packed rows per second.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one h3blk_forward over the 32768-row t2va-shaped packed sequence at
real dimensions (hidden 5376, 56 x 128 heads, SwiGLU 14336), inputs and
weights resident in HBM; both are larger than the 126 MB L2, so no flush is
needed between steps. The bf16 path gives `value`; the rotated W8A8 path on
the same shapes with two-time conditioning (4 modulation sets) is reported
under "w8a8". Per-kernel times come from CUDA events the library records on
its launch stream inside the timed region. `e2e` times the same C-ABI call with
the step's inputs copied from pinned host memory and the block output copied
back, inside the timed region. `cpu_baseline` times the fp64 CPU oracle on a
bounded sample of the same workload (rank 0, one GPU only).

With N > 1 (torchrun) every rank runs an independent replica on its own GPU
(the block has no cross-sequence exchange): weak scaling, value = rows of all
ranks / max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "H3 block fwd packed rows/s @32k rows (bf16, W8A8) at 1 B200; % tensor peak"
UNIT = "rows/s"
PROFILES = os.path.join(ROOT, "profiles")
# the library's kernel launches per block forward: tile summary, pre-norm,
# rotary table, QKV GEMM, attention, out-projection GEMM, pre-norm, FFN up,
# FFN down (bf16); W8A8 adds the modulation rearrangement and the two
# standalone rotate + quantise passes; block-sparse adds pooling and selection
LAUNCHES_BF16 = 9
LAUNCHES_W8A8 = 12
KERNEL_SOURCES = {  # interval name -> source file of its kernel (traffic records are tied to it)
    "attention": "joint_video_audio_b200/csrc/attn.cu",
    "qkv_gemm": "joint_video_audio_b200/csrc/gemm.cu",
    "out_proj_gemm": "joint_video_audio_b200/csrc/gemm.cu",
    "ffn_up_gemm": "joint_video_audio_b200/csrc/gemm.cu",
    "ffn_down_gemm": "joint_video_audio_b200/csrc/gemm.cu",
    "norm1": "joint_video_audio_b200/csrc/norm_quant.cu",
    "norm2": "joint_video_audio_b200/csrc/norm_quant.cu",
}


# --------------------------------------------------------------------------- distributed plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def init_dist(backend):
    import datetime

    import torch.distributed as dist
    ws, rank, _ = dist_env()
    if ws > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return ws, rank


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def aggregate_throughput(rows_per_rank: int, steps: int, world: int, max_seconds: float) -> float:
    """Weak scaling: every rank processes `rows_per_rank` rows per step."""
    return rows_per_rank * steps * world / max_seconds


# --------------------------------------------------------------------------- helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d.get("hbm_gbs"), "bf16_tflops": d.get("bf16_tflops"),
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def source_sha(rel):
    with open(os.path.join(ROOT, rel), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(interval, workload):
    """DRAM bytes per launch from a committed ncu summary, if its recorded
    kernel-source hash still matches the current source (else None)."""
    src = KERNEL_SOURCES.get(interval)
    if not src or not os.path.isdir(PROFILES):
        return None
    sha = source_sha(src)
    for fn in sorted(os.listdir(PROFILES)):
        if not fn.endswith(".md"):
            continue
        txt = open(os.path.join(PROFILES, fn)).read()
        for m in re.finditer(r"traffic\s+interval=(\w+)\s+workload=(\S+)\s+source_sha=(\w+)\s+dram_bytes_per_launch=(\d+)", txt):
            if m.group(1) == interval and m.group(2) == workload and m.group(3) == sha:
                return int(m.group(4))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), float(f[3]) if f[3] not in ("[N/A]", "N/A") else 0.0, f[5:9]))
            except ValueError:
                continue
        os.remove(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [r for r in rows if r[2] > 300.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded),
                "power_w_median": statistics.median(r[2] for r in loaded), "power_w_max": max(r[2] for r in loaded)}


def attention_flops(dims, layout):
    """4 H D sum over documents of (rows in the document)^2: masked-out work is
    not counted."""
    import numpy as np
    n_pad = int((layout.tag == -1).sum())
    n_val = layout.n - n_pad
    return 4.0 * dims.heads * dims.head_dim * (float(n_val) ** 2 + float(n_pad) ** 2)


def gemm_flops(dims, n):
    C, HD, F = dims.hidden, dims.heads * dims.head_dim, dims.ffn
    return {"qkv_gemm": 2.0 * n * C * 3 * HD, "out_proj_gemm": 2.0 * n * HD * C,
            "ffn_up_gemm": 2.0 * n * C * 2 * F, "ffn_down_gemm": 2.0 * n * F * C}


def hbm_bytes(dims, n, quant):
    """Algorithmic DRAM bytes of the bandwidth-bound kernels (one launch)."""
    C, HD, F = dims.hidden, dims.heads * dims.head_dim, dims.ffn
    if quant:
        return {"norm1": n * (2 * C + C + 4), "norm2": n * (2 * C + C + 4),
                "quant_o": n * (2 * HD + HD + 4), "quant_a": n * (2 * F + F + 4)}
    return {"norm1": n * 4 * C, "norm2": n * 4 * C}


# --------------------------------------------------------------------------- GPU arm

def measure_int8_peak(torch, device):
    """Dense int8 tensor throughput of the library GEMM (torch._int_mm) at
    8192^3, best of 10, as the INT8 roofline denominator."""
    try:
        a = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=device)
        b = torch.randint(-127, 128, (8192, 8192), dtype=torch.int8, device=device).t()
        for _ in range(3):
            torch._int_mm(a, b)
        best = 1e9
        for _ in range(10):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            torch._int_mm(a, b)
            e.record()
            e.synchronize()
            best = min(best, s.elapsed_time(e) / 1e3)
        del a, b
        return {"tops": 2.0 * 8192 ** 3 / best / 1e12,
                "source": "int8 burst: torch._int_mm 8192^3, best of 10, measured in this run"}
    except Exception as ex:  # noqa: BLE001
        print(f"int8 peak measurement failed: {ex}", file=sys.stderr)
        return None


class WeightCache:
    """Host and device copies of the block weights, drawn once per weight
    shape (every real-dimension workload shares them: same dims, same seed)."""

    def __init__(self, torch, j, hi, device):
        self.torch, self.j, self.hi, self.device = torch, j, hi, device
        self.host, self.dev = {}, {}

    @staticmethod
    def _key(dims):
        return (dims.hidden, dims.heads, dims.head_dim, dims.ffn)

    def inputs(self, dims, lay):
        k = self._key(dims)
        if k not in self.host:
            self.host[k] = self.hi.make_weights(dims)
        return self.hi.Inputs(dims, lay, self.hi.make_x(dims, lay.n), self.hi.make_table(dims), self.host[k])

    def device_weights(self, inp, blk):
        k = self._key(inp.dims) + (int(inp.dims.quant),)
        if k not in self.dev:
            if k[:4] + (0,) not in self.dev:
                self.dev[k[:4] + (0,)] = self.j.DeviceWeights.from_host(inp.weights, self.device)
            if inp.dims.quant:
                self.dev[k] = blk.prepare_int8(self.dev[k[:4] + (0,)])
        return self.dev[k]


def run_gpu_case(torch, j, hi, name, steps, warmup, device, peaks, int8_peak, clocks=None, e2e=False, density=1.0,
                 cache=None):
    from joint_video_audio_b200 import _binding as B
    dims, lay = hi.workload(name)
    cache = cache or WeightCache(torch, j, hi, device)
    inp = cache.inputs(dims, lay)
    n = lay.n
    x = inp.x.to(device)
    tag, tidx, pos = inp.tag.to(device), inp.tidx.to(device), inp.pos.to(device).contiguous()
    table = inp.table.to(device)
    blk = j.H3Block(dims)
    if density < 1.0:
        blk.set_attention_density(density)
    w = cache.device_weights(inp, blk)
    ws = blk.workspace(n, device)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream(device)

    def step():
        blk.forward(x, tag, tidx, pos, table, w, out=out, workspace=ws)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    if blk.check(ws, n) != 0:
        raise RuntimeError(f"{name}: device error word set after warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(B.H3BLK_TIMING_POINTS)] for _ in range(steps)]
    for row in ev:  # torch creates the underlying cudaEvent_t on first record
        for e in row:
            e.record(stream)
    barrier(device)
    torch.cuda.synchronize(device)
    if clocks:
        clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        B.h3blk_set_kernel_events(blk.handle, [e.cuda_event for e in ev[i]])
        step()
    t1.record(stream)
    torch.cuda.synchronize(device)
    clk = clocks.stop() if clocks else None
    barrier(device)
    B.h3blk_set_kernel_events(blk.handle, None)
    secs = t0.elapsed_time(t1) / 1e3
    secs_max = max_over_ranks(secs, device)
    kernels = {}
    for k, nm in enumerate(B.TIMING_INTERVALS):
        ms = [ev[i][k].elapsed_time(ev[i][k + 1]) for i in range(steps)]
        kernels[nm] = {"ms": statistics.mean(ms)}
    step_ms = sum(v["ms"] for v in kernels.values())
    for v in kernels.values():
        v["share"] = v["ms"] / step_ms if step_ms > 0 else None
    fl = gemm_flops(dims, n)
    fl["attention"] = attention_flops(dims, lay)
    bt = hbm_bytes(dims, n, dims.quant)
    # Kernels are timed one launch at a time inside a step of tens of
    # milliseconds, so the burst peaks apply; the sustained bf16 fraction is
    # kept beside them.
    tens_peak = peaks["bf16_tflops"]
    i8_peak = int8_peak["tops"] if int8_peak else None
    for nm, v in kernels.items():
        if nm in fl and v["ms"] > 0:
            v["tflops"] = fl[nm] / (v["ms"] / 1e3) / 1e12
            p = (i8_peak if (dims.quant and nm != "attention") else tens_peak)
            v["frac_of_peak"] = v["tflops"] / p if p else None
            if not (dims.quant and nm != "attention"):
                v["frac_of_sustained"] = v["tflops"] / peaks["bf16_tflops_sustained"]
        if nm in bt and v["ms"] > 0:
            v["gbs"] = bt[nm] / (v["ms"] / 1e3) / 1e9
            v["frac_of_peak"] = v["gbs"] / peaks["hbm_gbs"]
    dominant = max((k for k in kernels if k in fl or k in bt), key=lambda k: kernels[k]["ms"])
    d = kernels[dominant]
    if dominant in fl:
        quant_gemm = dims.quant and dominant != "attention"
        roof = {"kernel": dominant, "bound": "tensor", "achieved": d["tflops"],
                "peak": i8_peak if quant_gemm else tens_peak, "unit": "TOPS" if quant_gemm else "TFLOP/s",
                "peak_kind": (int8_peak["source"] if quant_gemm else f"bf16 burst, of {peaks['source']}")}
    else:
        roof = {"kernel": dominant, "bound": "hbm", "achieved": d["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_kind": f"hbm copy, of {peaks['source']}"}
    roof["frac"] = roof["achieved"] / roof["peak"] if roof["peak"] else None
    roof["traffic"] = recorded_traffic(dominant, name)
    ideal_s = sum(fl[k] / ((i8_peak if (dims.quant and k != "attention") else tens_peak) * 1e12)
                  for k in fl) + sum(bt.values()) / (peaks["hbm_gbs"] * 1e9)
    res = {"workload": name, "n_rows": n, "n_valid": lay.n_valid, "n_pad": lay.n_pad,
           "seconds": secs_max, "ms_per_step": secs_max / steps * 1e3,
           "block_frac_of_ideal": ideal_s / (secs_max / steps),
           "value": aggregate_throughput(n, steps, int(os.environ.get("WORLD_SIZE", "1")), secs_max),
           "kernels": kernels, "roofline": roof, "clocks": clk,
           "gpu_launches": steps * (LAUNCHES_W8A8 if dims.quant else LAUNCHES_BF16) + steps * (2 if density < 1.0 else 0)}
    if density < 1.0:
        # work actually done: the kept (query tile, key tile) pairs
        lists = blk.stage(ws, n, "KV_LIST")
        kept = int(lists[:, :, 0].sum().item())
        total = lists.shape[0] * lists.shape[1] * sum(1 for t in range(lists.shape[2] - 1)
                                                       if lay.tag[t * 128:(t + 1) * 128].max() >= 0)
        kept_flops = kept * 2 * 4 * 128 * 128 * dims.head_dim
        a = kernels["attention"]
        res["sparse"] = {"density": density, "kept_tile_fraction": kept / total,
                         "attention_ms": a["ms"], "kept_tflops": kept_flops / (a["ms"] / 1e3) / 1e12,
                         "dense_equivalent_tflops": a.get("tflops")}
    if e2e:
        res["e2e"] = run_e2e(torch, blk, inp, w, ws, steps, warmup, device)
    del ws, w, out, x
    torch.cuda.empty_cache()
    return res


def compact_kernels(kernels):
    """{interval: [ms, fraction of its roofline]} with 4 significant digits."""
    return {k: [float(f"{v['ms']:.4g}"), (float(f"{v['frac_of_peak']:.3g}") if v.get("frac_of_peak") else None)]
            for k, v in kernels.items() if k != "prep"}


def run_e2e(torch, blk, inp, w, ws, steps, warmup, device):
    """Same C-ABI call, with every step's inputs copied in from pinned host
    memory and its block output copied back to pinned host memory, all inside
    the timed region. As a serving loop would, the copies run on their own
    streams, double-buffered, so step i+1's upload and step i-1's download
    overlap step i's compute; every step still moves all of its bytes."""
    hx = inp.x.pin_memory()
    htag, htidx, hpos = inp.tag.pin_memory(), inp.tidx.pin_memory(), inp.pos.contiguous().pin_memory()
    htable = inp.table.pin_memory()
    hins = (hx, htag, htidx, hpos, htable)
    houts = [torch.empty_like(inp.x).pin_memory() for _ in range(2)]
    dins = [[torch.empty_like(t, device=device) for t in hins] for _ in range(2)]
    douts = [torch.empty_like(hx, device=device) for _ in range(2)]
    s_h2d, s_cmp, s_d2h = (torch.cuda.Stream(device) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    started = [False, False]

    def step(i):
        b = i % 2
        with torch.cuda.stream(s_h2d):
            if started[b]:
                s_h2d.wait_event(ev_cmp[b])      # step i-2 finished reading buffer b
            for d, h in zip(dins[b], hins):
                d.copy_(h, non_blocking=True)
            ev_in[b].record(s_h2d)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[b])
            if started[b]:
                s_cmp.wait_event(ev_out[b])      # step i-2's output has left the device
            x, tag, tidx, pos, table = dins[b]
            blk.forward(x, tag, tidx, pos, table, w, out=douts[b], workspace=ws)
            ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_d2h):
            s_d2h.wait_event(ev_cmp[b])
            houts[b].copy_(douts[b], non_blocking=True)
            ev_out[b].record(s_d2h)
        started[b] = True

    for i in range(max(1, warmup)):
        step(i)
    torch.cuda.synchronize(device)
    barrier(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_h2d)
    s_cmp.wait_event(t0)
    s_d2h.wait_event(t0)
    for i in range(steps):
        step(i)
    s_d2h.wait_stream(s_cmp)
    t1.record(s_d2h)
    torch.cuda.synchronize(device)
    secs = max_over_ranks(t0.elapsed_time(t1) / 1e3, device)
    assert torch.equal(houts[(steps - 1) % 2], douts[(steps - 1) % 2].cpu())
    h2d = sum(t.numel() * t.element_size() for t in hins)
    d2h = houts[0].numel() * houts[0].element_size()
    n = inp.layout.n
    return {"value": aggregate_throughput(n, steps, int(os.environ.get("WORLD_SIZE", "1")), secs), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": secs / steps * 1e3,
            "overlap": "uploads, compute and downloads on three streams, double-buffered"}


def run_modulation(torch, j, hi, device, peaks, steps):
    """The modulation-table producer at real dimensions with two-time
    conditioning (4 timestep sets, 4 modality tags): device time per call and
    achieved HBM bandwidth over the bytes it must stream (every weight once,
    the table written once)."""
    from dataclasses import replace
    dims, md = replace(hi.REAL, n_t=4), hi.REAL_MOD
    p = hi.make_modulation_params(dims, md, two_time=True)
    t_now, t_end = hi.two_time_sets([0.83, 0.41], [0.55, 0.12])
    blk = j.H3Block(dims)
    w = j.ModulationWeights(p, device)
    for _ in range(3):
        j.modulation_table(blk, w, t_now, t_end, 0.35)
    torch.cuda.synchronize(device)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(steps):
        j.modulation_table(blk, w, t_now, t_end, 0.35)
    t1.record()
    torch.cuda.synchronize(device)
    ms = t0.elapsed_time(t1) / steps
    mlp = 4 * (md.time_hidden * md.freq_dim + md.time_hidden + md.time_dim * md.time_hidden + md.time_dim)
    nbytes = 2 * mlp + dims.n_tags * 6 * dims.hidden * (2 * md.time_dim + 4) + 4 * dims.n_tags * 4 * 6 * dims.hidden
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"ms": ms, "bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / peaks["hbm_gbs"],
            "config": "real dims, 4 tags x 4 two-time sets, freq 256 -> 5376 -> 2688 -> 6 x 5376"}


def run_model(torch, j, hi, device, steps, warmup, quant):
    """The whole transformer forward (input projections, 2 token-refiner
    blocks over the text rows, the block stack, norm_out and both heads) at real
    dimensions on the 32k layout, replayed as one CUDA graph: 50 bf16 layers,
    or 47 rotated-W8A8 layers with two-time conditioning. Random weights drawn
    on the device. Also times the same graph without the stack (the shell)."""
    from dataclasses import replace
    if quant:
        dims = replace(hi.REAL, n_t=4, quant=1)
        lay = hi.layout_two_time(hi.layout_t2va_32k())
        sd = replace(hi.REAL_SHELL, n_layers=47)
    else:
        dims, lay, sd = hi.REAL, hi.layout_t2va_32k(), hi.REAL_SHELL
    params = hi.make_model_params_device(dims, hi.REAL_MOD, sd, two_time=bool(quant), device=device)
    m = j.Model(dims, sd)
    dm = m.load(params, device)
    del params
    mi = hi.make_model_inputs(dims, sd, lay, two_time=bool(quant))
    di = j.DeviceInputs.from_model_inputs(mi, device)
    vo, ao, ws = m.buffers(dm, di)
    g = m.graph(dm, di, vo, ao, ws)
    shell = j.Model(dims, replace(sd, n_layers=0))
    g0 = shell.graph(dm, di, vo, ao, ws)

    def timed(graph, n):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for a, b in ev:
            a.record()
            graph.launch()
            b.record()
        torch.cuda.synchronize(device)
        return [a.elapsed_time(b) for a, b in ev]

    timed(g, warmup)
    ms = statistics.mean(timed(g, steps))
    status = j.Model.check(ws)
    timed(g0, 3)
    shell_ms = statistics.mean(timed(g0, 5))
    kern, other = g.nodes
    out = {"workload": lay.name, "layers": sd.n_layers, "refiner_layers": sd.n_refiner,
           "mode": "w8a8" if quant else "bf16", "n_rows": lay.n, "ms_per_forward": ms,
           "rows_per_s": lay.n / (ms / 1e3), "shell_ms": shell_ms,
           "ms_per_layer": (ms - shell_ms) / max(1, sd.n_layers), "graph_kernels": kern,
           "graph_other_nodes": other, "gpu_launches": kern * steps, "steps": steps, "warmup": warmup,
           "status": status,
           "weights_gb": round(dm.nbytes() / 1e9, 1)}
    del g, g0, dm, di, vo, ao, ws
    torch.cuda.empty_cache()
    return out


# --------------------------------------------------------------------------- CPU oracle arm

def cpu_oracle_sample(name="t2va_32k", kv_rows=1024, q_rows=8, seed=0):
    """Times the fp64 oracle on a bounded sample of the workload and
    extrapolates to the full block: k/v projection of `kv_rows` rows (linear in
    rows) and the rest of the block for `q_rows` query rows attending to all N
    keys. Returns (rows_per_second, seconds_of_sample, description, threads)."""
    import numpy as np

    import h3_inputs as hi
    from oracle.h3_block import BlockOracle, documents
    dims, lay = hi.workload(name)
    inp = hi.make_inputs(dims, lay, seed=seed)
    ob = BlockOracle(dims, inp.weights)
    n = lay.n
    x = inp.x[:kv_rows]
    t0 = time.perf_counter()
    k_s, v_s = ob.kv_all(x, lay.tag[:kv_rows], lay.tidx[:kv_rows], lay.pos[:kv_rows], inp.table)
    t_kv = time.perf_counter() - t0
    k_all = np.resize(k_s, (n,) + k_s.shape[1:])
    v_all = np.resize(v_s, (n,) + v_s.shape[1:])
    rows = hi.sample_rows(lay, k=q_rows, k_pad=0, seed=seed)
    t0 = time.perf_counter()
    ob.query(inp.x[rows], lay.tag[rows], lay.tidx[rows], lay.pos[rows], inp.table, k_all, v_all, documents(lay.tag))
    t_q = time.perf_counter() - t0
    t_full = n * (t_kv / kv_rows) + n * (t_q / q_rows)
    try:
        from threadpoolctl import threadpool_info
        threads = max((p.get("num_threads", 1) for p in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        threads = os.cpu_count()
    desc = (f"fp64 oracle on {name}: k/v projection of {kv_rows} of {n} rows and the rest of the block for "
            f"{q_rows} query rows attending to all {n} keys; full-block time extrapolated linearly in rows")
    return n / t_full, t_kv + t_q, desc, threads


# --------------------------------------------------------------------------- main

def headline_config(hi, workload, world):
    """The `config` object of the JSON line; both arms print the same one."""
    dims, lay = hi.workload(workload)
    return {"workload": workload, "n_rows": lay.n, "n_valid": lay.n_valid, "hidden": dims.hidden,
            "heads": dims.heads, "head_dim": dims.head_dim, "ffn": dims.ffn, "parallelism": f"replicas x{world}",
            "flush": "none: inputs (352 MB) and weights (771 MB) exceed the 126 MB L2"}


def r4(v):
    return float(f"{v:.4g}") if isinstance(v, (int, float)) and v is not None else v


def extra(name, obj):
    """Secondary results, one plain-text line each, printed before the JSON
    line so that the JSON line is the last line of the output."""
    print(f"extra {name}: " + json.dumps(obj), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="t2va_32k")
    ap.add_argument("--no-w8a8", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip real_8k, the padded 32k and ref2va_54k legs")
    ap.add_argument("--no-model", action="store_true", help="skip the whole-model forward legs")
    ap.add_argument("--no-sparse", action="store_true", help="skip the block-sparse attention leg")
    args = ap.parse_args()
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"
    ws_, rank, local = dist_env()
    import h3_inputs as hi

    if args.impl == "reference":
        if rank != 0:
            return
        per_step, rates = [], []
        desc = threads = None
        for i in range(args.warmup + args.steps):
            rps, secs, desc, threads = cpu_oracle_sample(args.workload, kv_rows=512, q_rows=4)
            if i >= args.warmup:
                per_step.append(secs)
                rates.append(rps)
        value = statistics.mean(rates)
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(per_step) * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": headline_config(hi, args.workload, ws_),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    import torch
    backend = "nccl"
    world, rank = init_dist(backend)
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    import joint_video_audio_b200 as j
    peaks = load_peaks()
    int8_peak = measure_int8_peak(torch, device)
    cache = WeightCache(torch, j, hi, device)
    main_res = run_gpu_case(torch, j, hi, args.workload, args.steps, args.warmup, device, peaks, int8_peak,
                            clocks=ClockSampler(local), e2e=not args.no_e2e, cache=cache)
    w8 = None
    if not args.no_w8a8:
        w8 = run_gpu_case(torch, j, hi, "w8a8_t2va_32k", args.steps, args.warmup, device, peaks, int8_peak,
                          clocks=ClockSampler(local), e2e=not args.no_e2e, cache=cache)
    others = {}
    if not args.no_configs:
        for name in ("real_8k", "t2va_32k_pad168", "ref2va_54k"):
            others[name] = run_gpu_case(torch, j, hi, name, args.steps, args.warmup, device, peaks, int8_peak,
                                        clocks=ClockSampler(local), cache=cache)
    sparse = None
    if not args.no_sparse:
        sp = run_gpu_case(torch, j, hi, args.workload, args.steps, args.warmup, device, peaks, int8_peak,
                          density=0.25, cache=cache)
        sparse = {"workload": sp["workload"], "value": sp["value"], "unit": UNIT, "ms_per_step": sp["ms_per_step"],
                  **sp["sparse"], "gpu_launches": sp["gpu_launches"]}
    del cache
    torch.cuda.empty_cache()
    modt = run_modulation(torch, j, hi, device, peaks, args.steps)
    models = []
    if not args.no_model:
        for q in (0, 1):
            models.append(run_model(torch, j, hi, device, min(args.steps, 3), 3, q))
    cpu = cpu8 = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rps, secs, desc, threads = cpu_oracle_sample(args.workload)
        cpu = {"value": rps, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
               "sample_seconds": secs}
        if w8:
            rps, secs, desc, threads = cpu_oracle_sample("w8a8_t2va_32k")
            cpu8 = {"value": rps, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc,
                    "sample_seconds": secs}
    if rank == 0:
        # full detail first, as plain-text lines
        extra("bf16_kernels", main_res["kernels"])
        if w8:
            extra("w8a8", {k: w8.get(k) for k in ("workload", "value", "ms_per_step", "roofline", "kernels", "clocks",
                                                   "e2e", "gpu_launches", "block_frac_of_ideal")} | {"cpu_baseline": cpu8})
        for name, r in others.items():
            extra(name, {k: r[k] for k in ("n_rows", "n_valid", "n_pad", "value", "ms_per_step", "roofline",
                                           "kernels", "clocks", "gpu_launches", "block_frac_of_ideal")})
        if sparse:
            extra("sparse_attention", sparse)
        extra("modulation_table", modt)
        for m in models:
            extra(f"model_forward_{m['mode']}", m)
        extra("peaks", {"bf16_burst_tflops": peaks["bf16_tflops"], "bf16_sustained_tflops": peaks["bf16_tflops_sustained"],
                        "hbm_gbs": peaks["hbm_gbs"], "source": peaks["source"], "int8": int8_peak})
        # the JSON line: compact, so that it fits whole in a short log tail
        roof = {k: r4(v) for k, v in main_res["roofline"].items()}
        line = {"metric": METRIC, "value": main_res["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": main_res["ms_per_step"], "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": headline_config(hi, args.workload, world),
                "roofline": roof, "cpu_baseline": cpu, "e2e": main_res.get("e2e"),
                "gpu_launches": main_res["gpu_launches"], "clocks": main_res["clocks"],
                "block_frac_of_ideal": r4(main_res["block_frac_of_ideal"]),
                "kernels_ms_frac": compact_kernels(main_res["kernels"])}
        if w8:
            line["w8a8"] = {"workload": w8["workload"], "value": r4(w8["value"]), "ms_per_step": r4(w8["ms_per_step"]),
                            "e2e_value": r4(w8["e2e"]["value"]) if w8.get("e2e") else None,
                            "block_frac_of_ideal": r4(w8["block_frac_of_ideal"]),
                            "roofline": {k: r4(v) for k, v in w8["roofline"].items() if k != "peak_kind"},
                            "clocks_sm_mhz": (w8["clocks"] or {}).get("sm_mhz"),
                            "clocks_reasons": (w8["clocks"] or {}).get("reasons"),
                            "cpu_baseline_value": r4(cpu8["value"]) if cpu8 else None,
                            "kernels_ms_frac": compact_kernels(w8["kernels"])}
        if others:
            line["configs"] = {name: {"value": r4(r["value"]), "ms_per_step": r4(r["ms_per_step"]),
                                      "attention_frac": r4(r["kernels"]["attention"].get("frac_of_peak")),
                                      "block_frac_of_ideal": r4(r["block_frac_of_ideal"])}
                               for name, r in others.items()}
        line["int8_peak_tops"] = r4(int8_peak["tops"]) if int8_peak else None
        print(json.dumps(line), flush=True)
    import torch.distributed as dist
    if dist.is_initialized():
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
