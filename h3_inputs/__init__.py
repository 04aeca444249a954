"""Seeded synthetic inputs for one MiniMax-H3 transformer block.

This module is shared by the CPU oracle (``oracle/``), the tests and the
benchmark. It holds no arithmetic of the block itself: only the dimensions,
the packed row layouts (modality tag, timestep index and (t, h, w) rotary
position per row) and seeded random tensors of the stated distributions.

Where the layouts come from:

* "MiniMaxH3Transformer3DModel" (diffusers API page), introduction: one packed
  1-D sequence of text, conditioning image/video, audio and target-video rows;
  padding rows carry tag -1 and form their own attention document.
* Same page, ``forward`` parameters: per-row ``token_tags``,
  ``timestep_indices`` and ``position_ids`` of shape (seq_len, 3).
* Same page, constructor parameters: hidden 5376, 56 heads of 128, ffn 14336,
  rope_theta 1e4, norm_eps and qk_norm_eps 1e-5.
* The t2va geometry (124 frames at 1344x768 -> a 31 x 24 x 42 latent grid of
  2x2 patches) follows the diffusers MiniMax-H3 pipeline page, memory section.

Values: x ~ N(0, 1); every weight ~ N(0, 1/fan_in); modulation table ~
N(0, 0.1^2); per-head norm gains 1 + N(0, 0.1^2). Everything is drawn in fp32 with
``numpy.random.default_rng(seed)`` and rounded to bf16 where the block stores
bf16 (x, weights, gains). The modulation table stays fp32.
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

TAG_PAD = -1


@dataclass(frozen=True)
class Dims:
    hidden: int
    heads: int
    head_dim: int
    ffn: int
    n_tags: int
    n_t: int
    rope_pairs: tuple  # (t, h, w) rotary pairs; the remaining head_dim/2 pairs pass through
    rope_theta: float = 10000.0
    norm_eps: float = 1e-5
    qk_norm_eps: float = 1e-5
    quant: int = 0  # 0: bf16 linears, 1: rotated W8A8 linears

    @property
    def hd(self) -> int:
        return self.heads * self.head_dim


TINY = Dims(hidden=256, heads=6, head_dim=64, ffn=768, n_tags=4, n_t=2, rope_pairs=(8, 12, 12))
REAL = Dims(hidden=5376, heads=56, head_dim=128, ffn=14336, n_tags=4, n_t=2, rope_pairs=(16, 24, 24))


@dataclass
class Layout:
    """Per-row structure of one packed sequence."""
    name: str
    tag: np.ndarray    # int32 [N], -1 = padding
    tidx: np.ndarray   # int32 [N]
    pos: np.ndarray    # int32 [N, 3] (t, h, w)
    segments: list = field(default_factory=list)  # (label, start, count)

    @property
    def n(self) -> int:
        return int(self.tag.shape[0])

    @property
    def n_valid(self) -> int:
        return int((self.tag != TAG_PAD).sum())

    @property
    def n_pad(self) -> int:
        return self.n - self.n_valid


class _Builder:
    """Appends row segments in sequence order."""

    def __init__(self, name):
        self.name = name
        self.tags, self.tidx, self.pos, self.segments = [], [], [], []
        self.n = 0

    def add(self, label, tag, tidx, pos):
        pos = np.asarray(pos, dtype=np.int32).reshape(-1, 3)
        k = pos.shape[0]
        tidx = np.broadcast_to(np.asarray(tidx, dtype=np.int32), (k,))
        self.tags.append(np.full(k, tag, dtype=np.int32))
        self.tidx.append(np.array(tidx, dtype=np.int32))
        self.pos.append(pos)
        self.segments.append((label, self.n, k))
        self.n += k

    def build(self) -> Layout:
        return Layout(self.name, np.concatenate(self.tags), np.concatenate(self.tidx),
                      np.concatenate(self.pos), self.segments)


def text_positions(n):
    i = np.arange(n, dtype=np.int32)
    return np.stack([i, i, i], axis=1)


def audio_positions(n, t0=0):
    j = np.arange(n, dtype=np.int32) + t0
    z = np.zeros(n, dtype=np.int32)
    return np.stack([j, z, z], axis=1)


def grid_positions(t, h, w, t0=0):
    tt, hh, ww = np.meshgrid(np.arange(t) + t0, np.arange(h), np.arange(w), indexing="ij")
    return np.stack([tt.ravel(), hh.ravel(), ww.ravel()], axis=1).astype(np.int32)


def pad_positions(n):
    return np.zeros((n, 3), dtype=np.int32)


def _round_up(n, m):
    return (n + m - 1) // m * m


# Tag numbering used by every measured layout: 0 text, 1 conditioning
# (image / video references), 2 audio, 3 target video. A tag is only an index
# into the modulation table.
TAG_TEXT, TAG_COND, TAG_AUDIO, TAG_VIDEO = 0, 1, 2, 3


def layout_tiny(seed=0) -> Layout:
    """320 rows: 64 text, 32 audio, 192 video on a (3, 8, 8) grid, 32 padding.
    Per-row timestep index drawn uniformly from {0, 1}."""
    b = _Builder("tiny_320")
    b.add("text", TAG_TEXT, 0, text_positions(64))
    b.add("audio", TAG_AUDIO, 0, audio_positions(32))
    b.add("video", TAG_VIDEO, 0, grid_positions(3, 8, 8))
    b.add("pad", TAG_PAD, 0, pad_positions(32))
    lay = b.build()
    rng = np.random.default_rng(seed + 1000)
    lay.tidx = rng.integers(0, 2, size=lay.n).astype(np.int32)
    return lay


def layout_t2va(n_text, n_audio, grid, pad_to=256, drop_video_tail=0, name=None) -> Layout:
    """Text, target audio, target video grid, then padding up to ``pad_to``.
    Video and text rows use timestep index 0, audio rows index 1."""
    t, h, w = grid
    b = _Builder(name or f"t2va_{n_text}+{n_audio}+{t}x{h}x{w}")
    b.add("text", TAG_TEXT, 0, text_positions(n_text))
    b.add("audio", TAG_AUDIO, 1, audio_positions(n_audio))
    vid = grid_positions(t, h, w)
    if drop_video_tail:
        vid = vid[: vid.shape[0] - drop_video_tail]
    b.add("video", TAG_VIDEO, 0, vid)
    n = b.n
    npad = _round_up(n, pad_to) - n
    if drop_video_tail:
        npad = drop_video_tail
    if npad:
        b.add("pad", TAG_PAD, 0, pad_positions(npad))
    return b.build()


def layout_real_8k() -> Layout:
    """8192 padless rows: 512 text, 256 audio, 7424 video on a (29, 16, 16) grid."""
    return layout_t2va(512, 256, (29, 16, 16), name="real_8k")


def layout_t2va_32k() -> Layout:
    """32768 padless rows: 512 text, 1008 audio, 31248 video on (31, 24, 42):
    124 frames at 1344x768 after 4x temporal and 32x spatial reduction."""
    return layout_t2va(512, 1008, (31, 24, 42), name="t2va_32k")


def layout_t2va_32k_padded() -> Layout:
    """Variant of the 32k layout with 168 padding rows at the tail
    (V = 32600, P = 168): the last 168 video rows are replaced by padding."""
    return layout_t2va(512, 1008, (31, 24, 42), drop_video_tail=168, name="t2va_32k_pad168")


def layout_ref2va() -> Layout:
    """ref2va-shaped sequence: 512 text; 9 image references of 1x24x42 and
    3 video references of 4x24x42 (conditioning tag, timestep index 2);
    3 audio references of 128 rows (audio tag, index 2); 1008 target audio
    rows (index 1); a 31x24x42 target video grid (index 0); then padding to a
    multiple of 256. References advance one shared rotary time axis in order."""
    b = _Builder("ref2va_54k")
    b.add("text", TAG_TEXT, 0, text_positions(512))
    clock = 0
    for _ in range(9):
        b.add("image_ref", TAG_COND, 2, grid_positions(1, 24, 42, t0=clock))
        clock += 1
    for _ in range(3):
        b.add("video_ref", TAG_COND, 2, grid_positions(4, 24, 42, t0=clock))
        clock += 4
    for _ in range(3):
        b.add("audio_ref", TAG_AUDIO, 2, audio_positions(128, t0=clock))
        clock += 128
    b.add("audio", TAG_AUDIO, 1, audio_positions(1008))
    b.add("video", TAG_VIDEO, 0, grid_positions(31, 24, 42))
    npad = _round_up(b.n, 256) - b.n
    b.add("pad", TAG_PAD, 0, pad_positions(npad))
    return b.build()


def layout_two_time(base: Layout, seed=0) -> Layout:
    """Two-time conditioning: timestep index = 2 * t_now + t_end, with
    t_now, t_end drawn uniformly from {0, 1} per row (4 modulation sets)."""
    rng = np.random.default_rng(seed + 2000)
    t_now = rng.integers(0, 2, size=base.n)
    t_end = rng.integers(0, 2, size=base.n)
    return replace(base, name=base.name + "_twotime",
                   tidx=(2 * t_now + t_end).astype(np.int32))


# --------------------------------------------------------------------------
# Named workloads
# --------------------------------------------------------------------------

WORKLOADS = {
    "tiny_320": (TINY, layout_tiny),
    "real_8k": (REAL, layout_real_8k),
    "t2va_32k": (REAL, layout_t2va_32k),
    "t2va_32k_pad168": (REAL, layout_t2va_32k_padded),
    "ref2va_54k": (replace(REAL, n_t=3), layout_ref2va),
    "w8a8_t2va_32k": (replace(REAL, n_t=4, quant=1), lambda: layout_two_time(layout_t2va_32k())),
}


def workload(name, seed=0):
    dims, mk = WORKLOADS[name]
    lay = mk(seed) if name == "tiny_320" else mk()
    return dims, lay


# --------------------------------------------------------------------------
# Random tensors
# --------------------------------------------------------------------------

def _normal(rng, shape, std):
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        a *= np.float32(std)
    return a


def to_bf16(a: np.ndarray) -> torch.Tensor:
    """Round an fp32 array to bf16 (round to nearest even), as a CPU tensor."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


@dataclass
class Weights:
    wqkv: torch.Tensor   # bf16 [3*H*D, C]: rows q heads, then k heads, then v heads
    q_gain: torch.Tensor  # bf16 [D]
    k_gain: torch.Tensor  # bf16 [D]
    wo: torch.Tensor     # bf16 [C, H*D]
    w13: torch.Tensor    # bf16 [2F, C]: rows 0..F-1 = W1 (gate), F..2F-1 = W3 (up)
    w2: torch.Tensor     # bf16 [C, F]


def make_weights(dims: Dims, seed=0, unit_gains=False) -> Weights:
    rng = np.random.default_rng(seed + 10)
    C, HD, F, D = dims.hidden, dims.hd, dims.ffn, dims.head_dim
    wqkv = to_bf16(_normal(rng, (3 * HD, C), 1.0 / np.sqrt(C)))
    wo = to_bf16(_normal(rng, (C, HD), 1.0 / np.sqrt(HD)))
    w13 = to_bf16(_normal(rng, (2 * F, C), 1.0 / np.sqrt(C)))
    w2 = to_bf16(_normal(rng, (C, F), 1.0 / np.sqrt(F)))
    if unit_gains:
        qg = torch.ones(D, dtype=torch.bfloat16)
        kg = torch.ones(D, dtype=torch.bfloat16)
    else:
        qg = to_bf16(1.0 + _normal(rng, (D,), 0.1))
        kg = to_bf16(1.0 + _normal(rng, (D,), 0.1))
    return Weights(wqkv, qg, kg, wo, w13, w2)


def make_x(dims: Dims, n: int, seed=0) -> torch.Tensor:
    rng = np.random.default_rng(seed + 20)
    return to_bf16(_normal(rng, (n, dims.hidden), 1.0))


def make_table(dims: Dims, seed=0) -> torch.Tensor:
    """fp32 [n_tags][n_t][6][C]; the 6 vectors are shift1, scale1, gate1,
    shift2, scale2, gate2."""
    rng = np.random.default_rng(seed + 30)
    return torch.from_numpy(_normal(rng, (dims.n_tags, dims.n_t, 6, dims.hidden), 0.1))


@dataclass
class Inputs:
    dims: Dims
    layout: Layout
    x: torch.Tensor       # bf16 [N, C]
    table: torch.Tensor   # fp32 [n_tags, n_t, 6, C]
    weights: Weights

    @property
    def tag(self):
        return torch.from_numpy(self.layout.tag)

    @property
    def tidx(self):
        return torch.from_numpy(self.layout.tidx)

    @property
    def pos(self):
        return torch.from_numpy(self.layout.pos)


def make_inputs(name_or_dims, layout: Layout | None = None, seed=0, unit_gains=False) -> Inputs:
    if isinstance(name_or_dims, str):
        dims, layout = workload(name_or_dims, seed)
    else:
        dims = name_or_dims
    return Inputs(dims, layout, make_x(dims, layout.n, seed), make_table(dims, seed),
                  make_weights(dims, seed, unit_gains))


def sample_rows(layout: Layout, k=256, k_pad=8, seed=0) -> np.ndarray:
    """Seeded subset of rows used to compare against the oracle on large
    sequences: ``k`` non-padding rows plus up to ``k_pad`` padding rows."""
    rng = np.random.default_rng(seed + 40)
    valid = np.nonzero(layout.tag != TAG_PAD)[0]
    pad = np.nonzero(layout.tag == TAG_PAD)[0]
    rows = rng.choice(valid, size=min(k, valid.size), replace=False)
    if pad.size:
        rows = np.concatenate([rows, rng.choice(pad, size=min(k_pad, pad.size), replace=False)])
    return np.sort(rows).astype(np.int64)


# --------------------------------------------------------------------------
# Modulation-table producer (timestep embedding -> time MLP -> per-tag AdaLN)
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class ModDims:
    """Timestep embedding / MLP sizes ("MiniMaxH3Transformer3DModel",
    constructor: freq_dim, time_embed_hidden_dim, time_embed_dim)."""
    freq_dim: int = 256
    time_hidden: int = 5376
    time_dim: int = 2688


REAL_MOD = ModDims()
TINY_MOD = ModDims(freq_dim=64, time_hidden=128, time_dim=64)


@dataclass
class ModParams:
    md: ModDims
    w1: torch.Tensor      # fp32 [time_hidden, freq_dim]
    b1: torch.Tensor      # fp32 [time_hidden]
    w2: torch.Tensor      # fp32 [time_dim, time_hidden]
    b2: torch.Tensor      # fp32 [time_dim]
    w1_r: torch.Tensor | None   # second-time copy (two-time conditioning)
    b1_r: torch.Tensor | None
    w2_r: torch.Tensor | None
    b2_r: torch.Tensor | None
    adaln_w: torch.Tensor  # bf16 [n_tags, 6C, time_dim]
    adaln_b: torch.Tensor  # fp32 [n_tags, 6C]


def make_modulation_params(dims: Dims, md: ModDims, seed=0, two_time=False) -> ModParams:
    rng = np.random.default_rng(seed + 50)
    f = lambda a: torch.from_numpy(a)  # noqa: E731

    def mlp():
        return (f(_normal(rng, (md.time_hidden, md.freq_dim), 1.0 / np.sqrt(md.freq_dim))),
                f(_normal(rng, (md.time_hidden,), 0.02)),
                f(_normal(rng, (md.time_dim, md.time_hidden), 1.0 / np.sqrt(md.time_hidden))),
                f(_normal(rng, (md.time_dim,), 0.02)))
    w1, b1, w2, b2 = mlp()
    r = mlp() if two_time else (None, None, None, None)
    aw = to_bf16(_normal(rng, (dims.n_tags, 6 * dims.hidden, md.time_dim), 0.1 / np.sqrt(md.time_dim)))
    ab = f(_normal(rng, (dims.n_tags, 6 * dims.hidden), 0.02))
    return ModParams(md, w1, b1, w2, b2, *r, aw, ab)


def two_time_sets(t_now, t_end):
    """Per-set timesteps for the two-time table index 2 * i + j: set (i, j)
    pairs t_now[i] with t_end[j]."""
    tn = [t_now[i] for i in range(len(t_now)) for _ in range(len(t_end))]
    te = [t_end[j] for _ in range(len(t_now)) for j in range(len(t_end))]
    return np.asarray(tn, dtype=np.float32), np.asarray(te, dtype=np.float32)


# --------------------------------------------------------------------------
# Model shell around the block stack
# ("MiniMaxH3Transformer3DModel", constructor: num_layers, num_refiner_layers,
# in_channels x patch_size, audio_in_channels, text_dim, final_norm_eps;
# forward: video_indices, audio_indices, text_indices)
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class ShellDims:
    video_in: int = 96       # in_channels 24 x patch (1, 2, 2)
    audio_in: int = 32
    text_dim: int = 5120
    n_layers: int = 50
    n_refiner: int = 2
    final_norm_eps: float = 1e-5


REAL_SHELL = ShellDims()
TINY_SHELL = ShellDims(video_in=16, audio_in=8, text_dim=128, n_layers=2, n_refiner=1)


@dataclass
class Layer:
    """One block of the stack with its AdaLN projection."""
    w: Weights
    adaln_w: torch.Tensor   # bf16 [n_tags, 6C, time_dim]
    adaln_b: torch.Tensor   # fp32 [n_tags, 6C]


@dataclass
class ModelParams:
    sd: ShellDims
    time: ModParams             # time MLP; its adaln_w / adaln_b are not used by the model
    layers: list                # [Layer] * n_layers
    refiner: list               # [Layer] * n_refiner
    refiner_gain: torch.Tensor  # bf16 [C]
    out_adaln_w: torch.Tensor   # bf16 [n_tags, 2C, time_dim]
    out_adaln_b: torch.Tensor   # fp32 [n_tags, 2C]
    proj_in_w: torch.Tensor     # fp32 [C, video_in]
    proj_in_b: torch.Tensor     # fp32 [C]
    audio_in_w: torch.Tensor    # fp32 [C, audio_in]
    audio_in_b: torch.Tensor    # fp32 [C]
    ctx_w: torch.Tensor         # bf16 [C, text_dim]
    ctx_b: torch.Tensor         # fp32 [C]
    proj_out_w: torch.Tensor    # fp32 [video_in, C]
    proj_out_b: torch.Tensor    # fp32 [video_in]
    audio_out_w: torch.Tensor   # fp32 [audio_in, C]
    audio_out_b: torch.Tensor   # fp32 [audio_in]


def _adaln(rng, dims: Dims, md: ModDims, n_vec: int):
    aw = to_bf16(_normal(rng, (dims.n_tags, n_vec * dims.hidden, md.time_dim), 0.1 / np.sqrt(md.time_dim)))
    ab = torch.from_numpy(_normal(rng, (dims.n_tags, n_vec * dims.hidden), 0.02))
    return aw, ab


def make_model_params(dims: Dims, md: ModDims, sd: ShellDims, seed=0, two_time=False) -> ModelParams:
    """Every weight ~ N(0, 1/fan_in) (AdaLN projections 0.1/sqrt(fan_in)),
    biases N(0, 0.02^2), the refiner's output-norm gain 1 + N(0, 0.1^2)."""
    time = make_modulation_params(dims, md, seed, two_time)
    rng = np.random.default_rng(seed + 60)
    C = dims.hidden
    f = lambda a: torch.from_numpy(a)  # noqa: E731

    def layer(k):
        aw, ab = _adaln(rng, dims, md, 6)
        return Layer(make_weights(dims, seed + 1000 * (k + 1)), aw, ab)
    layers = [layer(k) for k in range(sd.n_layers)]
    refiner = [layer(100 + k) for k in range(sd.n_refiner)]
    oaw, oab = _adaln(rng, dims, md, 2)
    return ModelParams(
        sd, time, layers, refiner,
        refiner_gain=to_bf16(1.0 + _normal(rng, (C,), 0.1)),
        out_adaln_w=oaw, out_adaln_b=oab,
        proj_in_w=f(_normal(rng, (C, sd.video_in), 1.0 / np.sqrt(sd.video_in))),
        proj_in_b=f(_normal(rng, (C,), 0.02)),
        audio_in_w=f(_normal(rng, (C, sd.audio_in), 1.0 / np.sqrt(sd.audio_in))),
        audio_in_b=f(_normal(rng, (C,), 0.02)),
        ctx_w=to_bf16(_normal(rng, (C, sd.text_dim), 1.0 / np.sqrt(sd.text_dim))),
        ctx_b=f(_normal(rng, (C,), 0.02)),
        proj_out_w=f(_normal(rng, (sd.video_in, C), 1.0 / np.sqrt(C))),
        proj_out_b=f(_normal(rng, (sd.video_in,), 0.02)),
        audio_out_w=f(_normal(rng, (sd.audio_in, C), 1.0 / np.sqrt(C))),
        audio_out_b=f(_normal(rng, (sd.audio_in,), 0.02)))


def model_indices(layout: Layout):
    """(video, audio, text) row indices of a packed layout: video rows are the
    target-video and conditioning (image / video reference) rows, audio rows
    every audio-tagged row, text rows the text-tagged ones; padding rows are in
    none of them. Each list is in sequence order."""
    t = layout.tag
    video = np.nonzero((t == TAG_VIDEO) | (t == TAG_COND))[0].astype(np.int32)
    audio = np.nonzero(t == TAG_AUDIO)[0].astype(np.int32)
    text = np.nonzero(t == TAG_TEXT)[0].astype(np.int32)
    return video, audio, text


@dataclass
class ModelInputs:
    layout: Layout
    video_idx: np.ndarray   # int32 [Nv]
    audio_idx: np.ndarray   # int32 [Na]
    text_idx: np.ndarray    # int32 [Nt]
    video: torch.Tensor     # fp32 [Nv, video_in], patchified latent rows
    audio: torch.Tensor     # fp32 [Na, audio_in]
    text: torch.Tensor      # bf16 [Nt, text_dim], text-encoder states
    t_now: np.ndarray       # fp32 [n_t], per modulation set
    t_end: np.ndarray       # fp32 [n_t]
    gate: float


def make_model_inputs(dims: Dims, sd: ShellDims, layout: Layout, seed=0, two_time=False,
                      gate=0.35) -> ModelInputs:
    """Latent rows ~ N(0, 1), text states ~ N(0, 1) in bf16; timesteps drawn
    uniformly in [0, 1] per set (two-time: t_now pairs, t_end pairs, expanded
    to the 2 i + j sets)."""
    rng = np.random.default_rng(seed + 70)
    v, a, t = model_indices(layout)
    video = torch.from_numpy(_normal(rng, (v.size, sd.video_in), 1.0))
    audio = torch.from_numpy(_normal(rng, (a.size, sd.audio_in), 1.0))
    text = to_bf16(_normal(rng, (t.size, sd.text_dim), 1.0))
    if two_time:
        assert dims.n_t == 4
        tn, te = two_time_sets(rng.uniform(0, 1, 2).astype(np.float32), rng.uniform(0, 1, 2).astype(np.float32))
    else:
        tn = rng.uniform(0, 1, dims.n_t).astype(np.float32)
        te, gate = tn.copy(), 0.0
    return ModelInputs(layout, v, a, t, video, audio, text, tn, te, float(gate))


def make_model_params_device(dims: Dims, md: ModDims, sd: ShellDims, seed=0, two_time=False,
                             device="cuda") -> ModelParams:
    """The same distributions as make_model_params, drawn on the device with a
    seeded torch generator (not the same values): for timing full-size models
    whose weights would take minutes to draw on the host. Block weights come
    as h3_inputs.Weights of device tensors."""
    g = torch.Generator(device=device)
    g.manual_seed(seed + 80)
    C, HD, F, D, Td = dims.hidden, dims.hd, dims.ffn, dims.head_dim, md.time_dim

    def n(shape, std, dtype=torch.bfloat16, mean=0.0):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32 if dtype == torch.float32 else dtype)
        t.mul_(std)
        if mean:
            t.add_(mean)
        return t

    def mlp():
        return (n((md.time_hidden, md.freq_dim), 1.0 / np.sqrt(md.freq_dim), torch.float32),
                n((md.time_hidden,), 0.02, torch.float32),
                n((Td, md.time_hidden), 1.0 / np.sqrt(md.time_hidden), torch.float32),
                n((Td,), 0.02, torch.float32))

    def adaln(n_vec):
        return n((dims.n_tags, n_vec * C, Td), 0.1 / np.sqrt(Td)), n((dims.n_tags, n_vec * C), 0.02, torch.float32)

    def layer():
        w = Weights(n((3 * HD, C), 1.0 / np.sqrt(C)), n((D,), 0.1, mean=1.0), n((D,), 0.1, mean=1.0),
                    n((C, HD), 1.0 / np.sqrt(HD)), n((2 * F, C), 1.0 / np.sqrt(C)), n((C, F), 1.0 / np.sqrt(F)))
        return Layer(w, *adaln(6))

    w1, b1, w2, b2 = mlp()
    r = mlp() if two_time else (None, None, None, None)
    time = ModParams(md, w1, b1, w2, b2, *r, torch.zeros(1, 1, 1, dtype=torch.bfloat16, device=device),
                     torch.zeros(1, 1, device=device))
    layers = [layer() for _ in range(sd.n_layers)]
    refiner = [layer() for _ in range(sd.n_refiner)]
    oaw, oab = adaln(2)
    f32 = torch.float32
    return ModelParams(
        sd, time, layers, refiner, refiner_gain=n((C,), 0.1, mean=1.0), out_adaln_w=oaw, out_adaln_b=oab,
        proj_in_w=n((C, sd.video_in), 1.0 / np.sqrt(sd.video_in), f32), proj_in_b=n((C,), 0.02, f32),
        audio_in_w=n((C, sd.audio_in), 1.0 / np.sqrt(sd.audio_in), f32), audio_in_b=n((C,), 0.02, f32),
        ctx_w=n((C, sd.text_dim), 1.0 / np.sqrt(sd.text_dim)), ctx_b=n((C,), 0.02, f32),
        proj_out_w=n((sd.video_in, C), 1.0 / np.sqrt(C), f32), proj_out_b=n((sd.video_in,), 0.02, f32),
        audio_out_w=n((sd.audio_in, C), 1.0 / np.sqrt(C), f32), audio_out_b=n((sd.audio_in,), 0.02, f32))
