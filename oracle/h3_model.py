"""fp64 CPU oracle of the model shell around the block stack.

TEST INFRASTRUCTURE ONLY (same rules as oracle/h3_block.py): only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg may use it.

What the pages fix ("MiniMaxH3Transformer3DModel", diffusers API page):

* Introduction: modality-specific behaviour comes only from the two input
  patch projections, the per-row modality tag that selects the AdaLN
  parameters, and the two output heads; the patch projections, the timestep
  MLP and the two heads are float32, the block stack bfloat16.
* Constructor: num_layers blocks, num_refiner_layers token-refiner blocks on
  the projected text stream, in_channels x prod(patch_size) video inputs,
  audio_in_channels audio inputs, text_dim text states, final_norm_eps for the
  refiner's output norm and norm_out.
* forward: the video, audio and text rows arrive in the order of
  video_indices, audio_indices and text_indices (their positions in the packed
  sequence); the outputs are the video and audio velocities in that same order.

Readings taken where the pages are silent (listed in the design notes):

m1. Input projections are affine: proj_in(v) = W v + b (fp32),
    audio_proj_in likewise; context_embedder(e) = W e + b with a bf16 weight
    (it is not among the fp32 modules) and an fp32 bias.
m2. Packed rows that no index addresses (padding) start as zeros.
m3. A token-refiner layer is the same block as the stack's, applied to the
    text rows alone (one attention document of the text rows), each row keeping
    its packed-sequence tag, timestep index and (t, h, w) position, modulated by
    the refiner layer's own AdaLN projection; after the last refiner layer an
    RMSNorm (final_norm_eps) with a learned gain.
m4. Each layer of the stack (and of the refiner) owns its AdaLN projection:
    its table is produced from the shared time embedding as in
    oracle/h3_modulation.py.
m5. norm_out is an AdaLN RMSNorm, rmsnorm(x)(1 + scale) + shift, with
    (shift, scale) from a final per-tag projection of the time embedding (two
    vectors of C per tag and set, in that order); padding rows get zeros.
m6. The heads are affine fp32 maps of the normed rows gathered by
    video_indices / audio_indices: proj_out (C -> video_in), audio_proj_out
    (C -> audio_in).
"""
from __future__ import annotations

import numpy as np

from .h3_block import BlockOracle, f64, modulation, rmsnorm
from .h3_modulation import two_time_embedding, modulation_table


def affine(x, w, b):
    """y = x W^T + b over the rows of x."""
    return np.matmul(f64(x), f64(w).T) + f64(b)


def scatter_rows(n_rows, hidden, parts):
    """Packed [n_rows, hidden] sequence: rows idx of each (idx, values) part
    take those values; every other row is zero."""
    x = np.zeros((n_rows, hidden))
    for idx, vals in parts:
        x[np.asarray(idx, dtype=np.int64)] = vals
    return x


def time_embedding(p, t_now, t_end, gate):
    """Shared time embedding E [n_sets, time_dim] of the model's timestep sets."""
    tp = p.time
    mlp = (tp.w1, tp.b1, tp.w2, tp.b2)
    mlp_r = None if tp.w1_r is None else (tp.w1_r, tp.b1_r, tp.w2_r, tp.b2_r)
    return two_time_embedding(t_now, t_end, gate, mlp, mlp_r, tp.md.freq_dim)


def layer_table(E, adaln_w, adaln_b, n_vec):
    """[n_tags, n_sets, n_vec, C] table of one layer from its projection."""
    tab = modulation_table(E, adaln_w, adaln_b)
    n_tags, K, o = tab.shape
    return tab.reshape(n_tags, K, n_vec, o // n_vec)


def refine_text(dims, layers, tables, gain, eps, r, tag, tidx, pos):
    """Token refiner over the text rows alone (reading m3)."""
    from dataclasses import replace
    bdims = replace(dims, quant=0)
    for lay, tab in zip(layers, tables):
        r = BlockOracle(bdims, lay.w).forward(r, tag, tidx, pos, tab)["out"]
    return rmsnorm(f64(r), eps) * f64(gain)


def norm_out(x, table_o, tag, tidx, eps):
    """AdaLN RMSNorm with the final (shift, scale) table (reading m5)."""
    m = modulation(f64(table_o), np.asarray(tag), np.asarray(tidx))
    return rmsnorm(f64(x), eps) * (1.0 + m[:, 1]) + m[:, 0]


class ModelOracle:
    """Full forward: input projections, token refiner, packed assembly, the
    block stack, norm_out and the two heads. ``dims`` is the block's Dims (its
    quant applies to the stack only), ``p`` an h3_inputs.ModelParams."""

    def __init__(self, dims, p):
        self.d = dims
        self.p = p

    def tables(self, t_now, t_end, gate):
        E = time_embedding(self.p, t_now, t_end, gate)
        return {
            "E": E,
            "layers": [layer_table(E, L.adaln_w, L.adaln_b, 6) for L in self.p.layers],
            "refiner": [layer_table(E, L.adaln_w, L.adaln_b, 6) for L in self.p.refiner],
            "out": layer_table(E, self.p.out_adaln_w, self.p.out_adaln_b, 2),
        }

    def shell_in(self, mi, tabs):
        """Packed input sequence x0 (before the stack), fp64."""
        p, d, lay = self.p, self.d, mi.layout
        parts = [(mi.video_idx, affine(mi.video, p.proj_in_w, p.proj_in_b)),
                 (mi.audio_idx, affine(mi.audio, p.audio_in_w, p.audio_in_b))]
        if len(mi.text_idx):
            t = mi.text_idx
            r = affine(mi.text, p.ctx_w, p.ctx_b)
            r = refine_text(d, p.refiner, tabs["refiner"], p.refiner_gain, p.sd.final_norm_eps, r,
                            lay.tag[t], lay.tidx[t], lay.pos[t])
            parts.append((t, r))
        return scatter_rows(lay.n, d.hidden, parts)

    def heads(self, x, mi, tabs, rows=None):
        """Both heads. x holds every packed row, or only ``rows`` (sorted);
        then only the video / audio rows among them are returned, with their
        positions in video_idx / audio_idx."""
        p, lay = self.p, mi.layout
        rows = np.arange(lay.n) if rows is None else np.asarray(rows)
        at = {int(r): j for j, r in enumerate(rows)}
        h = norm_out(x, tabs["out"], lay.tag[rows], lay.tidx[rows], p.sd.final_norm_eps)
        vsel = np.array([i for i, r in enumerate(mi.video_idx) if int(r) in at], dtype=np.int64)
        asel = np.array([i for i, r in enumerate(mi.audio_idx) if int(r) in at], dtype=np.int64)
        hv = h[[at[int(r)] for r in mi.video_idx[vsel]]] if vsel.size else np.zeros((0, h.shape[1]))
        ha = h[[at[int(r)] for r in mi.audio_idx[asel]]] if asel.size else np.zeros((0, h.shape[1]))
        return (affine(hv, p.proj_out_w, p.proj_out_b), affine(ha, p.audio_out_w, p.audio_out_b), vsel, asel)

    def forward(self, mi, n_layers=None, rows=None):
        """Returns dict: video, audio (velocities, for the positions
        video_sel / audio_sel of the index tensors), x0 (packed input), x
        (stack output, of ``rows`` only when given) and the tables. With
        ``rows``, the last layer and the heads are evaluated for those packed
        rows only; every earlier layer needs all rows."""
        lay = mi.layout
        tabs = self.tables(mi.t_now, mi.t_end, mi.gate)
        x0 = self.shell_in(mi, tabs)
        x = x0
        L = len(self.p.layers) if n_layers is None else n_layers
        for k in range(L):
            sub = rows if k == L - 1 else None
            x = BlockOracle(self.d, self.p.layers[k].w).forward(x, lay.tag, lay.tidx, lay.pos,
                                                                tabs["layers"][k], rows=sub)["out"]
        if rows is not None and L == 0:
            x = x0[np.asarray(rows)]
        v, a, vsel, asel = self.heads(x, mi, tabs, rows)
        return {"video": v, "audio": a, "video_sel": vsel, "audio_sel": asel, "x0": x0, "x": x, "tables": tabs}
