"""fp64 CPU oracle of the modulation-table producer that feeds the block.

TEST INFRASTRUCTURE ONLY (same rules as oracle/h3_block.py): only tests/,
__graft_entry__.smoke() and bench.py's CPU-baseline leg may use it.

What the pages fix ("MiniMaxH3Transformer3DModel", diffusers API page,
constructor parameters): a sinusoidal timestep embedding of freq_dim = 256
channels, timesteps consumed unscaled in [0, 1]; a timestep MLP with inner
dimension time_embed_hidden_dim = 5376 and output time_embed_dim = 2688, whose
output is the input of every AdaLN projection; the MLP is float32 while the
block stack is bfloat16 (introduction). The per-row modality tag selects the
AdaLN modulation parameters (introduction). "HyperFlow ..." model card, "How it
works": a two-time embedder adds a second copy of the time embedder for the
step endpoint r and blends the two embeddings with a fixed gate; conditioning
rows keep r = t.

Readings taken where the pages are silent (listed in the design notes):
1. Embedding channel layout: [cos(t w_0..w_{h-1}), sin(t w_0..w_{h-1})] with
   h = freq_dim / 2 and w_i = 10000^(-i / h).
2. Time MLP: E(t) = W2 silu(W1 e(t) + b1) + b2.
3. Two-time blend: E = (1 - g) E(t) + g E_r(r), E_r a second MLP of the same
   shape; g = 0 gives the plain embedding.
4. AdaLN projection, one weight set per modality tag:
   table[tag][k] = A_tag silu(E_k) + a_tag, 6 * hidden outputs in the order
   shift1, scale1, gate1, shift2, scale2, gate2; A_tag is bf16 (inside the
   block stack), everything else fp32.
"""
from __future__ import annotations

import numpy as np

from .h3_block import f64, silu


def timestep_frequencies(freq_dim, base=10000.0):
    """w_i = base^(-i / h), i = 0..h-1, h = freq_dim / 2."""
    h = freq_dim // 2
    return base ** (-np.arange(h, dtype=np.float64) / h)


def sinusoidal_embedding(t, freq_dim):
    """e(t) = [cos(t w), sin(t w)] for each timestep t (unscaled): [K, freq_dim]."""
    t = np.asarray(t, dtype=np.float64).reshape(-1, 1)
    a = t * timestep_frequencies(freq_dim)[None, :]
    return np.concatenate([np.cos(a), np.sin(a)], axis=1)


def time_mlp(e, w1, b1, w2, b2):
    """E = W2 silu(W1 e + b1) + b2 (rows of e are timesteps)."""
    return np.matmul(silu(np.matmul(e, f64(w1).T) + f64(b1)), f64(w2).T) + f64(b2)


def two_time_embedding(t_now, t_end, gate, mlp, mlp_r, freq_dim):
    """(1 - g) E(t_now) + g E_r(t_end); mlp / mlp_r are (w1, b1, w2, b2)."""
    e = time_mlp(sinusoidal_embedding(t_now, freq_dim), *mlp)
    if gate == 0.0:
        return e
    er = time_mlp(sinusoidal_embedding(t_end, freq_dim), *mlp_r)
    return (1.0 - gate) * e + gate * er


def modulation_table(E, adaln_w, adaln_b):
    """table[tag][k] = A_tag silu(E_k) + a_tag -> [n_tags, K, 6C]."""
    s = silu(f64(E))                                  # [K, time_dim]
    A = f64(adaln_w)                                  # [n_tags, 6C, time_dim]
    return np.einsum("kd,tod->tko", s, A) + f64(adaln_b)[:, None, :]


def produce(params, t_now, t_end, gate):
    """Full producer: [n_tags, K, 6, C] fp64."""
    E = two_time_embedding(t_now, t_end, gate, params["mlp"], params.get("mlp_r"), params["freq_dim"])
    tab = modulation_table(E, params["adaln_w"], params["adaln_b"])
    n_tags, K, six_c = tab.shape
    return tab.reshape(n_tags, K, 6, six_c // 6)
