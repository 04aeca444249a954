"""Plain fp64 CPU oracle for one MiniMax-H3 transformer block forward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library never
calls it, and it shares no code with the CUDA path: the two meet only through
the seeded inputs of ``h3_inputs``.

Every quantity is computed in float64 from the same bf16 / fp32 input values
the GPU reads, with no intermediate rounding. Library primitives used as steps:
``numpy.matmul`` (the linears), ``numpy.exp``/``cos``/``sin``/``sqrt``.

What the block computes (sources are the pages' titles and sections):

* "MiniMaxH3Transformer3DModel" (diffusers API page), introduction: one packed
  sequence, full self-attention over it, no cross-attention and no per-modality
  weights; the per-row modality tag selects the AdaLN modulation; padding rows
  (tag -1) form their own attention document.
* Same page, constructor parameters: hidden_size, heads x head_dim (larger than
  hidden), SwiGLU ffn_dim, rope_theta, norm_eps of the pre-attention and
  pre-feed-forward norms, qk_norm_eps of the per-head query/key norms.
* Same page, ``forward`` parameters: per-row timestep index, modality tag and
  (t, h, w) rotary coordinates.
* "HyperFlow H3 Flash Brings MiniMax H3 Video to One GPU", section "How it got
  smaller and faster": rotated W8A8 INT8 linears.

The pages give the ingredients but not the block's equations. Readings taken
where they are silent (each one is listed with its reason in the design notes):

1. Sequential pre-norm AdaLN block: h = rmsnorm(x)(1+scale1)+shift1;
   x1 = x + gate1 * out_proj(attn(h)); h2 = rmsnorm(x1)(1+scale2)+shift2;
   out = x1 + gate2 * ffn(h2).
2. The pre-norms are RMSNorm with no learned gain (AdaLN supplies the scale).
3. The 6 modulation vectors are ordered shift1, scale1, gate1, shift2, scale2,
   gate2; the table is fp32 [n_tags][n_t][6][C]. Padding rows get all zeros.
4. Per-head QK RMSNorm over head_dim with a gain vector [head_dim] shared by
   all heads, applied before RoPE; v is not normed.
5. 3D RoPE: pairs of adjacent channels (2j, 2j+1); the first p_t pairs rotate
   with the t coordinate, the next p_h with h, the next p_w with w, the rest
   pass through. For an axis with n pairs the i-th pair has frequency
   theta^(-i/n). Rotation (a, b) -> (a cos phi - b sin phi, a sin phi + b cos phi).
6. Attention scale 1/sqrt(head_dim); document of a row = (tag == -1).
7. W8A8: block-diagonal normalised Sylvester Hadamard on each 128-channel
   chunk of a linear's input (activations a' = H a, weights W' = W H);
   per-token symmetric int8 activations, per-output-channel int8 weights,
   s = amax / 127, q = clamp(round-half-even(v / s), -127, 127), s = 0 when
   amax = 0; int32 accumulate; y = acc * s_a[row] * s_w[col].
"""
from __future__ import annotations

import numpy as np

TAG_PAD = -1
MOD_SHIFT1, MOD_SCALE1, MOD_GATE1, MOD_SHIFT2, MOD_SCALE2, MOD_GATE2 = range(6)


def f64(t):
    """Any torch tensor / array -> float64 numpy array (exact for bf16/fp32)."""
    if hasattr(t, "detach"):
        t = t.detach().float().cpu().numpy()
    return np.asarray(t, dtype=np.float64)


# --------------------------------------------------------------------------
# AdaLN modulation and the pre-norms
# --------------------------------------------------------------------------

def modulation(table, tag, tidx):
    """Per-row modulation vectors m[r] = table[tag[r]][tidx[r]] ([R, 6, C] for
    a block's table, [R, 2, C] for norm_out's);
    zero for padding rows, which have no table row.
    ("MiniMaxH3Transformer3DModel", introduction: the per-row modality tag
    selects the AdaLN modulation parameters; forward: timestep_indices.)"""
    table = f64(table)
    tag = np.asarray(tag)
    tidx = np.asarray(tidx)
    m = np.zeros((tag.shape[0],) + table.shape[2:], dtype=np.float64)
    valid = tag != TAG_PAD
    m[valid] = table[tag[valid], tidx[valid]]
    return m


def rmsnorm(x, eps):
    """x / sqrt(mean(x^2) + eps) over the last axis, no gain."""
    x = f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def adaln(x, shift, scale, eps):
    """Pre-norm with AdaLN modulation: rmsnorm(x) * (1 + scale) + shift.
    ("MiniMaxH3Transformer3DModel", constructor: norm_eps of the
    pre-attention and pre-feed-forward norms.)"""
    return rmsnorm(x, eps) * (1.0 + scale) + shift


# --------------------------------------------------------------------------
# Per-head QK norm and 3D RoPE
# --------------------------------------------------------------------------

def qk_rmsnorm(xh, gain, eps):
    """Per-head RMSNorm over head_dim with a shared [head_dim] gain.
    xh: [R, H, D]. ("MiniMaxH3Transformer3DModel", constructor: qk_norm_eps of
    the per-head query/key norms.)"""
    return rmsnorm(xh, eps) * f64(gain)


def rope_frequencies(n_pairs, theta):
    """Frequencies of one axis with n pairs: theta^(-i/n), i = 0..n-1.
    ("MiniMaxH3Transformer3DModel", constructor: rope_theta is the base of the
    rotary frequency schedule.)"""
    i = np.arange(n_pairs, dtype=np.float64)
    return theta ** (-i / n_pairs)


def rope_angles(pos, rope_pairs, theta, head_dim):
    """Angle of every rotary pair of every row: [R, head_dim/2]; pairs past
    p_t + p_h + p_w get angle 0 (they pass through)."""
    pos = np.asarray(pos, dtype=np.float64)
    ang = np.zeros((pos.shape[0], head_dim // 2), dtype=np.float64)
    j = 0
    for axis, n in enumerate(rope_pairs):
        ang[:, j:j + n] = pos[:, axis:axis + 1] * rope_frequencies(n, theta)[None, :]
        j += n
    return ang


def apply_rope(xh, pos, rope_pairs, theta):
    """Rotate adjacent channel pairs (2j, 2j+1) of every head by the row's
    angles. xh: [R, H, D]. ("MiniMaxH3Transformer3DModel", forward:
    position_ids are the (t, h, w) rotary coordinates of every row.)"""
    xh = f64(xh)
    D = xh.shape[-1]
    ang = rope_angles(pos, rope_pairs, theta, D)[:, None, :]  # [R, 1, D/2]
    c, s = np.cos(ang), np.sin(ang)
    a, b = xh[..., 0::2], xh[..., 1::2]
    out = np.empty_like(xh)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


# --------------------------------------------------------------------------
# Document-masked attention
# --------------------------------------------------------------------------

def documents(tag):
    """Attention document of every row: 1 for padding rows, 0 otherwise.
    ("MiniMaxH3Transformer3DModel", introduction: padding rows are kept in
    their own attention document by a boolean mask.)"""
    return (np.asarray(tag) == TAG_PAD).astype(np.int64)


def softmax(s, axis=-1):
    """Max-subtracted softmax."""
    s = s - np.max(s, axis=axis, keepdims=True)
    e = np.exp(s)
    return e / np.sum(e, axis=axis, keepdims=True)


def attention(q, k, v, doc_q, doc_k):
    """o[r, h] = sum_j softmax_j(q[r,h] . k[j,h] / sqrt(D)) v[j,h] over the keys
    j of the query's document. q: [Rq, H, D], k/v: [Rk, H, D] -> [Rq, H, D]."""
    q, k, v = f64(q), f64(k), f64(v)
    D = q.shape[-1]
    out = np.zeros_like(q)
    doc_q = np.asarray(doc_q)
    doc_k = np.asarray(doc_k)
    for d in np.unique(doc_q):
        qi = np.nonzero(doc_q == d)[0]
        kj = np.nonzero(doc_k == d)[0]
        if kj.size == 0:
            continue
        # (a document holding every key is used in place: no gathered copy)
        kd = k if kj.size == k.shape[0] else k[kj]
        vd = v if kj.size == v.shape[0] else v[kj]
        qh = q[qi].transpose(1, 0, 2)            # [H, rq, D]
        kh = kd.transpose(1, 2, 0)               # [H, D, rk]
        vh = vd.transpose(1, 0, 2)               # [H, rk, D]
        p = softmax(np.matmul(qh, kh) / np.sqrt(D))
        out[qi] = np.matmul(p, vh).transpose(1, 0, 2)
    return out


# --------------------------------------------------------------------------
# SwiGLU
# --------------------------------------------------------------------------

def silu(g):
    return g / (1.0 + np.exp(-g))


def swiglu(g, u):
    """silu(gate) * up. ("MiniMaxH3Transformer3DModel", constructor: ffn_dim is
    the inner dimension of the SwiGLU feed-forward layers.)"""
    return silu(g) * u


# --------------------------------------------------------------------------
# Rotated W8A8 pieces
# --------------------------------------------------------------------------

def sylvester_hadamard(n):
    """Unnormalised Sylvester Hadamard matrix of order n (a power of two):
    H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]."""
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    assert h.shape[0] == n
    return h


def rotate_blocks(a, block=128):
    """Apply H/sqrt(block) to each contiguous ``block``-channel chunk of the
    last axis: a'[..., chunk] = H a[..., chunk] / sqrt(block).
    ("HyperFlow H3 Flash ...", "How it got smaller and faster": rotated
    W8A8 INT8 quantisation.)"""
    a = f64(a)
    K = a.shape[-1]
    assert K % block == 0
    hn = sylvester_hadamard(block).astype(np.float64) / np.sqrt(block)
    r = a.reshape(a.shape[:-1] + (K // block, block))
    return np.matmul(r, hn.T).reshape(a.shape)


def quantize_rows(v):
    """Symmetric per-row int8: s = amax/127, q = clamp(rint(v/s), -127, 127);
    a row with amax = 0 gets s = 0 and q = 0. Returns (int8 q, float64 s)."""
    v = f64(v)
    amax = np.max(np.abs(v), axis=-1)
    s = amax / 127.0
    safe = np.where(s > 0, s, 1.0)
    q = np.clip(np.rint(v / safe[..., None]), -127, 127)
    q[s == 0] = 0
    return q.astype(np.int8), s


def int8_matmul_exact(a_q, w_q):
    """Exact integer product acc[r, c] = sum_k a_q[r, k] * w_q[c, k] (int64).

    Computed as a float64 matrix product: every term is an integer of
    magnitude <= 127 * 127, so every partial sum, in any order, is an integer
    below 127^2 K < 2^53 and is represented exactly; the result is then the
    exact integer sum (asserted bound on K)."""
    a = np.asarray(a_q)
    w = np.asarray(w_q)
    K = a.shape[-1]
    assert 127 * 127 * K < 2 ** 53
    assert np.abs(a).max(initial=0) <= 127 and np.abs(w).max(initial=0) <= 127
    acc = np.matmul(a.astype(np.float64), w.astype(np.float64).T)
    return np.rint(acc).astype(np.int64)


def prepare_int8_weight(w):
    """Rotate the input channels of a weight [out, in] (W' = W H) and
    quantise each output channel: returns (int8 [out, in], float64 s_w[out])."""
    return quantize_rows(rotate_blocks(w))


def w8a8_linear(a, wq, sw):
    """Rotated W8A8 linear: rotate and quantise the activation rows, integer
    product, dequantise with the two scales."""
    aq, sa = quantize_rows(rotate_blocks(a))
    acc = int8_matmul_exact(aq, wq)
    return acc.astype(np.float64) * sa[:, None] * sw[None, :]


def bf16_round(x):
    """Round to the nearest bfloat16 value (ties to even), returned as float64.
    Used only by the faithful mode of the block oracle."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


# --------------------------------------------------------------------------
# The block
# --------------------------------------------------------------------------

class BlockOracle:
    """One block forward in fp64, optionally for a subset of query rows.

    ``dims`` carries hidden, heads, head_dim, ffn, rope_pairs, rope_theta,
    norm_eps, qk_norm_eps and quant. ``weights`` carries bf16 wqkv [3HD, C],
    q_gain/k_gain [D], wo [C, HD], w13 [2F, C] (W1 rows then W3 rows) and
    w2 [C, F].

    ``faithful=True`` is a diagnostic, not the contract: it rounds to bf16 at
    the points where the block's stages are stored as bf16 (h1 and h2 on the
    bf16 path, q, k, v, o, x1, a and out on both), so that a difference
    against the GPU can be told apart from the rounding of those stores. The
    default computes every stage in fp64 with no intermediate rounding.
    """

    def __init__(self, dims, weights, faithful=False):
        self.d = dims
        self.faithful = bool(faithful)
        self.quant = int(getattr(dims, "quant", 0))
        self.wqkv = f64(weights.wqkv)
        self.q_gain = f64(weights.q_gain)
        self.k_gain = f64(weights.k_gain)
        self.wo = f64(weights.wo)
        self.w13 = f64(weights.w13)
        self.w2 = f64(weights.w2)
        if self.quant:
            self.int8 = {name: prepare_int8_weight(w) for name, w in
                         (("qkv", self.wqkv), ("o", self.wo), ("13", self.w13), ("2", self.w2))}

    def _store(self, a):
        """A stage as the block stores it: bf16 in faithful mode, else as is."""
        return bf16_round(a) if self.faithful else a

    def _store_bf16_path(self, a):
        """h1 / h2: stored as bf16 on the bf16 path only (the W8A8 path
        quantises them straight from fp32)."""
        return bf16_round(a) if (self.faithful and not self.quant) else a

    # linear y = a W^T, bf16 weights or rotated W8A8; ``rows`` (a slice)
    # selects output channels (weight rows), which leaves every computed
    # column unchanged
    def linear(self, a, name, rows=None):
        if self.quant:
            wq, sw = self.int8[name]
            if rows is not None:
                wq, sw = wq[rows], sw[rows]
            return w8a8_linear(a, wq, sw)
        w = {"qkv": self.wqkv, "o": self.wo, "13": self.w13, "2": self.w2}[name]
        if rows is not None:
            w = w[rows]
        return np.matmul(a, w.T)

    def _split_heads(self, y):
        return y.reshape(y.shape[0], self.d.heads, self.d.head_dim)

    def qkv(self, h1, pos, part=("q", "k", "v")):
        """QKV projection, per-head QK RMSNorm, 3D RoPE. Returns a dict of
        [R, H, D] arrays for the requested parts."""
        d = self.d
        HD = d.hd
        names = [p for p in ("q", "k", "v") if p in part]
        first = {"q": 0, "k": 1, "v": 2}[names[0]]
        assert [{"q": 0, "k": 1, "v": 2}[p] for p in names] == list(range(first, first + len(names)))
        y = self.linear(h1, "qkv", rows=slice(first * HD, (first + len(names)) * HD))
        ys = {p: y[:, i * HD:(i + 1) * HD] for i, p in enumerate(names)}
        out = {}
        if "q" in part:
            q = qk_rmsnorm(self._split_heads(ys["q"]), self.q_gain, d.qk_norm_eps)
            out["q"] = self._store(apply_rope(q, pos, d.rope_pairs, d.rope_theta))
        if "k" in part:
            k = qk_rmsnorm(self._split_heads(ys["k"]), self.k_gain, d.qk_norm_eps)
            out["k"] = self._store(apply_rope(k, pos, d.rope_pairs, d.rope_theta))
        if "v" in part:
            out["v"] = self._store(self._split_heads(ys["v"]))
        return out

    def kv_all(self, x, tag, tidx, pos, table, kv_chunk=4096):
        """k and v ([N, H, D]) of every row of the sequence."""
        d = self.d
        x = f64(x)
        table = f64(table)
        N = x.shape[0]
        k_all = np.empty((N, d.heads, d.head_dim))
        v_all = np.empty((N, d.heads, d.head_dim))
        for s in range(0, N, kv_chunk):
            e = min(N, s + kv_chunk)
            m = modulation(table, tag[s:e], tidx[s:e])
            h = self._store_bf16_path(adaln(x[s:e], m[:, MOD_SHIFT1], m[:, MOD_SCALE1], d.norm_eps))
            kv = self.qkv(h, pos[s:e], part=("k", "v"))
            k_all[s:e], v_all[s:e] = kv["k"], kv["v"]
        return k_all, v_all

    def query(self, x_rows, tag_rows, tidx_rows, pos_rows, table, k_all, v_all, doc_all, o_given=None):
        """Every stage of the block for the given query rows, attending to
        the keys / values of the whole sequence (or taking the attention
        output ``o_given`` [R, H, D] from another attention, e.g. block-sparse)."""
        d = self.d
        xr = f64(x_rows)
        m = modulation(f64(table), tag_rows, tidx_rows)
        h1 = self._store_bf16_path(adaln(xr, m[:, MOD_SHIFT1], m[:, MOD_SCALE1], d.norm_eps))
        q = self.qkv(h1, pos_rows, part=("q",))["q"]
        if o_given is None:
            o = attention(q, k_all, v_all, documents(tag_rows), doc_all).reshape(xr.shape[0], d.hd)
        else:
            o = f64(o_given).reshape(xr.shape[0], d.hd)
        o = self._store(o)
        x1 = self._store(xr + m[:, MOD_GATE1] * self.linear(o, "o"))
        h2 = self._store_bf16_path(adaln(x1, m[:, MOD_SHIFT2], m[:, MOD_SCALE2], d.norm_eps))
        g_u = self.linear(h2, "13")
        a = self._store(swiglu(g_u[:, :d.ffn], g_u[:, d.ffn:]))
        out = self._store(x1 + m[:, MOD_GATE2] * self.linear(a, "2"))
        return {"h1": h1, "q": q, "o": o, "x1": x1, "h2": h2, "a": a, "out": out}

    def forward(self, x, tag, tidx, pos, table, rows=None, kv_chunk=4096, keep=None):
        """Block forward. ``rows`` (sorted indices) restricts every per-row
        stage to those query rows; k and v are always computed for all rows,
        since every query sees every key of its document. ``keep`` (bool
        [blocks, heads, tiles]) replaces dense attention with block-sparse
        attention over those tiles. Returns a dict of
        stages for the returned rows: h1, q, k, v, o, x1, h2, a, out (and the
        full-sequence k, v under "k_all", "v_all")."""
        x = f64(x)
        tag = np.asarray(tag)
        tidx = np.asarray(tidx)
        pos = np.asarray(pos)
        N = x.shape[0]
        rows = np.arange(N) if rows is None else np.asarray(rows)
        k_all, v_all = self.kv_all(x, tag, tidx, pos, table, kv_chunk)
        o_given = None
        if keep is not None:
            # block-sparse attention (oracle/h3_sparse.py) with the given kept tiles
            from .h3_sparse import sparse_attention
            m = modulation(f64(table), tag, tidx)
            h1 = self._store_bf16_path(adaln(x, m[:, MOD_SHIFT1], m[:, MOD_SCALE1], self.d.norm_eps))
            q_all = self.qkv(h1, pos, part=("q",))["q"]
            o_given = sparse_attention(q_all, k_all, v_all, tag, keep, rows=rows)[rows]
        r = self.query(x[rows], tag[rows], tidx[rows], pos[rows], table, k_all, v_all, documents(tag), o_given)
        r.update({"rows": rows, "k": k_all[rows], "v": v_all[rows], "k_all": k_all, "v_all": v_all})
        return r
