"""GPU parity: the CUDA path through the C-ABI against the fp64 oracle and
against exact / library references, on seeded inputs."""
from dataclasses import replace

import numpy as np
import pytest
import torch

import h3_inputs as hi
from oracle import h3_block as orc
from tests._parity import GpuCase, assert_intermediate, assert_stage, blob_tensor as _blob_tensor, errors, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a B200"
    import joint_video_audio_b200  # noqa: F401  (fails loudly if libh3blk.so is missing)
    yield


# ---------------------------------------------------------------- kernel level

@pytest.mark.parametrize("M,N,K", [(300, 384, 256), (128, 128, 64), (1, 256, 128), (1029, 768, 5376)])
def test_gemm_bf16_matches_fp32_reference(M, N, K):
    import joint_video_audio_b200 as j
    g = torch.Generator().manual_seed(M * 7 + N)
    a = torch.randn(M, K, generator=g).to(torch.bfloat16)
    b = (torch.randn(N, K, generator=g) / K ** 0.5).to(torch.bfloat16)
    c = j.gemm_bf16(a.cuda(), b.cuda())
    torch.cuda.synchronize()
    ref = a.double() @ b.double().T
    assert_stage("gemm_bf16", c, ref)


@pytest.mark.parametrize("M,N,K", [(257, 256, 384), (128, 384, 128), (64, 128, 14336)])
def test_gemm_s8_exact(M, N, K):
    import joint_video_audio_b200 as j
    g = torch.Generator().manual_seed(M + N + K)
    a = torch.randint(-127, 128, (M, K), generator=g, dtype=torch.int8)
    b = torch.randint(-127, 128, (N, K), generator=g, dtype=torch.int8)
    c = j.gemm_s8_s32(a.cuda(), b.cuda()).cpu()
    ref = orc.int8_matmul_exact(a.numpy(), b.numpy())
    assert np.array_equal(c.numpy().astype(np.int64), ref)


def test_gemm_s8_extreme_values_exact():
    import joint_video_audio_b200 as j
    K = 14336
    a = torch.full((128, K), 127, dtype=torch.int8)
    a[1] = -127
    b = torch.full((128, K), 127, dtype=torch.int8)
    c = j.gemm_s8_s32(a.cuda(), b.cuda()).cpu()
    assert int(c[0, 0]) == 231225344 and int(c[1, 5]) == -231225344


@pytest.mark.parametrize("rows,K", [(5, 256), (33, 7168), (17, 14336), (3, 5376)])
def test_rotate_quantize_vs_oracle(rows, K):
    import joint_video_audio_b200 as j
    g = torch.Generator().manual_seed(rows * K)
    x = (torch.randn(rows, K, generator=g) * 0.7).to(torch.bfloat16)
    x[0] = 0  # amax = 0 row
    q, s = j.rotate_quantize(x.cuda())
    q, s = q.cpu().numpy().astype(np.int64), s.cpu().numpy().astype(np.float64)
    rq, rs = orc.quantize_rows(orc.rotate_blocks(x))
    assert np.all(q[0] == 0) and s[0] == 0
    np.testing.assert_allclose(s, rs, rtol=1e-5)
    d = np.abs(q - rq.astype(np.int64))
    assert d.max() <= 1
    assert np.mean(d == 0) >= 0.999


# ---------------------------------------------------------------- tiny block

@pytest.fixture(scope="module")
def tiny():
    inp = hi.make_inputs("tiny_320")
    case = GpuCase(inp)
    case.run()
    lay = inp.layout
    ref = orc.BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    return case, ref


def test_tiny_stage_h1(tiny):
    case, ref = tiny
    assert_intermediate("h1", case.stage("H1"), ref["h1"])


def test_tiny_stage_qkv(tiny):
    case, ref = tiny
    q, k, v = case.qkv()
    assert_intermediate("q", q, ref["q"])
    assert_intermediate("k", k, ref["k"])
    assert_intermediate("v", v, ref["v"])


def test_tiny_partial_rotary_split():
    """Rotary pairs that follow no axis pass through unrotated (the page's own
    split rotates 48 of 64 pairs at head_dim 128): 20 of 32 pairs rotated here,
    the rest read (sin, cos) = (0, 1) from the table and are skipped."""
    lay = hi.layout_tiny()
    inp = hi.make_inputs(replace(hi.TINY, rope_pairs=(4, 8, 8)), lay)
    case = GpuCase(inp)
    case.run()
    ref = orc.BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    q, k, v = case.qkv()
    assert_intermediate("q", q, ref["q"])
    assert_intermediate("k", k, ref["k"])
    assert_stage("out", case.out, ref["out"])


def test_tiny_stage_attention(tiny):
    case, ref = tiny
    assert_intermediate("o", case.stage("O"), ref["o"])


def test_tiny_stages_x1_h2_a_out(tiny):
    case, ref = tiny
    assert_intermediate("x1", case.stage("X1"), ref["x1"])
    assert_intermediate("h2", case.stage("H2"), ref["h2"])
    assert_intermediate("a", case.stage("A"), ref["a"])
    assert_stage("out", case.out, ref["out"])


def _bf16_ulp(r):
    """Spacing of bf16 values at |r| (8 significant bits)."""
    a = np.maximum(np.abs(r), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def test_tiny_stages_vs_faithful_oracle(tiny):
    """Against the oracle's diagnostic mode that rounds to bf16 where the GPU
    stores bf16 (h1, q, k, v, o, x1, a, out), h1 from the inputs and q, k, v
    from the GPU's h1: the fp32 arithmetic of the norm and of the QKV GEMM +
    QK-norm + RoPE epilogue is off from fp64 by far less than one bf16
    spacing of an O(1) value (fp32 sums of a few hundred products, and the
    hardware sine / cosine at about 2^-21 absolute), so the stored
    h1, q, k and v can differ from the rounded fp64 values only where a value
    sits next to a rounding boundary: by at most one spacing plus that
    absolute error (which matters only for values near zero, where the
    rotation cancels), and rarely (>= 99 % identical)."""
    case, _ = tiny
    inp = case.inp
    lay = inp.layout
    ob = orc.BlockOracle(inp.dims, inp.weights, faithful=True)
    rf = ob.forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    # q, k, v from the GPU's own h1: a legitimate one-spacing difference in
    # an h1 value moves every q of its row by far more than a q spacing
    h1_g = case.stage("H1")
    rq = ob.qkv(to64(h1_g), lay.pos)
    q, k, v = case.qkv()
    d_ = inp.dims
    ang = orc.rope_angles(lay.pos, d_.rope_pairs, d_.rope_theta, d_.head_dim)     # [N, D/2]
    for name, g, f in (("h1", h1_g, rf["h1"]), ("q", q, rq["q"]), ("k", k, rq["k"]), ("v", v, rq["v"])):
        g, f = to64(g), to64(f)
        d = np.abs(g - f)
        same = float(np.mean(d == 0))
        bound = _bf16_ulp(f) + 2.0 ** -16
        if name in ("q", "k"):
            # the rotary angle pos * freq is formed in fp32 (relative error
            # 2^-23) and its sine / cosine carry about 2^-21 absolute: a pair of
            # norm r moves by up to r (|angle| 2^-22 + 2^-20)
            pair = np.sqrt(f[..., 0::2] ** 2 + f[..., 1::2] ** 2)
            slack = pair * (np.abs(ang)[:, None, :] * 2.0 ** -22 + 2.0 ** -20)
            bound = bound + np.repeat(slack, 2, axis=-1)
        bad = np.argwhere(d > bound)
        detail = [(tuple(int(i) for i in b), float(g[tuple(b)]), float(f[tuple(b)]), float(bound[tuple(b)]))
                  for b in bad[:4]]
        assert bad.size == 0, f"{name}: {len(bad)} values more than one bf16 spacing off: {detail}"
        assert same >= 0.99, f"{name}: only {same:.4f} identical to the faithful oracle"


def test_tiny_padding_rows_unchanged_and_isolated(tiny):
    case, ref = tiny
    pad = torch.from_numpy(case.inp.layout.tag == -1).cuda()
    out0 = case.run().clone()
    assert torch.equal(out0[pad], case.x[pad])
    x2 = case.x.clone()
    x2[pad] = (torch.randn(int(pad.sum()), case.dims.hidden, device="cuda") * 7).to(torch.bfloat16)
    out1 = case.run(x=x2).clone()
    assert torch.equal(out1[~pad], out0[~pad])
    assert torch.equal(out1[pad], x2[pad])
    case.run()


def test_tiny_zero_gates_identity(tiny):
    case, _ = tiny
    t = case.table.clone()
    t[:, :, 2] = 0
    t[:, :, 5] = 0
    out = case.run(table=t).clone()
    assert torch.equal(out, case.x)
    case.run()


def test_tiny_bad_index_reported():
    import joint_video_audio_b200 as j
    inp = hi.make_inputs("tiny_320")
    case = GpuCase(inp)
    case.tag[3] = 9  # outside n_tags
    case.run()
    assert case.block.check(case.ws, case.n) == j.capi.H3BLK_ERR_BAD_INDEX
    case.tag[3] = 0
    case.tidx[5] = -3
    case.run()
    assert case.block.check(case.ws, case.n) == j.capi.H3BLK_ERR_BAD_INDEX
    case.tidx[5] = 0
    case.run()
    assert case.block.check(case.ws, case.n) == j.capi.H3BLK_OK


@pytest.mark.parametrize("n", [1, 2, 127, 129, 255, 300])
def test_tiny_ragged_lengths(n):
    full = hi.layout_tiny()
    n_pad = n // 4  # the tail keeps some padding rows
    sel = np.r_[np.arange(n - n_pad), np.arange(full.n - n_pad, full.n)]
    lay = hi.Layout(f"tiny_{n}", full.tag[sel], full.tidx[sel], full.pos[sel])
    inp = hi.make_inputs(hi.TINY, lay)
    case = GpuCase(inp)
    case.run()
    ref = orc.BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    assert_intermediate("o", case.stage("O"), ref["o"])
    assert_stage("out", case.out, ref["out"])


def test_tiny_padding_anywhere():
    base = hi.layout_tiny()
    perm = np.random.default_rng(5).permutation(base.n)
    lay = hi.Layout("tiny_perm", base.tag[perm], base.tidx[perm], base.pos[perm])
    inp = hi.make_inputs(hi.TINY, lay)
    case = GpuCase(inp)
    case.run()
    ref = orc.BlockOracle(inp.dims, inp.weights).forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    assert_intermediate("o", case.stage("O"), ref["o"])
    assert_stage("out", case.out, ref["out"])


@pytest.fixture(scope="module")
def tiny_w8a8():
    inp = hi.make_inputs("tiny_320")
    inp.dims = replace(inp.dims, quant=1)
    case = GpuCase(inp)
    case.run()
    lay = inp.layout
    ob = orc.BlockOracle(inp.dims, inp.weights)
    ref = ob.forward(inp.x, lay.tag, lay.tidx, lay.pos, inp.table)
    return case, ob, ref


def _int8_agree(name, got, ref):
    d = np.abs(np.asarray(got, dtype=np.int64) - np.asarray(ref, dtype=np.int64))
    assert d.max() <= 1, f"{name}: int8 operands differ by {d.max()}"
    assert np.mean(d == 0) >= 0.999, f"{name}: only {np.mean(d == 0):.4%} identical"


def test_tiny_w8a8_weights_match_oracle(tiny_w8a8):
    case, ob, _ = tiny_w8a8
    d = case.dims
    hd = d.heads * d.head_dim
    shapes = {"qkv": (3 * hd, d.hidden), "o": (d.hidden, hd), "13": (2 * d.ffn, d.hidden), "2": (d.hidden, d.ffn)}
    ptrs = {"qkv": (case.w.c.wqkv, case.w.c.s_qkv), "o": (case.w.c.wo, case.w.c.s_o),
            "13": (case.w.c.w13, case.w.c.s_13), "2": (case.w.c.w2, case.w.c.s_2)}
    for name, (rows, cols) in shapes.items():
        wq = _blob_tensor(case.w, ptrs[name][0], rows * cols, torch.int8).view(rows, cols).cpu().numpy()
        sw = _blob_tensor(case.w, ptrs[name][1], rows, torch.float32).cpu().numpy()
        rq, rs = ob.int8[name]
        _int8_agree(f"w_{name}", wq, rq)
        np.testing.assert_allclose(sw, rs, rtol=1e-5)


def test_tiny_w8a8_activation_operands(tiny_w8a8):
    case, _, ref = tiny_w8a8
    q, s = case.stage("H1_Q8").cpu().numpy(), case.stage("H1_SCALE").cpu().numpy()
    rq, rs = orc.quantize_rows(orc.rotate_blocks(ref["h1"]))
    _int8_agree("h1_q8", q, rq)
    np.testing.assert_allclose(s, rs, rtol=1e-4)
    # the attention output is quantised from its bf16 value
    oq = case.stage("O_Q8").cpu().numpy()
    rq, _ = orc.quantize_rows(orc.rotate_blocks(case.stage("O").float().cpu().numpy()))
    _int8_agree("o_q8", oq, rq)
    aq = case.stage("A_Q8").cpu().numpy()
    rq, _ = orc.quantize_rows(orc.rotate_blocks(case.stage("A").float().cpu().numpy()))
    _int8_agree("a_q8", aq, rq)


def test_tiny_w8a8_ffn_up_from_gpu_operands(tiny_w8a8):
    """The int8 FFN-up GEMM + dequantisation + SwiGLU, recomputed exactly from
    the GPU's own int8 operands."""
    case, _, _ = tiny_w8a8
    d = case.dims
    h2q = case.stage("H2_Q8").cpu().numpy()
    h2s = case.stage("H2_SCALE").cpu().numpy().astype(np.float64)
    wq = _blob_tensor(case.w, case.w.c.w13, 2 * d.ffn * d.hidden, torch.int8).view(2 * d.ffn, d.hidden).cpu().numpy()
    sw = _blob_tensor(case.w, case.w.c.s_13, 2 * d.ffn, torch.float32).cpu().numpy().astype(np.float64)
    y = orc.int8_matmul_exact(h2q, wq).astype(np.float64) * h2s[:, None] * sw[None, :]
    a = orc.swiglu(y[:, :d.ffn], y[:, d.ffn:])
    assert_intermediate("a (from GPU operands)", case.stage("A"), a)


def test_tiny_w8a8_block(tiny_w8a8):
    case, _, ref = tiny_w8a8
    q, k, v = case.qkv()
    assert_intermediate("q", q, ref["q"])
    assert_intermediate("k", k, ref["k"])
    assert_intermediate("o", case.stage("O"), ref["o"])
    assert_stage("out", case.out, ref["out"])
