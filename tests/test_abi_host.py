"""Host-side tests of the C-ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before touching any GPU."""
import ctypes as C
import os
import re
import subprocess

import pytest

import h3_inputs as hi
import joint_video_audio_b200 as j
from joint_video_audio_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h3blk.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"H3BLK_API\s+[\w\s\*]*?\b(h3blk_\w+)\s*\(", txt)))


def test_header_declarations_match_binding():
    assert declared_symbols() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (h3blk_\w+)", out))
    missing = set(declared_symbols()) - exported
    assert not missing, missing
    lib = C.CDLL(B.LIB_PATH)
    for s in declared_symbols():
        assert getattr(lib, s) is not None


def test_version_and_error_strings():
    assert B.h3blk_version() >= 100
    for st in range(6):
        assert B.error_string(st)
    assert "unknown" in B.error_string(99)


def _cfg(**kw):
    base = dict(hidden=256, heads=6, head_dim=64, ffn=768, n_tags=4, n_t=2, rope_pairs_t=8, rope_pairs_h=12,
                rope_pairs_w=12, rope_theta=1e4, norm_eps=1e-5, qk_norm_eps=1e-5, quant=0)
    base.update(kw)
    return B.h3blk_config(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, B.H3BLK_OK),
    ({"quant": 1}, B.H3BLK_OK),
    ({"hidden": 0}, B.H3BLK_ERR_INVALID_ARG),
    ({"n_t": 0}, B.H3BLK_ERR_INVALID_ARG),
    ({"rope_theta": -1.0}, B.H3BLK_ERR_INVALID_ARG),
    ({"quant": 2}, B.H3BLK_ERR_INVALID_ARG),
    ({"hidden": 200}, B.H3BLK_ERR_UNSUPPORTED),
    ({"ffn": 700}, B.H3BLK_ERR_UNSUPPORTED),
    ({"head_dim": 96}, B.H3BLK_ERR_UNSUPPORTED),
    ({"heads": 3}, B.H3BLK_ERR_UNSUPPORTED),          # 3 * 64 not a multiple of 128
    ({"rope_pairs_w": 13}, B.H3BLK_ERR_UNSUPPORTED),  # 8 + 12 + 13 > 32
])
def test_create_validation(kw, status):
    assert B.h3blk_create_status(_cfg(**kw)) == status


def test_create_null():
    assert B.h3blk_create_status(None) == B.H3BLK_ERR_INVALID_ARG


def test_real_and_page_rope_splits_accepted():
    # the page's own split: 16 pairs per axis, 96 of 128 channels rotated
    assert B.h3blk_create_status(_cfg(hidden=5376, heads=56, head_dim=128, ffn=14336,
                                      rope_pairs_t=16, rope_pairs_h=16, rope_pairs_w=16)) == B.H3BLK_OK
    assert B.h3blk_create_status(_cfg(hidden=5376, heads=56, head_dim=128, ffn=14336,
                                      rope_pairs_t=16, rope_pairs_h=24, rope_pairs_w=24)) == B.H3BLK_OK


def test_workspace_layout():
    blk = j.H3Block(hi.REAL)
    n = 32768
    ws = blk.workspace_bytes(n)
    C_, HD, F = 5376, 7168, 14336
    # h1, qkv, o, x1, h2, a in bf16, and the rotary (sin, cos) table: 64
    # pairs x 8 bytes per row
    stages = n * 2 * (C_ + 3 * HD + HD + C_ + C_ + F) + n * 64 * 8
    assert ws >= stages
    assert ws < stages + 4 * 1024 * 1024
    seen = []
    for name in ("ERROR", "H1", "QKV", "O", "X1", "H2", "A"):
        off, nb = B.h3blk_stage_view(blk.handle, n, name)
        assert off % 256 == 0 and off + nb <= ws
        seen.append((off, off + nb))
    seen.sort()
    for (a0, a1), (b0, b1) in zip(seen, seen[1:]):
        assert a1 <= b0  # no two stages overlap
    with pytest.raises(B.H3BlkError):
        B.h3blk_stage_view(blk.handle, n, "H1_Q8")  # not produced by the bf16 path
    assert blk.workspace_bytes(1) > 0
    with pytest.raises(B.H3BlkError):
        B.h3blk_workspace_bytes(blk.handle, 0)


def test_w8a8_layout_and_blob():
    from dataclasses import replace
    blk = j.H3Block(replace(hi.REAL, quant=1))
    n = 1000
    for name in ("H1_Q8", "H1_SCALE", "O_Q8", "O_SCALE", "H2_Q8", "H2_SCALE", "A_Q8", "A_SCALE"):
        off, nb = B.h3blk_stage_view(blk.handle, n, name)
        assert off % 256 == 0
    nb = B.h3blk_int8_weights_bytes(blk.handle)
    assert nb >= 385351680  # one int8 byte per weight


def _fake_forward(blk, n, **override):
    """A forward call whose pointers are fake host integers: every case here
    must be rejected by validation before any CUDA call is made."""
    ws = blk.workspace_bytes(max(n, 1))
    base = 1 << 40
    args = dict(x=base, tag=base + (1 << 30), tidx=base + (2 << 30), pos=base + (3 << 30),
                table=base + (4 << 30), out=base + (5 << 30), ws=base + (6 << 30), ws_bytes=ws)
    args.update(override)
    w = B.h3blk_weights(wqkv=base + (8 << 30), q_gain=base + (9 << 30), k_gain=base + (9 << 30) + 256,
                        wo=base + (10 << 30), w13=base + (11 << 30), w2=base + (12 << 30))
    return B.h3blk_forward(blk.handle, n, args["x"], args["tag"], args["tidx"], args["pos"], args["table"], w,
                           args["out"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("override", [
    {"x": 0}, {"tag": 0}, {"tidx": 0}, {"pos": 0}, {"table": 0}, {"out": 0}, {"ws": 0},
    {"x": (1 << 40) + 8},              # misaligned
    {"ws_bytes": 1024},                # workspace too small
    {"out": 1 << 40},                  # out aliases x
    {"out": (1 << 40) + (6 << 30)},    # out inside the workspace
])
def test_forward_rejects_bad_arguments(override):
    blk = j.H3Block(hi.TINY)
    assert _fake_forward(blk, 320, **override) == B.H3BLK_ERR_INVALID_ARG


@pytest.mark.parametrize("field", ["q_gain", "k_gain"])
def test_forward_rejects_misaligned_gains(field):
    # the QKV epilogue reads the gains 16 bytes at a time; the check runs
    # before any CUDA call, so the fake pointers are never dereferenced
    blk = j.H3Block(hi.TINY)
    n = 320
    ws = blk.workspace_bytes(n)
    base = 1 << 40
    wd = dict(wqkv=base + (8 << 30), q_gain=base + (9 << 30), k_gain=base + (9 << 30) + 256,
              wo=base + (10 << 30), w13=base + (11 << 30), w2=base + (12 << 30))
    wd[field] += 8
    w = B.h3blk_weights(**wd)
    assert B.h3blk_forward(blk.handle, n, base, base + (1 << 30), base + (2 << 30), base + (3 << 30),
                           base + (4 << 30), w, base + (5 << 30), base + (6 << 30), ws, None) == \
        B.H3BLK_ERR_INVALID_ARG


def test_forward_rejects_empty_sequence():
    blk = j.H3Block(hi.TINY)
    assert _fake_forward(blk, 0) == B.H3BLK_ERR_INVALID_ARG


def test_kernel_level_calls_reject_bad_sizes():
    assert B.h3blk_rotate_quantize(4, 100, 1 << 40, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_rotate_quantize(4, 128 * 200, 1 << 40, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_gemm_s8_s32(16, 100, 128, 1 << 40, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_gemm_s8_s32(16, 128, 64, 1 << 40, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_gemm_bf16(16, 128, 32, 1 << 40, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_gemm_bf16(16, 128, 64, 0, 1 << 41, 1 << 42, None) == B.H3BLK_ERR_INVALID_ARG


def test_modulation_producer_validation_before_gpu():
    blk = j.H3Block(hi.TINY)
    base = 1 << 40
    w = B.h3blk_mod_weights(freq_dim=64, time_hidden=128, time_dim=64, w1=base, b1=base, w2=base, b2=base,
                            adaln_w=base, adaln_b=base)
    assert B.h3blk_modulation_scratch_bytes(blk.handle, w) == hi.TINY.n_t * (128 + 64) * 4
    # bad sizes
    w_bad = B.h3blk_mod_weights(freq_dim=60, time_hidden=128, time_dim=64)
    assert B.h3blk_modulation_table(blk.handle, w_bad, [0.1, 0.2], None, 0.0, base, base, 1 << 20,
                                    None) == B.H3BLK_ERR_UNSUPPORTED
    # missing second-time weights with a non-zero gate
    assert B.h3blk_modulation_table(blk.handle, w, [0.1, 0.2], [0.0, 0.0], 0.5, base, base, 1 << 20,
                                    None) == B.H3BLK_ERR_INVALID_ARG
    # gate outside [0, 1], scratch too small, null table
    assert B.h3blk_modulation_table(blk.handle, w, [0.1, 0.2], None, 1.5, base, base, 1 << 20, None) == \
        B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_modulation_table(blk.handle, w, [0.1, 0.2], None, 0.0, base, base, 16, None) == \
        B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_modulation_table(blk.handle, w, [0.1, 0.2], None, 0.0, 0, base, 1 << 20, None) == \
        B.H3BLK_ERR_INVALID_ARG


# ---------------------------------------------------------------- model shell

def _fake_model(n_layers=2, n_refiner=1, video_in=16, audio_in=8, text_dim=128):
    mc = B.h3blk_model_config(n_layers=n_layers, n_refiner=n_refiner, video_in=video_in, audio_in=audio_in,
                              text_dim=text_dim, final_norm_eps=1e-5)
    base = 1 << 40
    p = lambda k: base + (k << 28)  # noqa: E731  fake, 16-byte aligned device addresses
    time = B.h3blk_mod_weights(freq_dim=64, time_hidden=128, time_dim=64, w1=p(1), b1=p(2), w2=p(3), b2=p(4))
    blockw = lambda k: B.h3blk_weights(wqkv=p(k), q_gain=p(k + 1), k_gain=p(k + 2), wo=p(k + 3),  # noqa: E731
                                       w13=p(k + 4), w2=p(k + 5))
    layers = (B.h3blk_layer_weights * 2)(*[B.h3blk_layer_weights(w=blockw(20 + 10 * i), adaln_w=p(27 + 10 * i),
                                                                 adaln_b=p(28 + 10 * i)) for i in range(2)])
    refiner = (B.h3blk_layer_weights * 1)(B.h3blk_layer_weights(w=blockw(60), adaln_w=p(67), adaln_b=p(68)))
    w = B.h3blk_model_weights(time=time, layers=layers, refiner=refiner, refiner_gain=p(70), out_adaln_w=p(71),
                              out_adaln_b=p(72), proj_in_w=p(73), proj_in_b=p(74), audio_in_w=p(75),
                              audio_in_b=p(76), ctx_w=p(77), ctx_b=p(78), proj_out_w=p(79), proj_out_b=p(80),
                              audio_out_w=p(81), audio_out_b=p(82))
    inp = B.h3blk_model_inputs(n_rows=320, n_video=192, n_audio=32, n_text=64, tag=p(90), tidx=p(91), pos=p(92),
                               video_idx=p(93), audio_idx=p(94), text_idx=p(95), video=p(96), audio=p(97),
                               text=p(98), t_now=p(99), t_end=None, gate=0.0)
    return mc, w, inp, p


def _model_call(blk, mc, w, inp, p, ws_bytes=None, video_out=None, audio_out=None, ws=None):
    if ws_bytes is None:
        ws_bytes = B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, inp.n_rows, inp.n_text)
    return B.h3blk_model_forward(blk.handle, mc, w, inp, p(100) if video_out is None else video_out,
                                 p(101) if audio_out is None else audio_out, p(102) if ws is None else ws,
                                 ws_bytes, None)


def test_model_workspace_layout():
    blk = j.H3Block(hi.TINY)
    mc, w, inp, p = _fake_model()
    full = B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 64)
    no_text = B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 0)
    C = hi.TINY.hidden
    # two packed sequences and the block workspace at least; text buffers on top
    assert no_text >= 2 * 320 * C * 2 + blk.workspace_bytes(320)
    assert full >= no_text + 2 * 64 * C * 2
    with pytest.raises(B.H3BlkError):
        B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 321)


def test_model_forward_passes_validation_with_fake_pointers():
    """A well-formed call gets through every host check and only fails at
    the first CUDA call (no device here)."""
    blk = j.H3Block(hi.TINY)
    mc, w, inp, p = _fake_model()
    assert _model_call(blk, mc, w, inp, p) == B.H3BLK_ERR_CUDA


@pytest.mark.parametrize("case,status", [
    ("counts_exceed_rows", B.H3BLK_ERR_INVALID_ARG),
    ("negative_count", B.H3BLK_ERR_INVALID_ARG),
    ("video_in_not_multiple_of_4", B.H3BLK_ERR_UNSUPPORTED),
    ("video_in_too_wide", B.H3BLK_ERR_UNSUPPORTED),
    ("text_dim_not_multiple_of_64", B.H3BLK_ERR_UNSUPPORTED),
    ("null_layers", B.H3BLK_ERR_INVALID_ARG),
    ("layer_missing_weight", B.H3BLK_ERR_INVALID_ARG),
    ("gate_without_t_end", B.H3BLK_ERR_INVALID_ARG),
    ("gate_out_of_range", B.H3BLK_ERR_INVALID_ARG),
    ("workspace_too_small", B.H3BLK_ERR_INVALID_ARG),
    ("misaligned_video", B.H3BLK_ERR_INVALID_ARG),
    ("null_video_out", B.H3BLK_ERR_INVALID_ARG),
    ("null_text_with_text_rows", B.H3BLK_ERR_INVALID_ARG),
])
def test_model_forward_rejects_bad_arguments(case, status):
    blk = j.H3Block(hi.TINY)
    kw = {}
    mc_kw = {}
    if case == "video_in_not_multiple_of_4":
        mc_kw["video_in"] = 6
    if case == "video_in_too_wide":
        mc_kw["video_in"] = 132
    if case == "text_dim_not_multiple_of_64":
        mc_kw["text_dim"] = 100
    mc, w, inp, p = _fake_model(**mc_kw)
    if case == "counts_exceed_rows":
        inp.n_text = 100
    if case == "negative_count":
        inp.n_audio = -1
    if case == "null_layers":
        w.layers = None
    if case == "layer_missing_weight":
        w.layers[1].w.wo = None
    if case == "gate_without_t_end":
        inp.gate = 0.5
        w.time.w1_r = w.time.b1_r = w.time.w2_r = w.time.b2_r = p(5)
    if case == "gate_out_of_range":
        inp.gate = 1.5
    if case == "workspace_too_small":
        kw["ws_bytes"] = 4096
    if case == "misaligned_video":
        inp.video = p(96) + 4
    if case == "null_video_out":
        kw["video_out"] = 0
    if case == "null_text_with_text_rows":
        inp.text = None
    if case in ("video_in_not_multiple_of_4", "video_in_too_wide", "text_dim_not_multiple_of_64"):
        kw["ws_bytes"] = 1 << 40
    assert _model_call(blk, mc, w, inp, p, **kw) == status


def test_model_graph_create_validates_before_capture():
    blk = j.H3Block(hi.TINY)
    mc, w, inp, p = _fake_model()
    inp.n_video = 400
    with pytest.raises(B.H3BlkError) as e:
        B.h3blk_model_graph_create(blk.handle, mc, w, inp, p(100), p(101), p(102), 1 << 40)
    assert e.value.status == B.H3BLK_ERR_INVALID_ARG
    assert B.h3blk_graph_launch(None, None) == B.H3BLK_ERR_INVALID_ARG
    B.h3blk_graph_destroy(None)   # no-op


# ---------------------------------------------------------------- sequence parallelism

def test_ulysses_sizes_and_group_checks():
    blk = j.H3Block(hi.TINY)   # 6 heads of 64
    q, o = B.h3blk_ulysses_buffer_bytes(blk.handle, 320, 2)
    assert q == 320 * 3 * 3 * 64 * 2 and o == 160 * 6 * 64 * 2
    assert B.h3blk_ulysses_workspace_bytes(blk.handle, 320, 2) < blk.workspace_bytes(320)
    for n, world in ((320, 4), (322, 3)):
        with pytest.raises(B.H3BlkError) as e:
            B.h3blk_ulysses_buffer_bytes(blk.handle, n, world)
        assert e.value.status == B.H3BLK_ERR_UNSUPPORTED
    with pytest.raises(B.H3BlkError):
        B.h3blk_ulysses_workspace_bytes(blk.handle, 320, 9)


def _fake_ulysses(world=2, rank=0):
    base = 1 << 40
    p = lambda k: base + (k << 28)  # noqa: E731
    u = B.h3blk_ulysses(world=world, rank=rank)
    for d in range(world):
        u.qkv[d] = p(40 + d)
        u.o[d] = p(50 + d)
    w = B.h3blk_weights(wqkv=p(1), q_gain=p(2), k_gain=p(3), wo=p(4), w13=p(5), w2=p(6))
    return u, w, p


@pytest.mark.parametrize("case,status", [
    ("ok", B.H3BLK_ERR_CUDA),                     # passes every host check, fails at the first CUDA call
    ("rank_out_of_group", B.H3BLK_ERR_INVALID_ARG),
    ("missing_peer_qkv", B.H3BLK_ERR_INVALID_ARG),
    ("misaligned_peer", B.H3BLK_ERR_INVALID_ARG),
    ("workspace_too_small", B.H3BLK_ERR_INVALID_ARG),
    ("world_not_dividing_heads", B.H3BLK_ERR_UNSUPPORTED),
])
def test_ulysses_phases_validate_before_gpu(case, status):
    blk = j.H3Block(hi.TINY)
    u, w, p = _fake_ulysses()
    ws = B.h3blk_ulysses_workspace_bytes(blk.handle, 320, 2)
    if case == "rank_out_of_group":
        u.rank = 2
    if case == "missing_peer_qkv":
        u.qkv[1] = None
    if case == "misaligned_peer":
        u.qkv[1] = p(41) + 8
        u.o[1] = p(51) + 8
    if case == "workspace_too_small":
        ws = 64
    if case == "world_not_dividing_heads":
        u.world = 4
        u.qkv[2], u.qkv[3], u.o[2], u.o[3] = p(42), p(43), p(52), p(53)
    st = B.h3blk_ulysses_qkv(blk.handle, 320, u, p(10), p(11), p(12), p(13), p(14), w, p(20), ws, None)
    assert st == status
    if case in ("ok", "rank_out_of_group", "misaligned_peer", "workspace_too_small", "world_not_dividing_heads"):
        assert B.h3blk_ulysses_attention(blk.handle, 320, u, p(11), p(20), ws, None) == status
        # the output phase reads only this rank's own o buffer
        st_out = B.H3BLK_ERR_CUDA if case == "misaligned_peer" else status
        assert B.h3blk_ulysses_out(blk.handle, 320, u, p(10), p(11), p(12), p(14), w, p(15), p(20), ws,
                                   None) == st_out


def test_attention_density_setting():
    blk = j.H3Block(hi.TINY)
    dense = blk.workspace_bytes(320)
    for bad in (0.0, -0.5, 1.5, float("nan")):
        assert B.h3blk_set_attention_density(blk.handle, bad) == B.H3BLK_ERR_INVALID_ARG
    blk.set_attention_density(0.25)
    sparse = blk.workspace_bytes(320)
    n_tiles = 3
    assert sparse >= dense + 2 * (n_tiles + 1) // 2 * 6 * (1 + n_tiles) * 4
    off, nb = B.h3blk_stage_view(blk.handle, 320, "KV_LIST")
    assert nb == 2 * 6 * (1 + n_tiles) * 4
    # sequence parallelism is single-mode: block-sparse is refused there
    with pytest.raises(B.H3BlkError) as e:
        B.h3blk_ulysses_workspace_bytes(blk.handle, 320, 2)
    assert e.value.status == B.H3BLK_ERR_UNSUPPORTED
    blk.set_attention_density(1.0)
    assert blk.workspace_bytes(320) == dense


@pytest.mark.parametrize("limit_ms,word", [(0, 256), (2001, 256), (50, 0), (50, 258)])
def test_selftest_wait_validates_before_gpu(limit_ms, word):
    st = C.c_int32()
    rc = B._lib.h3blk_selftest_wait(0, limit_ms, word, None, C.byref(st))
    assert rc == B.H3BLK_ERR_INVALID_ARG


def test_block_sparse_mode_sizes_block_and_model_workspaces():
    """Block-sparse attention needs its pooled sums and kept-tile lists in the
    workspace: the block's and the model's sizes both grow with the mode, and
    density 1 is dense again."""
    blk = j.H3Block(hi.TINY)
    mc, w, _, _ = _fake_model()
    dense_blk = blk.workspace_bytes(320)
    dense_model = B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 64)
    blk.set_attention_density(0.3)
    assert blk.workspace_bytes(320) > dense_blk
    assert B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 64) > dense_model
    blk.set_attention_density(1.0)
    assert blk.workspace_bytes(320) == dense_blk
    assert B.h3blk_model_workspace_bytes(blk.handle, mc, w.time, 320, 64) == dense_model


def test_debug_accumulator_dump_validation():
    """The test-only s32 accumulator dump: W8A8 handles only, gemm in -1..3,
    a non-null 16-byte aligned buffer; -1 switches it off."""
    from dataclasses import replace
    lib = B._lib
    bf = j.H3Block(hi.TINY)
    assert lib.h3blk_set_debug_accumulators(bf.handle, 0, 1 << 20, 4096) == B.H3BLK_ERR_UNSUPPORTED
    assert lib.h3blk_set_debug_accumulators(bf.handle, -1, None, 0) == B.H3BLK_OK
    q = j.H3Block(replace(hi.TINY, quant=1))
    for gemm in (-2, 4):
        assert lib.h3blk_set_debug_accumulators(q.handle, gemm, 1 << 20, 4096) == B.H3BLK_ERR_INVALID_ARG
    assert lib.h3blk_set_debug_accumulators(q.handle, 0, None, 4096) == B.H3BLK_ERR_INVALID_ARG
    assert lib.h3blk_set_debug_accumulators(q.handle, 0, (1 << 20) + 4, 4096) == B.H3BLK_ERR_INVALID_ARG
    assert lib.h3blk_set_debug_accumulators(q.handle, 0, 1 << 20, 0) == B.H3BLK_ERR_INVALID_ARG
    for gemm in range(4):
        assert lib.h3blk_set_debug_accumulators(q.handle, gemm, 1 << 20, 4096) == B.H3BLK_OK
    assert lib.h3blk_set_debug_accumulators(q.handle, -1, None, 0) == B.H3BLK_OK
    assert lib.h3blk_set_debug_accumulators(None, -1, None, 0) == B.H3BLK_ERR_INVALID_ARG


def test_noalloc_check_validates_status_pointer():
    assert B._lib.h3blk_attention_noalloc_check(None, None) == B.H3BLK_ERR_INVALID_ARG
