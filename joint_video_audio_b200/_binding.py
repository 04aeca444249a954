"""ctypes binding of libh3blk (include/h3blk.h): the same entry points under
the same names, plus argument marshalling for torch tensors. Every step of the
block runs in the library's CUDA kernels; nothing here computes.

If libh3blk.so is missing the import fails: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libh3blk.so")

H3BLK_OK = 0
H3BLK_ERR_INVALID_ARG = 1
H3BLK_ERR_UNSUPPORTED = 2
H3BLK_ERR_CUDA = 3
H3BLK_ERR_TIMEOUT = 4
H3BLK_ERR_BAD_INDEX = 5

STAGES = ["H1", "QKV", "O", "X1", "H2", "A", "H1_Q8", "H1_SCALE", "O_Q8", "O_SCALE",
          "H2_Q8", "H2_SCALE", "A_Q8", "A_SCALE", "ERROR", "KV_LIST"]
STAGE = {name: i for i, name in enumerate(STAGES)}

# every symbol include/h3blk.h declares
EXPORTS = ["h3blk_create", "h3blk_destroy", "h3blk_workspace_bytes", "h3blk_stage_view", "h3blk_forward",
           "h3blk_check", "h3blk_int8_weights_bytes", "h3blk_prepare_int8_weights", "h3blk_rotate_quantize",
           "h3blk_gemm_s8_s32", "h3blk_gemm_bf16", "h3blk_error_string", "h3blk_version",
           "h3blk_set_kernel_events", "h3blk_attention_noalloc", "h3blk_attention_noalloc_check",
           "h3blk_modulation_scratch_bytes",
           "h3blk_modulation_table", "h3blk_model_workspace_bytes", "h3blk_model_forward", "h3blk_model_check",
           "h3blk_model_graph_create", "h3blk_graph_launch", "h3blk_graph_info", "h3blk_graph_destroy",
           "h3blk_ulysses_buffer_bytes", "h3blk_ulysses_workspace_bytes", "h3blk_ulysses_qkv",
           "h3blk_ulysses_attention", "h3blk_ulysses_out", "h3blk_set_attention_density",
           "h3blk_selftest_wait", "h3blk_set_debug_accumulators"]

H3BLK_MAX_RANKS = 8

H3BLK_TIMING_POINTS = 11
TIMING_INTERVALS = ["prep", "norm1", "qkv_gemm", "attention", "quant_o", "out_proj_gemm", "norm2",
                    "ffn_up_gemm", "quant_a", "ffn_down_gemm"]


class h3blk_config(C.Structure):
    _fields_ = [("hidden", C.c_int), ("heads", C.c_int), ("head_dim", C.c_int), ("ffn", C.c_int),
                ("n_tags", C.c_int), ("n_t", C.c_int), ("rope_pairs_t", C.c_int), ("rope_pairs_h", C.c_int),
                ("rope_pairs_w", C.c_int), ("rope_theta", C.c_float), ("norm_eps", C.c_float),
                ("qk_norm_eps", C.c_float), ("quant", C.c_int)]


class h3blk_weights(C.Structure):
    _fields_ = [("wqkv", C.c_void_p), ("q_gain", C.c_void_p), ("k_gain", C.c_void_p), ("wo", C.c_void_p),
                ("w13", C.c_void_p), ("w2", C.c_void_p), ("s_qkv", C.c_void_p), ("s_o", C.c_void_p),
                ("s_13", C.c_void_p), ("s_2", C.c_void_p)]


class h3blk_mod_weights(C.Structure):
    _fields_ = [("freq_dim", C.c_int), ("time_hidden", C.c_int), ("time_dim", C.c_int),
                ("w1", C.c_void_p), ("b1", C.c_void_p), ("w2", C.c_void_p), ("b2", C.c_void_p),
                ("w1_r", C.c_void_p), ("b1_r", C.c_void_p), ("w2_r", C.c_void_p), ("b2_r", C.c_void_p),
                ("adaln_w", C.c_void_p), ("adaln_b", C.c_void_p)]


class h3blk_model_config(C.Structure):
    _fields_ = [("n_layers", C.c_int), ("n_refiner", C.c_int), ("video_in", C.c_int), ("audio_in", C.c_int),
                ("text_dim", C.c_int), ("final_norm_eps", C.c_float)]


class h3blk_layer_weights(C.Structure):
    _fields_ = [("w", h3blk_weights), ("adaln_w", C.c_void_p), ("adaln_b", C.c_void_p)]


class h3blk_model_weights(C.Structure):
    _fields_ = [("time", h3blk_mod_weights), ("layers", C.POINTER(h3blk_layer_weights)),
                ("refiner", C.POINTER(h3blk_layer_weights)), ("refiner_gain", C.c_void_p),
                ("out_adaln_w", C.c_void_p), ("out_adaln_b", C.c_void_p),
                ("proj_in_w", C.c_void_p), ("proj_in_b", C.c_void_p),
                ("audio_in_w", C.c_void_p), ("audio_in_b", C.c_void_p),
                ("ctx_w", C.c_void_p), ("ctx_b", C.c_void_p),
                ("proj_out_w", C.c_void_p), ("proj_out_b", C.c_void_p),
                ("audio_out_w", C.c_void_p), ("audio_out_b", C.c_void_p)]


class h3blk_model_inputs(C.Structure):
    _fields_ = [("n_rows", C.c_int64), ("n_video", C.c_int64), ("n_audio", C.c_int64), ("n_text", C.c_int64),
                ("tag", C.c_void_p), ("tidx", C.c_void_p), ("pos", C.c_void_p),
                ("video_idx", C.c_void_p), ("audio_idx", C.c_void_p), ("text_idx", C.c_void_p),
                ("video", C.c_void_p), ("audio", C.c_void_p), ("text", C.c_void_p),
                ("t_now", C.c_void_p), ("t_end", C.c_void_p), ("gate", C.c_float)]


class h3blk_ulysses(C.Structure):
    _fields_ = [("world", C.c_int), ("rank", C.c_int), ("qkv", C.c_void_p * 8), ("o", C.c_void_p * 8)]


class H3BlkError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: status {status} ({error_string(status)})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing; build it with `python joint_video_audio_b200/build.py`")
    lib = C.CDLL(LIB_PATH)
    vp, i64, i32, sz = C.c_void_p, C.c_int64, C.c_int, C.c_size_t
    sig = {
        "h3blk_create": (i32, [C.POINTER(h3blk_config), C.POINTER(vp)]),
        "h3blk_destroy": (None, [vp]),
        "h3blk_workspace_bytes": (i32, [vp, i64, C.POINTER(sz)]),
        "h3blk_stage_view": (i32, [vp, i64, i32, C.POINTER(sz), C.POINTER(sz)]),
        "h3blk_forward": (i32, [vp, i64, vp, vp, vp, vp, vp, C.POINTER(h3blk_weights), vp, vp, sz, vp]),
        "h3blk_check": (i32, [vp, i64, vp, vp, C.POINTER(i32)]),
        "h3blk_int8_weights_bytes": (i32, [vp, C.POINTER(sz)]),
        "h3blk_prepare_int8_weights": (i32, [vp, C.POINTER(h3blk_weights), vp, sz, C.POINTER(h3blk_weights), vp]),
        "h3blk_rotate_quantize": (i32, [i64, i32, vp, vp, vp, vp]),
        "h3blk_gemm_s8_s32": (i32, [i64, i32, i32, vp, vp, vp, vp]),
        "h3blk_gemm_bf16": (i32, [i64, i32, i32, vp, vp, vp, vp]),
        "h3blk_error_string": (C.c_char_p, [i32]),
        "h3blk_version": (i32, []),
        "h3blk_set_kernel_events": (i32, [vp, C.POINTER(vp), i32]),
        "h3blk_attention_noalloc": (i32, [i64, i32, i32, i32, i32, vp, vp, vp, vp, vp]),
        "h3blk_attention_noalloc_check": (i32, [vp, C.POINTER(i32)]),
        "h3blk_selftest_wait": (i32, [i32, i32, vp, vp, C.POINTER(i32)]),
        "h3blk_set_debug_accumulators": (i32, [vp, i32, vp, C.c_size_t]),
        "h3blk_modulation_scratch_bytes": (i32, [vp, C.POINTER(h3blk_mod_weights), C.POINTER(sz)]),
        "h3blk_modulation_table": (i32, [vp, C.POINTER(h3blk_mod_weights), C.POINTER(C.c_float),
                                          C.POINTER(C.c_float), C.c_float, vp, vp, sz, vp]),
        "h3blk_model_workspace_bytes": (i32, [vp, C.POINTER(h3blk_model_config), C.POINTER(h3blk_mod_weights),
                                               i64, i64, C.POINTER(sz)]),
        "h3blk_model_forward": (i32, [vp, C.POINTER(h3blk_model_config), C.POINTER(h3blk_model_weights),
                                       C.POINTER(h3blk_model_inputs), vp, vp, vp, sz, vp]),
        "h3blk_model_check": (i32, [vp, vp, C.POINTER(i32)]),
        "h3blk_model_graph_create": (i32, [vp, C.POINTER(h3blk_model_config), C.POINTER(h3blk_model_weights),
                                            C.POINTER(h3blk_model_inputs), vp, vp, vp, sz, C.POINTER(vp)]),
        "h3blk_graph_launch": (i32, [vp, vp]),
        "h3blk_graph_info": (i32, [vp, C.POINTER(i32), C.POINTER(i32)]),
        "h3blk_graph_destroy": (None, [vp]),
        "h3blk_set_attention_density": (i32, [vp, C.c_float]),
        "h3blk_ulysses_buffer_bytes": (i32, [vp, i64, i32, C.POINTER(sz), C.POINTER(sz)]),
        "h3blk_ulysses_workspace_bytes": (i32, [vp, i64, i32, C.POINTER(sz)]),
        "h3blk_ulysses_qkv": (i32, [vp, i64, C.POINTER(h3blk_ulysses), vp, vp, vp, vp, vp, C.POINTER(h3blk_weights),
                                    vp, sz, vp]),
        "h3blk_ulysses_attention": (i32, [vp, i64, C.POINTER(h3blk_ulysses), vp, vp, sz, vp]),
        "h3blk_ulysses_out": (i32, [vp, i64, C.POINTER(h3blk_ulysses), vp, vp, vp, vp, C.POINTER(h3blk_weights), vp,
                                    vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


_lib = _load()


def _check(fn, status):
    if status != H3BLK_OK:
        raise H3BlkError(fn, status)


# ---------------------------------------------------------------- raw entry points

def error_string(status: int) -> str:
    return _lib.h3blk_error_string(status).decode()


def h3blk_error_string(status: int) -> str:
    return error_string(status)


def h3blk_version() -> int:
    return _lib.h3blk_version()


def h3blk_create(cfg: h3blk_config) -> int:
    h = C.c_void_p()
    _check("h3blk_create", _lib.h3blk_create(C.byref(cfg), C.byref(h)))
    return h.value


def h3blk_create_status(cfg) -> int:
    """Status code of h3blk_create (for argument-validation tests)."""
    h = C.c_void_p()
    st = _lib.h3blk_create(C.byref(cfg) if cfg is not None else None, C.byref(h))
    if st == H3BLK_OK:
        _lib.h3blk_destroy(h)
    return st


def h3blk_destroy(handle: int) -> None:
    _lib.h3blk_destroy(handle)


def h3blk_workspace_bytes(handle: int, n_rows: int) -> int:
    n = C.c_size_t()
    _check("h3blk_workspace_bytes", _lib.h3blk_workspace_bytes(handle, n_rows, C.byref(n)))
    return n.value


def h3blk_stage_view(handle: int, n_rows: int, stage) -> tuple[int, int]:
    st = STAGE[stage] if isinstance(stage, str) else int(stage)
    off, nb = C.c_size_t(), C.c_size_t()
    _check("h3blk_stage_view", _lib.h3blk_stage_view(handle, n_rows, st, C.byref(off), C.byref(nb)))
    return off.value, nb.value


def h3blk_forward(handle, n_rows, x, tag, tidx, pos, mod_table, weights: h3blk_weights, out, workspace,
                  workspace_bytes, stream) -> int:
    """Raw call; pointers are ints. Returns the status code."""
    return _lib.h3blk_forward(handle, n_rows, x, tag, tidx, pos, mod_table, C.byref(weights), out, workspace,
                              workspace_bytes, stream)


def h3blk_check(handle, n_rows, workspace, stream) -> int:
    st = C.c_int()
    _check("h3blk_check", _lib.h3blk_check(handle, n_rows, workspace, stream, C.byref(st)))
    return st.value


def h3blk_int8_weights_bytes(handle) -> int:
    n = C.c_size_t()
    _check("h3blk_int8_weights_bytes", _lib.h3blk_int8_weights_bytes(handle, C.byref(n)))
    return n.value


def h3blk_prepare_int8_weights(handle, bf16_in: h3blk_weights, blob, blob_bytes, stream) -> h3blk_weights:
    out = h3blk_weights()
    _check("h3blk_prepare_int8_weights",
           _lib.h3blk_prepare_int8_weights(handle, C.byref(bf16_in), blob, blob_bytes, C.byref(out), stream))
    return out


def h3blk_rotate_quantize(rows, K, in_bf16, out_q, out_scale, stream) -> int:
    return _lib.h3blk_rotate_quantize(rows, K, in_bf16, out_q, out_scale, stream)


def h3blk_gemm_s8_s32(M, N, K, A, B, Cp, stream) -> int:
    return _lib.h3blk_gemm_s8_s32(M, N, K, A, B, Cp, stream)


def h3blk_gemm_bf16(M, N, K, A, B, Cp, stream) -> int:
    return _lib.h3blk_gemm_bf16(M, N, K, A, B, Cp, stream)


def h3blk_set_kernel_events(handle, events) -> None:
    """events: sequence of H3BLK_TIMING_POINTS raw cudaEvent_t values (ints), or None."""
    if not events:
        _check("h3blk_set_kernel_events", _lib.h3blk_set_kernel_events(handle, None, 0))
        return
    arr = (C.c_void_p * len(events))(*events)
    _check("h3blk_set_kernel_events", _lib.h3blk_set_kernel_events(handle, arr, len(events)))


def h3blk_attention_noalloc(n_rows, heads, head_dim, n_tags, n_t, qkv, tag, tidx, o, stream) -> int:
    """Raw call (pointers are ints); returns the status code. Uses the
    library's fixed device scratch instead of a caller workspace."""
    return _lib.h3blk_attention_noalloc(n_rows, heads, head_dim, n_tags, n_t, qkv, tag, tidx, o, stream)


def h3blk_attention_noalloc_check(stream) -> int:
    """Synchronises `stream` and returns the device-side status of the last
    h3blk_attention_noalloc call (H3BLK_OK, H3BLK_ERR_BAD_INDEX or
    H3BLK_ERR_TIMEOUT)."""
    st = C.c_int32()
    _check("h3blk_attention_noalloc_check", _lib.h3blk_attention_noalloc_check(stream, C.byref(st)))
    return st.value


def h3blk_selftest_wait(complete: bool, limit_ms: int, word, stream) -> int:
    """Test-only: one bounded pipeline wait on a barrier that completes
    (complete=True) or never does; returns the status h3blk_check would give
    (H3BLK_OK or H3BLK_ERR_TIMEOUT). `word` is a device int32 pointer."""
    st = C.c_int32()
    _check("h3blk_selftest_wait", _lib.h3blk_selftest_wait(1 if complete else 0, limit_ms, word, stream, C.byref(st)))
    return st.value


def h3blk_set_debug_accumulators(handle, gemm: int, buf, nbytes: int) -> None:
    """Test-only (W8A8): later forwards also dump int8 GEMM `gemm`'s raw int32
    accumulators (0 QKV, 1 out-proj, 2 FFN up, 3 FFN down; -1 off) to `buf`."""
    _check("h3blk_set_debug_accumulators", _lib.h3blk_set_debug_accumulators(handle, gemm, buf, nbytes))


def h3blk_modulation_scratch_bytes(handle, w: h3blk_mod_weights) -> int:
    n = C.c_size_t()
    _check("h3blk_modulation_scratch_bytes", _lib.h3blk_modulation_scratch_bytes(handle, C.byref(w), C.byref(n)))
    return n.value


def h3blk_modulation_table(handle, w: h3blk_mod_weights, t_now, t_end, gate, table, scratch, scratch_bytes,
                           stream) -> int:
    """t_now / t_end: host sequences of floats (t_end may be None). Returns the status code."""
    tn = (C.c_float * len(t_now))(*[float(v) for v in t_now])
    te = (C.c_float * len(t_end))(*[float(v) for v in t_end]) if t_end is not None else None
    return _lib.h3blk_modulation_table(handle, C.byref(w), tn, te, C.c_float(gate), table, scratch, scratch_bytes,
                                       stream)


def h3blk_model_workspace_bytes(handle, mc: h3blk_model_config, time: h3blk_mod_weights, n_rows, n_text) -> int:
    n = C.c_size_t()
    _check("h3blk_model_workspace_bytes",
           _lib.h3blk_model_workspace_bytes(handle, C.byref(mc), C.byref(time), n_rows, n_text, C.byref(n)))
    return n.value


def h3blk_model_forward(handle, mc, w, inp, video_out, audio_out, workspace, workspace_bytes, stream) -> int:
    """Raw call (pointers are ints); returns the status code."""
    return _lib.h3blk_model_forward(handle, C.byref(mc), C.byref(w), C.byref(inp), video_out, audio_out, workspace,
                                    workspace_bytes, stream)


def h3blk_model_check(workspace, stream) -> int:
    st = C.c_int()
    _check("h3blk_model_check", _lib.h3blk_model_check(workspace, stream, C.byref(st)))
    return st.value


def h3blk_model_graph_create(handle, mc, w, inp, video_out, audio_out, workspace, workspace_bytes) -> int:
    g = C.c_void_p()
    _check("h3blk_model_graph_create",
           _lib.h3blk_model_graph_create(handle, C.byref(mc), C.byref(w), C.byref(inp), video_out, audio_out,
                                         workspace, workspace_bytes, C.byref(g)))
    return g.value


def h3blk_graph_launch(graph, stream) -> int:
    return _lib.h3blk_graph_launch(graph, stream)


def h3blk_graph_info(graph) -> tuple[int, int]:
    k, o = C.c_int(), C.c_int()
    _check("h3blk_graph_info", _lib.h3blk_graph_info(graph, C.byref(k), C.byref(o)))
    return k.value, o.value


def h3blk_graph_destroy(graph) -> None:
    _lib.h3blk_graph_destroy(graph)


def h3blk_ulysses_buffer_bytes(handle, n_rows, world) -> tuple[int, int]:
    q, o = C.c_size_t(), C.c_size_t()
    _check("h3blk_ulysses_buffer_bytes", _lib.h3blk_ulysses_buffer_bytes(handle, n_rows, world, C.byref(q), C.byref(o)))
    return q.value, o.value


def h3blk_ulysses_workspace_bytes(handle, n_rows, world) -> int:
    n = C.c_size_t()
    _check("h3blk_ulysses_workspace_bytes", _lib.h3blk_ulysses_workspace_bytes(handle, n_rows, world, C.byref(n)))
    return n.value


def h3blk_ulysses_qkv(handle, n_rows, u, x_local, tag, tidx, pos, table, w, workspace, workspace_bytes, stream) -> int:
    return _lib.h3blk_ulysses_qkv(handle, n_rows, C.byref(u), x_local, tag, tidx, pos, table, C.byref(w), workspace,
                                  workspace_bytes, stream)


def h3blk_ulysses_attention(handle, n_rows, u, tag, workspace, workspace_bytes, stream) -> int:
    return _lib.h3blk_ulysses_attention(handle, n_rows, C.byref(u), tag, workspace, workspace_bytes, stream)


def h3blk_ulysses_out(handle, n_rows, u, x_local, tag, tidx, table, w, out_local, workspace, workspace_bytes,
                      stream) -> int:
    return _lib.h3blk_ulysses_out(handle, n_rows, C.byref(u), x_local, tag, tidx, table, C.byref(w), out_local,
                                  workspace, workspace_bytes, stream)


def h3blk_set_attention_density(handle, density) -> int:
    return _lib.h3blk_set_attention_density(handle, C.c_float(density))
