"""ctypes binding of the C ABI in include/hymba.h (argument marshalling only).

Every function of the header is exposed under its own name.  Loading fails
loudly when libhymba.so is missing: there is no fallback implementation.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhymba.so")

HYMBA_OK = 0
HYMBA_ERR_INVALID_ARG = 1
HYMBA_ERR_UNSUPPORTED = 2
HYMBA_ERR_WORKSPACE = 3
HYMBA_ERR_NOT_BOUND = 4
HYMBA_ERR_CUDA = 5
HYMBA_ERR_TIMEOUT = 6
HYMBA_ERR_DEVICE = 7
HYMBA_F32 = 0
HYMBA_BF16 = 1


class hymba_layer_config(C.Structure):
    _fields_ = [("d_model", C.c_int), ("n_heads", C.c_int), ("n_kv_heads", C.c_int),
                ("head_dim_qk", C.c_int), ("head_dim_v", C.c_int), ("d_inner", C.c_int),
                ("d_state", C.c_int), ("d_conv", C.c_int), ("dt_rank", C.c_int),
                ("n_meta", C.c_int), ("window", C.c_int), ("is_global", C.c_int),
                ("dtype", C.c_int), ("rms_eps", C.c_float), ("softmax_scale", C.c_float),
                ("rope_base", C.c_float), ("branch_chunks", C.c_int)]


class hymba_layer_weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("w_in", "conv_w", "conv_b", "w_x", "w_dt", "b_dt",
                                          "a_log", "d_skip", "beta_attn", "beta_ssm", "w_out")]


class hymba_kv_seq(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("batch", C.c_int), ("rows", C.c_int),
                ("owner", C.c_uint64)]


class hymba_kv_cache(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("batch", C.c_int), ("capacity", C.c_int),
                ("owner", C.c_uint64)]


class hymba_ssm_cache(C.Structure):
    _fields_ = [("h", C.c_void_p), ("conv", C.c_void_p)]


class hymba_meta_cache(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("h", C.c_void_p), ("conv", C.c_void_p),
                ("y", C.c_void_p), ("owner", C.c_uint64)]


class hymba_block_weights(C.Structure):
    _fields_ = [("norm1", C.c_void_p), ("norm2", C.c_void_p), ("w_gate_up", C.c_void_p),
                ("w_down", C.c_void_p), ("mlp_hidden", C.c_int)]


class hymba_prefill_layout(C.Structure):
    _fields_ = [(n, C.c_size_t) for n in ("q", "x_ssm", "gate", "u", "xdbl", "delta", "y_ssm",
                                          "o_attn", "fused", "rope", "sched", "total")]


class hymba_profile_entry(C.Structure):
    _fields_ = [("name", C.c_char * 32), ("calls", C.c_int), ("kernels", C.c_int),
                ("total_ms", C.c_double)]


class HymbaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


_lib = None

# name -> (restype, argtypes)
_SIGS = {
    "hymba_layer_create": (C.c_int, [C.POINTER(hymba_layer_config), C.POINTER(hymba_layer_weights),
                                     C.POINTER(C.c_void_p)]),
    "hymba_layer_destroy": (None, [C.c_void_p]),
    "hymba_layer_is_consumer": (C.c_int, [C.c_void_p]),
    "hymba_kv_share_bind": (C.c_int, [C.c_void_p, C.c_void_p]),
    "hymba_layer_prefill_workspace": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.POINTER(C.c_size_t)]),
    "hymba_layer_prefill_layout": (C.c_int, [C.c_void_p, C.c_int, C.c_int,
                                             C.POINTER(hymba_prefill_layout)]),
    "hymba_layer_prefill": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                      C.POINTER(hymba_kv_seq), C.POINTER(hymba_kv_cache),
                                      C.POINTER(hymba_ssm_cache), C.c_void_p, C.c_size_t, C.c_void_p]),
    "hymba_layer_meta_workspace": (C.c_int, [C.c_void_p, C.POINTER(C.c_size_t)]),
    "hymba_layer_meta_precompute": (C.c_int, [C.c_void_p, C.c_void_p, C.POINTER(hymba_meta_cache),
                                              C.POINTER(hymba_meta_cache), C.c_void_p, C.c_size_t,
                                              C.c_void_p]),
    "hymba_layer_prefill_cached_workspace": (C.c_int, [C.c_void_p, C.c_int, C.c_int,
                                                       C.POINTER(C.c_size_t)]),
    "hymba_layer_prefill_cached": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                             C.POINTER(hymba_meta_cache), C.POINTER(hymba_kv_seq),
                                             C.POINTER(hymba_kv_cache), C.POINTER(hymba_ssm_cache),
                                             C.c_void_p, C.c_size_t, C.c_void_p]),
    "hymba_block_prefill_workspace": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int, C.POINTER(C.c_size_t)]),
    "hymba_block_prefill": (C.c_int, [C.c_void_p, C.POINTER(hymba_block_weights), C.c_int, C.c_int,
                                      C.c_void_p, C.c_void_p, C.POINTER(hymba_kv_seq),
                                      C.POINTER(hymba_kv_cache), C.POINTER(hymba_ssm_cache), C.c_void_p,
                                      C.c_size_t, C.c_void_p]),
    "hymba_block_decode_workspace": (C.c_int, [C.c_void_p, C.c_int, C.c_int, C.c_int64, C.POINTER(C.c_size_t)]),
    "hymba_block_decode_step": (C.c_int, [C.c_void_p, C.POINTER(hymba_block_weights), C.c_int, C.c_int64,
                                          C.c_void_p, C.c_void_p, C.POINTER(hymba_kv_cache),
                                          C.POINTER(hymba_ssm_cache), C.c_void_p, C.c_size_t, C.c_void_p]),
    "hymba_layer_decode_workspace": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.POINTER(C.c_size_t)]),
    "hymba_layer_decode_step": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_void_p, C.c_void_p,
                                          C.POINTER(hymba_kv_cache), C.POINTER(hymba_ssm_cache),
                                          C.c_void_p, C.c_size_t, C.c_void_p]),
    "hymba_stream_status": (C.c_int, [C.c_void_p]),
    "hymba_last_error": (C.c_char_p, []),
    "hymba_status_string": (C.c_char_p, [C.c_int]),
    "hymba_version": (C.c_char_p, []),
    "hymba_debug_mask_bitmap": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                          C.c_void_p, C.c_void_p]),
    "hymba_debug_decode_mask": (C.c_int, [C.c_int64, C.c_int, C.c_int, C.c_int, C.c_int, C.c_void_p,
                                          C.c_void_p]),
    "hymba_debug_exp2_poly": (C.c_int, [C.c_int, C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p]),
    "hymba_layer_decode_step_static": (C.c_int, [C.c_void_p, C.c_int, C.c_int64, C.c_void_p, C.c_void_p,
                                                 C.POINTER(hymba_kv_cache), C.POINTER(hymba_ssm_cache),
                                                 C.c_void_p]),
    "hymba_set_wait_limit": (C.c_int, [C.c_int64, C.POINTER(C.c_int64)]),
    "hymba_debug_stall_next_prefill": (C.c_int, [C.c_int]),
    "hymba_profile_enable": (C.c_int, [C.c_int]),
    "hymba_profile_collect": (C.c_int, [C.POINTER(hymba_profile_entry), C.c_int, C.POINTER(C.c_int)]),
}
EXPORTED = tuple(_SIGS)


def lib():
    """The loaded libhymba.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hybrid_attention_ssm_head_b200.build`")
        lib_ = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib_, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib_
    return _lib


def check(status: int, what: str = "") -> None:
    if status != HYMBA_OK:
        msg = lib().hymba_last_error().decode()
        name = lib().hymba_status_string(status).decode()
        raise HymbaError(status, f"{what}: {name}: {msg}")


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> int | None:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


# ---- the entry points, same names as the header ------------------------------------------

def hymba_layer_create(cfg: hymba_layer_config, w: hymba_layer_weights) -> int:
    out = C.c_void_p()
    check(lib().hymba_layer_create(C.byref(cfg), C.byref(w), C.byref(out)), "hymba_layer_create")
    return out.value


def hymba_layer_destroy(layer: int) -> None:
    lib().hymba_layer_destroy(layer)


def hymba_layer_is_consumer(layer: int) -> bool:
    return bool(lib().hymba_layer_is_consumer(layer))


def hymba_kv_share_bind(consumer: int, producer: int) -> None:
    check(lib().hymba_kv_share_bind(consumer, producer), "hymba_kv_share_bind")


def hymba_layer_prefill_workspace(layer: int, batch: int, n_tokens: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_layer_prefill_workspace(layer, batch, n_tokens, C.byref(out)),
          "hymba_layer_prefill_workspace")
    return out.value


def hymba_layer_prefill_layout(layer: int, batch: int, n_tokens: int) -> hymba_prefill_layout:
    out = hymba_prefill_layout()
    check(lib().hymba_layer_prefill_layout(layer, batch, n_tokens, C.byref(out)),
          "hymba_layer_prefill_layout")
    return out


def hymba_layer_prefill(layer: int, batch: int, n_tokens: int, x, y, kv: hymba_kv_seq,
                        kv_cache: hymba_kv_cache | None, ssm_cache: hymba_ssm_cache | None,
                        workspace, workspace_bytes: int, stream=None) -> None:
    check(lib().hymba_layer_prefill(
        layer, batch, n_tokens, _ptr(x), _ptr(y), C.byref(kv),
        C.byref(kv_cache) if kv_cache is not None else None,
        C.byref(ssm_cache) if ssm_cache is not None else None,
        _ptr(workspace), workspace_bytes, _stream(stream)), "hymba_layer_prefill")


def hymba_layer_meta_workspace(layer: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_layer_meta_workspace(layer, C.byref(out)), "hymba_layer_meta_workspace")
    return out.value


def hymba_layer_meta_precompute(layer: int, x_meta, meta: hymba_meta_cache,
                                producer_meta: hymba_meta_cache | None, workspace, workspace_bytes: int,
                                stream=None) -> None:
    check(lib().hymba_layer_meta_precompute(
        layer, _ptr(x_meta), C.byref(meta), C.byref(producer_meta) if producer_meta is not None else None,
        _ptr(workspace), workspace_bytes, _stream(stream)), "hymba_layer_meta_precompute")


def hymba_layer_prefill_cached_workspace(layer: int, batch: int, n_tokens: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_layer_prefill_cached_workspace(layer, batch, n_tokens, C.byref(out)),
          "hymba_layer_prefill_cached_workspace")
    return out.value


def hymba_layer_prefill_cached(layer: int, batch: int, n_tokens: int, x, y, meta: hymba_meta_cache,
                               kv: hymba_kv_seq, kv_cache: hymba_kv_cache | None,
                               ssm_cache: hymba_ssm_cache | None, workspace, workspace_bytes: int,
                               stream=None) -> None:
    check(lib().hymba_layer_prefill_cached(
        layer, batch, n_tokens, _ptr(x), _ptr(y), C.byref(meta), C.byref(kv),
        C.byref(kv_cache) if kv_cache is not None else None,
        C.byref(ssm_cache) if ssm_cache is not None else None,
        _ptr(workspace), workspace_bytes, _stream(stream)), "hymba_layer_prefill_cached")


def make_block_weights(w: dict) -> hymba_block_weights:
    """From device tensors norm1, norm2 [d] fp32, w_gate_up [2F, d] (rows interleaved), w_down [d, F]."""
    return hymba_block_weights(_ptr(w["norm1"]), _ptr(w["norm2"]), _ptr(w["w_gate_up"]), _ptr(w["w_down"]),
                               int(w["w_down"].shape[1]))


def hymba_block_prefill_workspace(layer: int, mlp_hidden: int, batch: int, n_tokens: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_block_prefill_workspace(layer, mlp_hidden, batch, n_tokens, C.byref(out)),
          "hymba_block_prefill_workspace")
    return out.value


def hymba_block_prefill(layer: int, bw: hymba_block_weights, batch: int, n_tokens: int, x, y, kv: hymba_kv_seq,
                        kv_cache: hymba_kv_cache | None, ssm_cache: hymba_ssm_cache | None, workspace,
                        workspace_bytes: int, stream=None) -> None:
    check(lib().hymba_block_prefill(
        layer, C.byref(bw), batch, n_tokens, _ptr(x), _ptr(y), C.byref(kv),
        C.byref(kv_cache) if kv_cache is not None else None,
        C.byref(ssm_cache) if ssm_cache is not None else None,
        _ptr(workspace), workspace_bytes, _stream(stream)), "hymba_block_prefill")


def hymba_block_decode_workspace(layer: int, mlp_hidden: int, batch: int, max_pos: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_block_decode_workspace(layer, mlp_hidden, batch, max_pos, C.byref(out)),
          "hymba_block_decode_workspace")
    return out.value


def hymba_block_decode_step(layer: int, bw: hymba_block_weights, batch: int, pos: int, x_t, y_t,
                            kv_cache: hymba_kv_cache, ssm_cache: hymba_ssm_cache, workspace, workspace_bytes: int,
                            stream=None) -> None:
    check(lib().hymba_block_decode_step(layer, C.byref(bw), batch, pos, _ptr(x_t), _ptr(y_t), C.byref(kv_cache),
                                        C.byref(ssm_cache), _ptr(workspace), workspace_bytes, _stream(stream)),
          "hymba_block_decode_step")


def hymba_layer_decode_workspace(layer: int, batch: int, max_pos: int) -> int:
    out = C.c_size_t()
    check(lib().hymba_layer_decode_workspace(layer, batch, max_pos, C.byref(out)),
          "hymba_layer_decode_workspace")
    return out.value


def hymba_layer_decode_step(layer: int, batch: int, pos: int, x_t, y_t, kv_cache: hymba_kv_cache,
                            ssm_cache: hymba_ssm_cache, workspace, workspace_bytes: int,
                            stream=None) -> None:
    check(lib().hymba_layer_decode_step(layer, batch, pos, _ptr(x_t), _ptr(y_t), C.byref(kv_cache),
                                        C.byref(ssm_cache), _ptr(workspace), workspace_bytes,
                                        _stream(stream)), "hymba_layer_decode_step")


HYMBA_DECODE_STATIC_SCRATCH_BYTES = 40 << 20


def hymba_layer_decode_step_static(layer: int, batch: int, pos: int, x_t, y_t,
                                   kv_cache: hymba_kv_cache, ssm_cache: hymba_ssm_cache,
                                   stream=None) -> None:
    """hymba_layer_decode_step with the library's static scratch instead of a workspace."""
    check(lib().hymba_layer_decode_step_static(layer, batch, pos, _ptr(x_t), _ptr(y_t),
                                               C.byref(kv_cache), C.byref(ssm_cache),
                                               _stream(stream)), "hymba_layer_decode_step_static")


def hymba_stream_status(stream=None) -> None:
    check(lib().hymba_stream_status(_stream(stream)), "hymba_stream_status")


def hymba_last_error() -> str:
    return lib().hymba_last_error().decode()


def hymba_status_string(s: int) -> str:
    return lib().hymba_status_string(s).decode()


def hymba_version() -> str:
    return lib().hymba_version().decode()


def hymba_debug_mask_bitmap(L: int, n_meta: int, window: int, is_global: bool, bits,
                            tile_class=None, stream=None, path: int = 0) -> None:
    check(lib().hymba_debug_mask_bitmap(L, n_meta, window, int(is_global), path, _ptr(bits),
                                        _ptr(tile_class), _stream(stream)), "hymba_debug_mask_bitmap")


def hymba_debug_decode_mask(pos: int, n_meta: int, window: int, is_global: bool, capacity: int, bits,
                            stream=None) -> None:
    check(lib().hymba_debug_decode_mask(pos, n_meta, window, int(is_global), capacity, _ptr(bits),
                                        _stream(stream)), "hymba_debug_decode_mask")


def hymba_debug_exp2_poly(degree: int, x, y, n: int, stream=None) -> None:
    check(lib().hymba_debug_exp2_poly(degree, _ptr(x), _ptr(y), n, _stream(stream)),
          "hymba_debug_exp2_poly")


def hymba_set_wait_limit(cycles: int) -> int:
    """Sets the bounded-wait limit (0: default); returns the limit now in force."""
    out = C.c_int64()
    check(lib().hymba_set_wait_limit(cycles, C.byref(out)), "hymba_set_wait_limit")
    return out.value


def hymba_debug_stall_next_prefill(count: int) -> None:
    check(lib().hymba_debug_stall_next_prefill(count), "hymba_debug_stall_next_prefill")


def hymba_profile_enable(on: bool) -> None:
    check(lib().hymba_profile_enable(int(bool(on))), "hymba_profile_enable")


def hymba_profile_collect(max_entries: int = 64) -> list[tuple[str, int, int, float]]:
    """[(step name, calls, kernels launched, total ms)] since the last collect."""
    buf = (hymba_profile_entry * max_entries)()
    n = C.c_int()
    check(lib().hymba_profile_collect(buf, max_entries, C.byref(n)), "hymba_profile_collect")
    return [(buf[i].name.decode(), buf[i].calls, buf[i].kernels, buf[i].total_ms)
            for i in range(n.value)]


# ---- marshalling helpers ---------------------------------------------------------------

def make_config(d_model, n_heads, n_kv_heads, head_dim_qk, d_inner, d_state, d_conv, dt_rank,
                n_meta, window, is_global, dtype: str, rms_eps=1e-6, softmax_scale=0.0, rope_base=0.0,
                branch_chunks=4):
    """branch_chunks: batch chunks of the concurrent prefill (0 or 1: serial order)."""
    return hymba_layer_config(d_model, n_heads, n_kv_heads, head_dim_qk, d_inner // n_heads, d_inner,
                              d_state, d_conv, dt_rank, n_meta, window if not is_global else 0,
                              int(bool(is_global)), HYMBA_BF16 if dtype == "bf16" else HYMBA_F32,
                              rms_eps, softmax_scale, rope_base, branch_chunks)


def make_weights(w: dict) -> hymba_layer_weights:
    """From a dict of contiguous device tensors (keys as in the header)."""
    for k, t in w.items():
        if not t.is_contiguous():
            raise ValueError(f"weight {k} must be contiguous")
    return hymba_layer_weights(*[_ptr(w[n]) for n, _ in hymba_layer_weights._fields_])
