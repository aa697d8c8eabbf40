"""ctypes binding of librdt (include/rdt.h).  Argument marshalling only: every
step of the recurrent block runs in the library's CUDA kernels.  Importing this
module does not need a GPU; calling an entry point without the library or without
a CUDA device raises."""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int, c_size_t, c_void_p, c_char_p

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "librdt.so")

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace too small or misaligned",
          4: "CUDA runtime error", 5: "device-side wait timed out", 6: "device-side bounds check failed"}
RDT_OK, RDT_ERR_INVALID_ARG, RDT_ERR_UNSUPPORTED, RDT_ERR_WORKSPACE, RDT_ERR_CUDA, RDT_ERR_DEVICE_TIMEOUT, \
    RDT_ERR_DEVICE_BOUNDS = range(7)
RDT_FLAG_TRANSFORMER_OFF = 1
RDT_FLAG_TEST_GEMM_TIMEOUT = 2
RDT_FLAG_TEST_MLA_ATTN_TIMEOUT = 4


class RdtError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code})")
        self.code = code


class rdt_config(ctypes.Structure):
    _fields_ = [(n, c_int) for n in (
        "dim", "n_heads", "n_kv_heads", "attn_type", "kv_lora_rank", "q_lora_rank", "qk_rope_head_dim",
        "qk_nope_head_dim", "v_head_dim", "n_experts", "n_shared_experts", "top_k", "expert_dim", "lora_rank",
        "max_loop_iters", "loop_dim")] + [("rope_theta", c_float), ("loop_theta", c_float), ("norm_eps", c_float),
                                          ("dtype", c_int)]


WEIGHT_FIELDS = ("rec_norm_w", "attn_norm_w", "ffn_norm_w", "w_qkv", "w_o", "w_q_down", "q_norm_w", "w_q_up",
                 "w_kv_down", "kv_norm_w", "w_kv_up", "w_router", "router_bias", "w13", "w2", "lora_down", "lora_B",
                 "lora_scale", "log_A", "log_dt", "inj_B", "halt_w", "halt_b")


class rdt_weights(ctypes.Structure):
    _fields_ = [(n, c_void_p) for n in WEIGHT_FIELDS]


class rdt_kv_cache(ctypes.Structure):
    _fields_ = [("k", c_void_p), ("v", c_void_p), ("n_loops", c_int), ("batch", c_int), ("t_max", c_int)]


class rdt_trace(ctypes.Structure):
    _fields_ = [("row0", c_int), ("n_rows", c_int), ("h_in", c_void_p), ("f", c_void_p),
                ("biased_logits", c_void_p), ("p", c_void_p)]


class rdt_depth_batch(ctypes.Structure):
    _fields_ = [("cfg", POINTER(rdt_config)), ("w", POINTER(rdt_weights)), ("h0", c_void_p), ("e", c_void_p),
                ("halt_logit_offset", c_void_p), ("cache_len", c_void_p), ("batch", c_int), ("n_tokens", c_int),
                ("n_loops", c_int), ("act_threshold", c_float), ("h_out", c_void_p), ("halt_weights", c_void_p),
                ("expert_ids", c_void_p), ("cache", POINTER(rdt_kv_cache)), ("ws", c_void_p), ("ws_bytes", c_size_t)]


class rdt_kernel_time(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", c_int), ("total_ms", ctypes.c_double)]


EXPORTS = ("rdt_workspace_size", "rdt_recurrent_forward", "rdt_recurrent_decode_step", "rdt_block_forward",
           "rdt_block_forward_cached", "rdt_embed", "rdt_head", "rdt_head_rows", "rdt_greedy_tokens",
           "rdt_to_model_dtype", "rdt_read_device_status", "rdt_status_string", "rdt_version",
           "rdt_launch_count", "rdt_profile_start", "rdt_profile_stop", "rdt_recurrent_decode_step_static",
           "rdt_read_static_status", "rdt_recurrent_decode_step_ex",
           "rdt_depth_batch_workspace_size", "rdt_depth_batch_begin", "rdt_depth_batch_tick",
           "rdt_depth_batch_pending", "rdt_depth_batch_run")

_lib = None
_profiling = False


def load(path: str = LIB_PATH):
    """Load librdt.so and declare its signatures.  Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"librdt.so not found at {path}; build it with `python -m recurrent_depth_moe_b200.build`")
    lib = ctypes.CDLL(path)
    P = c_void_p
    lib.rdt_workspace_size.argtypes = [POINTER(rdt_config), c_int, c_int, c_int]
    lib.rdt_workspace_size.restype = c_size_t
    lib.rdt_recurrent_forward.argtypes = [POINTER(rdt_config), POINTER(rdt_weights), P, P, c_int, c_int, c_int, c_int,
                                          c_float, P, P, P, P, POINTER(rdt_kv_cache), POINTER(rdt_trace), c_int, P,
                                          c_size_t, P]
    lib.rdt_recurrent_forward.restype = c_int
    lib.rdt_recurrent_decode_step.argtypes = [POINTER(rdt_config), POINTER(rdt_weights), P, P, c_int, P, c_int,
                                              c_float, P, P, P, POINTER(rdt_kv_cache), P, c_size_t, P]
    lib.rdt_recurrent_decode_step.restype = c_int
    lib.rdt_recurrent_decode_step_ex.argtypes = [POINTER(rdt_config), POINTER(rdt_weights), P, P, c_int, P,
                                                 c_int, c_float, P, P, P, P, POINTER(rdt_kv_cache),
                                                 POINTER(rdt_trace), P, c_size_t, P]
    lib.rdt_recurrent_decode_step_ex.restype = c_int
    lib.rdt_depth_batch_workspace_size.argtypes = [POINTER(rdt_config), c_int, c_int, c_int]
    lib.rdt_depth_batch_workspace_size.restype = c_size_t
    for fn in ("rdt_depth_batch_begin",):
        getattr(lib, fn).argtypes = [POINTER(rdt_depth_batch), P]
        getattr(lib, fn).restype = c_int
    lib.rdt_depth_batch_tick.argtypes = [POINTER(rdt_depth_batch), c_int, P]
    lib.rdt_depth_batch_tick.restype = c_int
    lib.rdt_depth_batch_pending.argtypes = [POINTER(rdt_depth_batch), P]
    lib.rdt_depth_batch_pending.restype = ctypes.c_longlong
    lib.rdt_depth_batch_run.argtypes = [POINTER(rdt_depth_batch), c_int, P]
    lib.rdt_depth_batch_run.restype = c_int
    lib.rdt_block_forward.argtypes = [POINTER(rdt_config), POINTER(rdt_weights), P, P, c_int, c_int, c_int, P,
                                      c_size_t, P]
    lib.rdt_block_forward.restype = c_int
    lib.rdt_block_forward_cached.argtypes = [POINTER(rdt_config), POINTER(rdt_weights), P, P, c_int, c_int, c_int,
                                             P, POINTER(rdt_kv_cache), P, c_size_t, P]
    lib.rdt_block_forward_cached.restype = c_int
    lib.rdt_head_rows.argtypes = [POINTER(rdt_config), P, ctypes.c_longlong, c_int, P, P, c_int, P, P, c_size_t, P]
    lib.rdt_head_rows.restype = c_int
    lib.rdt_greedy_tokens.argtypes = [P, c_int, c_int, P, c_int, P]
    lib.rdt_greedy_tokens.restype = c_int
    lib.rdt_to_model_dtype.argtypes = [POINTER(rdt_config), P, P, ctypes.c_longlong, P]
    lib.rdt_to_model_dtype.restype = c_int
    lib.rdt_embed.argtypes = [POINTER(rdt_config), P, c_int, P, c_int, P, P]
    lib.rdt_embed.restype = c_int
    lib.rdt_head.argtypes = [POINTER(rdt_config), P, c_int, P, P, c_int, P, P, c_size_t, P]
    lib.rdt_head.restype = c_int
    lib.rdt_read_device_status.argtypes = [P, P]
    lib.rdt_read_device_status.restype = c_int
    lib.rdt_status_string.argtypes = [c_int]
    lib.rdt_status_string.restype = c_char_p
    lib.rdt_version.argtypes = []
    lib.rdt_version.restype = c_char_p
    lib.rdt_launch_count.argtypes = []
    lib.rdt_launch_count.restype = ctypes.c_ulonglong
    lib.rdt_profile_start.argtypes = []
    lib.rdt_profile_start.restype = c_int
    lib.rdt_profile_stop.argtypes = [POINTER(rdt_kernel_time), c_int]
    lib.rdt_profile_stop.restype = c_int
    _lib = lib
    return lib


def check(fn: str, code: int):
    if code != RDT_OK:
        raise RdtError(fn, code)


def launch_count() -> int:
    return int(load().rdt_launch_count())


def profile_start():
    global _profiling
    check("rdt_profile_start", load().rdt_profile_start())
    _profiling = True


def profiling() -> bool:
    """True between profile_start() and profile_stop(): the per-class CUDA events are
    recorded at launch time, so callers that would replay a captured CUDA graph run
    eagerly instead."""
    return _profiling


def profile_stop() -> dict:
    """{kernel class: (launches, total_ms)} recorded since profile_start()."""
    global _profiling
    _profiling = False
    buf = (rdt_kernel_time * 32)()
    n = load().rdt_profile_stop(buf, 32)
    if n < 0:
        raise RdtError("rdt_profile_stop", RDT_ERR_CUDA)
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n)}
