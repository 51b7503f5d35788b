"""ctypes mirror of include/amk.h.  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libamk.so")

c_i32, c_u32, c_i64, c_f32 = ctypes.c_int32, ctypes.c_uint32, ctypes.c_int64, ctypes.c_float
c_vp = ctypes.c_void_p
c_vpp = ctypes.POINTER(ctypes.c_void_p)

# status codes
AMK_OK = 0
STATUS = {
    0: "AMK_OK", -1: "AMK_ERR_INVALID_ARG", -2: "AMK_ERR_UNSUPPORTED",
    -3: "AMK_ERR_VALIDATION", -4: "AMK_ERR_POS_RANGE", -5: "AMK_ERR_LAUNCH",
    -6: "AMK_ERR_TIMEOUT", -7: "AMK_ERR_CUDA", -8: "AMK_ERR_OOM",
    -9: "AMK_ERR_POISONED", -10: "AMK_ERR_NO_DEVICE",
}
ERR = {v: k for k, v in STATUS.items()}
QUANT_BF16, QUANT_W8A16, QUANT_W4A16 = 0, 1, 2
ACC_READ, ACC_WRITE, ACC_ACCUM, ACC_READ_PREV, ACC_RESET, ACC_READ_FLAGGED = range(6)
BUF_OUTPUT = 1
RULES = {0: "ok", 1: "V1", 2: "V2", 3: "V3", 4: "V4", 5: "V5", 6: "V6", 7: "V7",
         8: "V8", 9: "V9", 10: "V10"}


class Config(ctypes.Structure):
    _fields_ = [("hidden", c_i32), ("n_layers", c_i32), ("n_heads", c_i32),
                ("n_kv_heads", c_i32), ("head_dim", c_i32), ("ffn", c_i32),
                ("vocab", c_i32), ("max_ctx", c_i32), ("rms_eps", c_f32),
                ("rope_theta", c_f32), ("tied_embeddings", c_i32), ("quant", c_i32)]


class Weights(ctypes.Structure):
    _fields_ = [("embed", c_vp), ("final_norm", c_vp), ("lm_head", c_vp),
                ("lm_head_scale", c_vp)] + [
        (n, c_vpp) for n in ("attn_norm", "ffn_norm", "wq", "wk", "wv", "wo", "wgate",
                             "wup", "wdown", "sq", "sk", "sv", "so", "sgate", "sup", "sdown")]


class Options(ctypes.Structure):
    _fields_ = [("ring_stages", c_i32), ("stage_bytes", c_i32), ("attn_splits", c_i32),
                ("tasks_per_sm", c_i32), ("n_sms", c_i32), ("wait_timeout_us", c_u32),
                ("debug_skip_signal_task", c_i32), ("profile", c_i32),
                ("l2_prefetch_kb", c_i32), ("ffn_fused", c_i32),
                ("pos0_plan", c_i32), ("inflight_kb", c_i32), ("copy_piece_kb", c_i32),
                ("sm_rotate", c_i32), ("debug_checks", c_i32), ("flagged_waits", c_i32)]


class GraphWait(ctypes.Structure):
    _fields_ = [("counter", c_i32), ("threshold", c_i32)]


class GraphAccess(ctypes.Structure):
    _fields_ = [("buffer", c_i32), ("kind", c_i32), ("begin", c_i64), ("end", c_i64)]


class GraphBuffer(ctypes.Structure):
    _fields_ = [("size", c_i64), ("flags", c_i32), ("pair", c_i32)]


class GraphTask(ctypes.Structure):
    _fields_ = [("sm", c_i32), ("wait_begin", c_i32), ("wait_count", c_i32),
                ("signal_begin", c_i32), ("signal_count", c_i32),
                ("access_begin", c_i32), ("access_count", c_i32)]


class Graph(ctypes.Structure):
    _fields_ = [("n_tasks", c_i32), ("n_counters", c_i32), ("n_buffers", c_i32),
                ("n_sms", c_i32), ("n_waits", c_i32), ("n_signals", c_i32),
                ("n_accesses", c_i32),
                ("tasks", ctypes.POINTER(GraphTask)), ("waits", ctypes.POINTER(GraphWait)),
                ("signals", ctypes.POINTER(c_i32)), ("accesses", ctypes.POINTER(GraphAccess)),
                ("buffers", ctypes.POINTER(GraphBuffer)),
                ("queue_offsets", ctypes.POINTER(c_i32)),
                ("queue_tasks", ctypes.POINTER(c_i32))]


class ValidationReport(ctypes.Structure):
    _fields_ = [("rule", c_i32), ("task_a", c_i32), ("task_b", c_i32), ("counter", c_i32),
                ("buffer", c_i32), ("message", ctypes.c_char * 256)]


class PlanStats(ctypes.Structure):
    _fields_ = [("n_tasks", c_i32), ("n_counters", c_i32), ("n_sms", c_i32),
                ("ring_stages", c_i32), ("stage_bytes", c_i32), ("attn_splits", c_i32),
                ("smem_bytes", c_i32), ("threads_per_cta", c_i32),
                ("weight_bytes", c_i64), ("kv_row_bytes", c_i64), ("epoch", c_i64),
                ("flagged_waits", c_i32), ("ffn_fused", c_i32)]


class ErrorInfo(ctypes.Structure):
    _fields_ = [("code", c_i32), ("task", c_i32), ("counter", c_i32), ("sm", c_i32),
                ("seen", c_u32), ("target", c_u32)]


class Workspace(ctypes.Structure):
    _fields_ = [("qkv", c_vp), ("xmid", c_vp), ("xout", c_vp), ("act", c_vp),
                ("qkv_rows", c_i32)]


# every function include/amk.h declares: name -> (restype, argtypes)
SIGNATURES = {
    "amk_version": (ctypes.c_char_p, []),
    "amk_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "amk_last_error": (ctypes.c_char_p, []),
    "amk_default_options": (ctypes.c_int, [ctypes.POINTER(Options)]),
    "amk_validate_graph": (ctypes.c_int, [ctypes.POINTER(Graph),
                                          ctypes.POINTER(ValidationReport)]),
    "amk_plan_create": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(Options), c_i32,
                                       ctypes.POINTER(c_vp), ctypes.POINTER(ValidationReport)]),
    "amk_plan_graph": (ctypes.c_int, [c_vp, ctypes.POINTER(Graph)]),
    "amk_plan_task_info": (ctypes.c_int, [c_vp, ctypes.POINTER(c_i32), ctypes.POINTER(c_i32)]),
    "amk_plan_destroy": (None, [c_vp]),
    "amk_plan_pos0": (c_vp, [c_vp]),
    "amk_create": (ctypes.c_int, [ctypes.POINTER(Config), ctypes.POINTER(Weights),
                                  ctypes.POINTER(Options), c_vp, ctypes.POINTER(c_vp)]),
    "amk_destroy": (None, [c_vp]),
    "amk_reset_kv": (ctypes.c_int, [c_vp]),
    "amk_decode_step": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp, ctypes.POINTER(c_i32)]),
    "amk_decode_step_host": (ctypes.c_int, [c_vp, c_i32, c_i32, c_vp, ctypes.POINTER(c_i32)]),
    "amk_get_kv": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(c_vp), ctypes.POINTER(c_vp)]),
    "amk_get_logits": (ctypes.c_int, [c_vp, ctypes.POINTER(c_vp)]),
    "amk_get_stats": (ctypes.c_int, [c_vp, ctypes.POINTER(PlanStats)]),
    "amk_plan_get_stats": (ctypes.c_int, [c_vp, ctypes.POINTER(PlanStats)]),
    "amk_get_error_info": (ctypes.c_int, [c_vp, ctypes.POINTER(ErrorInfo)]),
    "amk_get_workspace": (ctypes.c_int, [c_vp, ctypes.POINTER(Workspace)]),
    "amk_get_profile": (ctypes.c_int, [c_vp, ctypes.POINTER(ctypes.c_uint64), c_i64]),
    "amk_check_guards": (ctypes.c_int, [c_vp, ctypes.POINTER(c_i32)]),
    "amk_read_ceiling": (ctypes.c_int, [c_vp, c_i64, c_i32, c_i32, c_i32, c_i32, c_vp,
                                        ctypes.POINTER(ctypes.c_double)]),
    "amk_decode_step_noalloc": (ctypes.c_int, [c_vp, ctypes.POINTER(Weights), c_vp, c_i32,
                                               c_i32, c_vp, ctypes.POINTER(c_i32), c_vp]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded libamk.so.  Raises if the library is missing: there is no
    fallback path."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"libamk.so not found at {LIB_PATH}; build it with "
            "`python persistent_megakernel_decode_cta_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = L
    return L
