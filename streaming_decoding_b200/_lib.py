"""ctypes loader for libwedlm.so (argument marshalling only).

The library must have been built (``python -m streaming_decoding_b200.build``
or ``__graft_entry__.build()``).  There is no fallback: importing this module
without the shared library raises."""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB_PATH = os.path.join(HERE, "libwedlm.so")
HEADER = os.path.join(ROOT, "include", "wedlm.h")

c_i32, c_i64, c_f32, c_f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double
c_vp = ctypes.c_void_p


class ModelCfg(ctypes.Structure):
    _fields_ = [("n_layers", c_i32), ("d_model", c_i32), ("n_heads", c_i32), ("n_kv_heads", c_i32),
                ("head_dim", c_i32), ("ffn_dim", c_i32), ("vocab", c_i32), ("mask_id", c_i32),
                ("rope_theta", c_f64), ("rms_eps", c_f32), ("dtype", c_i32), ("max_batch", c_i32),
                ("max_window", c_i32), ("max_ctx", c_i32), ("num_pages", c_i32), ("prefill_chunk", c_i32)]


class StepParams(ctypes.Structure):
    _fields_ = [("lambda_", c_f32), ("tau", c_f32), ("tau_none", c_i32), ("logit_scale", c_f32),
                ("blockwise", c_i32), ("temperature", c_f32), ("seed", ctypes.c_uint64)]


class SeqStats(ctypes.Structure):
    _fields_ = [("steps", c_i64), ("forward_rows", c_i64), ("committed", c_i64), ("fills", c_i64),
                ("committed_len", c_i32), ("end", c_i32), ("window", c_i32), ("active", c_i32)]


def header_constants() -> dict:
    """#define WEDLM_* integer constants of include/wedlm.h."""
    out = {}
    with open(HEADER) as f:
        for m in re.finditer(r"#define\s+(WEDLM_[A-Z0-9_]+)\s+(-?\d+)", f.read()):
            out[m.group(1)] = int(m.group(2))
    return out


def header_functions() -> list:
    """Names of the functions include/wedlm.h declares."""
    with open(HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(wedlm_[a-z0-9_]+)\s*\(", text)))


_SIGS = {
    "wedlm_create": (c_i32, [ctypes.POINTER(ModelCfg), c_vp, ctypes.POINTER(c_vp)]),
    "wedlm_destroy": (None, [c_vp]),
    "wedlm_status_str": (ctypes.c_char_p, [c_i32]),
    "wedlm_last_error": (ctypes.c_char_p, [c_vp]),
    "wedlm_load_weights": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_i32, c_i32]),
    "wedlm_prefill": (c_i32, [c_vp, c_i32, c_vp, c_i32, c_i32, c_i32]),
    "wedlm_kv_reset": (c_i32, [c_vp, c_i32]),
    "wedlm_stream_step": (c_i32, [c_vp, ctypes.POINTER(StepParams), c_vp, c_vp, c_vp]),
    "wedlm_stream_step_async": (c_i32, [c_vp, ctypes.POINTER(StepParams), c_i32]),
    "wedlm_read_generated": (c_i32, [c_vp, c_i32, c_vp, c_i32, c_vp]),
    "wedlm_get_stats": (c_i32, [c_vp, c_i32, ctypes.POINTER(SeqStats)]),
    "wedlm_kernel_launches": (c_i32, [c_vp, ctypes.POINTER(c_i64)]),
    "wedlm_profile_enable": (c_i32, [c_vp, c_i32]),
    "wedlm_autotune": (c_i32, [c_vp, c_i32]),
    "wedlm_debug_capture": (c_i32, [c_vp, c_i32]),
    "wedlm_debug_keep_logits": (c_i32, [c_vp, c_i32]),
    "wedlm_debug_residual": (c_i32, [c_vp, c_i32, c_vp, c_i32]),
    "wedlm_gemm_plan": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "wedlm_gemm_schedule": (c_i32, [c_vp, c_i32, c_i32, c_vp]),
    "wedlm_profile_read": (c_i32, [c_vp, c_vp, c_vp]),
    "wedlm_debug_read": (c_i32, [c_vp, c_i32, c_vp, c_i64]),
    "wedlm_debug_kv": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp]),
    "wedlm_debug_get_window": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i32, c_vp]),
    "wedlm_debug_set_window": (c_i32, [c_vp, c_i32, c_vp, c_vp, c_i32]),
    "wedlm_reorder_window": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "wedlm_entropy_select": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_i32, c_i32, ctypes.POINTER(StepParams),
                                     c_vp, c_vp, c_vp, c_vp]),
    "wedlm_entropy_select_noalloc": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_i32, c_i32,
                                             ctypes.POINTER(StepParams), c_vp, c_vp, c_vp, c_vp]),
    "wedlm_entropy_select_workspace_bytes": (c_i32, [c_i32, c_i32, ctypes.POINTER(c_i64)]),
    "wedlm_entropy_select_async": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_vp, c_i32, c_i32, ctypes.POINTER(StepParams),
                                           c_vp, c_vp, c_vp, c_vp, c_i64, c_vp]),
    "wedlm_debug_set_page": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp]),
    "wedlm_debug_read_weight": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_i64]),
    "wedlm_debug_set_plan": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_i32, c_i32]),
    "wedlm_attention_workspace_bytes": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, ctypes.POINTER(c_i64)]),
    "wedlm_attention_bf16": (c_i32, [c_vp, c_vp, c_i32, c_i32, c_i32, c_vp, c_i32, c_vp, c_vp, c_i32, c_i32, c_i32,
                                     c_vp, c_vp, c_i64, c_vp]),
    "wedlm_linear_bf16": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_vp]),
    "wedlm_linear_bf16_plan": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp]),
    "wedlm_linear_bf16_sched": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m streaming_decoding_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class WedlmError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = load().wedlm_status_str(status).decode()
        super().__init__(f"{where}: {msg} ({status})" + (f": {detail}" if detail else ""))
