"""ctypes declarations of include/mk.h and the loader for libmk.so.

There is no fallback: if the library is missing or lacks a symbol, importing the
package's runtime raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmk.so")

MK_OK = 0
MK_ERR_ARG = -1
MK_ERR_TENSOR = -2
MK_ERR_CAPACITY = -3
MK_ERR_CUDA = -4
MK_ERR_DEVICE = -5
MK_ERR_RESIDENCY = -6

MK_DEVERR_BARRIER_TIMEOUT = 0x1
MK_DEVERR_PIPE_TIMEOUT = 0x2
MK_DEVERR_BAD_TOKEN = 0x4
MK_DEVERR_CAPACITY = 0x8

MK_DT_BF16 = 1
MK_DT_F32 = 2
MK_DT_Q4K = 3
MK_W_BF16 = 0
MK_W_Q4K = 1
MK_KV_BF16 = 0
MK_KV_Q8 = 1
MK_MAX_LAYERS = 128

# every symbol include/mk.h declares
EXPORTS = [
    "mk_query_sizes", "mk_load_weights", "mk_reset_state", "mk_set_position", "mk_prefill",
    "mk_decode_step", "mk_decode_step_noalloc", "mk_verify_drafts", "mk_verify_drafts_sampled", "mk_generate", "mk_sync_status", "mk_phase_trace", "mk_launch_count",
    "mk_linear", "mk_last_error", "mk_free",
]


class MkConfig(C.Structure):
    _fields_ = [
        ("n_layers", C.c_int32),
        ("pattern", C.c_char * (MK_MAX_LAYERS + 1)),
        ("hidden", C.c_int32),
        ("vocab", C.c_int32),
        ("rms_eps", C.c_float),
        ("dn_heads", C.c_int32),
        ("dn_dk", C.c_int32),
        ("dn_dv", C.c_int32),
        ("conv_width", C.c_int32),
        ("at_q_heads", C.c_int32),
        ("at_kv_heads", C.c_int32),
        ("at_head_dim", C.c_int32),
        ("rope_theta", C.c_float),
        ("at_out_gate", C.c_int32),
        ("ffn", C.c_int32),
        ("weight_format", C.c_int32),
        ("max_ctx", C.c_int32),
        ("max_draft", C.c_int32),
        ("kv_format", C.c_int32),
    ]


class MkTensor(C.Structure):
    _fields_ = [
        ("name", C.c_char_p),
        ("dtype", C.c_int32),
        ("ndim", C.c_int32),
        ("shape", C.c_int64 * 4),
        ("data", C.c_void_p),
        ("bytes", C.c_uint64),
    ]


class MkSizes(C.Structure):
    _fields_ = [
        ("packed_bytes", C.c_uint64),
        ("state_bytes", C.c_uint64),
        ("workspace_bytes", C.c_uint64),
        ("off_S", C.c_uint64),
        ("off_conv", C.c_uint64),
        ("off_k", C.c_uint64),
        ("off_v", C.c_uint64),
        ("off_pos", C.c_uint64),
        ("off_err", C.c_uint64),
        ("grid_ctas", C.c_int32),
        ("kv_row_bytes", C.c_int32),
        ("layer_table_entries", C.c_int32),
    ]


_lib = None


def load_library(path: str = LIB_PATH) -> C.CDLL:
    """Load libmk.so and declare its signatures. Raises if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m hybrid_deltanet_attention_b200.build` "
            "(this package has no CPU fallback)")
    lib = C.CDLL(path)
    vp, i32, i64 = C.c_void_p, C.c_int32, C.c_int64
    p_i32 = C.POINTER(C.c_int32)
    sig = {
        "mk_query_sizes": (C.c_int, [C.POINTER(MkConfig), C.POINTER(MkSizes)]),
        "mk_load_weights": (C.c_int, [C.POINTER(MkConfig), C.POINTER(MkTensor), i32, vp, vp, vp, vp,
                                      C.POINTER(vp)]),
        "mk_reset_state": (C.c_int, [vp, vp]),
        "mk_set_position": (C.c_int, [vp, i32, vp]),
        "mk_prefill": (C.c_int, [vp, vp, i32, vp, vp, vp]),
        "mk_decode_step": (C.c_int, [vp, vp, vp, vp, vp]),
        "mk_decode_step_noalloc": (C.c_int, [vp, vp, vp, vp, vp]),
        "mk_verify_drafts": (C.c_int, [vp, vp, i32, vp, vp, vp, vp]),
        "mk_verify_drafts_sampled": (C.c_int, [vp, vp, i32, C.c_float, vp, vp, vp, vp, vp]),
        "mk_generate": (C.c_int, [vp, vp, i32, vp, i32, vp]),
        "mk_sync_status": (C.c_int, [vp, vp, p_i32]),
        "mk_phase_trace": (C.c_int, [vp, vp, i32]),
        "mk_launch_count": (i64, [vp]),
        "mk_linear": (C.c_int, [vp, i64, i32, i32, vp, i64, i32, vp, i64, i32, vp, C.c_size_t, vp, vp]),
        "mk_last_error": (C.c_char_p, []),
        "mk_free": (None, [vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)          # AttributeError if a symbol is missing
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class MkError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"mk error {code}: {msg}")
        self.code = code


def check(rc: int) -> None:
    if rc != MK_OK:
        raise MkError(rc, (_lib.mk_last_error() or b"").decode(errors="replace"))
