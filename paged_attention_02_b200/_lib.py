"""ctypes binding of include/fia.h (libfia.so), argument marshalling only.

Every function keeps the C name and argument order.  The library is loaded
from this package's directory; if it is missing the import fails loudly --
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfia.so")

FIA_OK = 0
FIA_ERR_NULLPTR = 1
FIA_ERR_PARAM = 2
FIA_ERR_DTYPE = 3
FIA_ERR_SHAPE = 4
FIA_ERR_UNSUPPORTED = 5
FIA_ERR_WORKSPACE = 6
FIA_ERR_CUDA = 7

FIA_F16, FIA_BF16, FIA_F32, FIA_I8, FIA_I32 = 0, 1, 2, 3, 4
FIA_MASK_NONE, FIA_MASK_ALIBI, FIA_MASK_CAUSAL = 0, 3, 9
FIA_PATH_AUTO, FIA_PATH_DECODE, FIA_PATH_TENSOR = 0, 1, 2
FIA_KV_BNBSH, FIA_KV_BNNBSD = 0, 1
FIA_ANTIQUANT_PER_CHANNEL, FIA_ANTIQUANT_PER_TOKEN = 0, 1
FIA_SPARSE_NONE, FIA_SPARSE_BAND = 0, 4


class fia_tensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int), ("ndim", ctypes.c_int32),
                ("dims", ctypes.c_int64 * 4)]


class fia_ext(ctypes.Structure):
    _fields_ = [("pse", ctypes.POINTER(fia_tensor)), ("sink", ctypes.POINTER(fia_tensor)),
                ("kScale", ctypes.POINTER(fia_tensor)), ("kOffset", ctypes.POINTER(fia_tensor)),
                ("vScale", ctypes.POINTER(fia_tensor)), ("vOffset", ctypes.POINTER(fia_tensor)),
                ("lse", ctypes.POINTER(fia_tensor)), ("kvLayout", ctypes.c_int32),
                ("kAntiquantMode", ctypes.c_int32), ("vAntiquantMode", ctypes.c_int32),
                ("sparseMode", ctypes.c_int32), ("preTokens", ctypes.c_int64),
                ("nextTokens", ctypes.c_int64), ("path", ctypes.c_int32)]


class fia_plan_info(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int32), ("kernels_per_run", ctypes.c_int32),
                ("work_items", ctypes.c_int64), ("grid", ctypes.c_int32),
                ("split_tokens", ctypes.c_int32), ("error_word_offset", ctypes.c_int64)]


class FiaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, fia_status_string(status), status))


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            "libfia.so is not built (%s); run `python -m paged_attention_02_b200.build`" % LIB_PATH)
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    T = ctypes.POINTER(fia_tensor)
    lib.fia_get_workspace_size.argtypes = [T, T, T, T, ctypes.POINTER(ctypes.c_int32),
                                           ctypes.POINTER(ctypes.c_int32), ctypes.c_int32, T,
                                           ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                           ctypes.c_float, ctypes.POINTER(fia_ext), T,
                                           ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(P)]
    lib.fia_get_workspace_size.restype = ctypes.c_int
    lib.fia_run.argtypes = [P, ctypes.c_uint64, P, P]
    lib.fia_run.restype = ctypes.c_int
    lib.fia_op_destroy.argtypes = [P]
    lib.fia_op_destroy.restype = None
    lib.fia_status_string.argtypes = [ctypes.c_int]
    lib.fia_status_string.restype = ctypes.c_char_p
    lib.fia_op_set_timing_events.argtypes = [P, P, P]
    lib.fia_op_set_timing_events.restype = ctypes.c_int
    lib.fia_op_get_plan_info.argtypes = [P, ctypes.POINTER(fia_plan_info)]
    lib.fia_op_get_plan_info.restype = ctypes.c_int
    lib.fia_decode_run_static.argtypes = [P, P]
    lib.fia_decode_run_static.restype = ctypes.c_int
    lib.fia_decode_static_error_word.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.fia_decode_static_error_word.restype = ctypes.c_int
    lib.fia_op_set_wait_limit.argtypes = [P, ctypes.c_uint64, ctypes.c_int32]
    lib.fia_op_set_wait_limit.restype = ctypes.c_int
    return lib


_lib = _load()
lib = _lib


def fia_status_string(s: int) -> str:
    return _lib.fia_status_string(int(s)).decode()


def fia_get_workspace_size(query, key, value, block_tables, seq_len, kv_seq_len, batch, slopes,
                           mask_type, head_num, kv_head_num, qk_scale, ext, attn_out,
                           workspace_size, op) -> int:
    return _lib.fia_get_workspace_size(query, key, value, block_tables, seq_len, kv_seq_len,
                                       batch, slopes, mask_type, head_num, kv_head_num,
                                       qk_scale, ext, attn_out, workspace_size, op)


def fia_run(workspace, workspace_size, op, stream) -> int:
    return _lib.fia_run(workspace, workspace_size, op, stream)


def fia_op_destroy(op) -> None:
    _lib.fia_op_destroy(op)


def fia_op_set_timing_events(op, start, stop) -> int:
    return _lib.fia_op_set_timing_events(op, start, stop)


def fia_op_get_plan_info(op, info) -> int:
    return _lib.fia_op_get_plan_info(op, info)


def fia_op_set_wait_limit(op, wait_limit_ns, stall) -> int:
    return _lib.fia_op_set_wait_limit(op, wait_limit_ns, stall)


FIA_STATIC_WORKSPACE_BYTES = 32 * 1024 * 1024


def fia_decode_run_static(op, stream) -> int:
    """Decode-path run with the library's fixed scratch array (no workspace
    argument, no allocation); see include/fia.h."""
    return _lib.fia_decode_run_static(op, stream)


def fia_decode_static_error_word(op, word) -> int:
    """Error word of the last fia_decode_run_static call on the op's device
    (a synchronous 4-byte copy)."""
    return _lib.fia_decode_static_error_word(op, word)
