"""ctypes binding of libcsa2.so: the C ABI of include/csa2.h, same names.

Argument marshalling only -- every step of the decode path runs in the CUDA
kernels of libcsa2.so.  Importing this module loads the library and fails
loudly if it has not been built; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa2.so")

CSA2_OK = 0
CSA2_ERR_INVALID_ARG = -1
CSA2_ERR_UNSUPPORTED = -2
CSA2_ERR_WORKSPACE = -3
CSA2_ERR_CUDA = -4
CSA2_ERR_TIMEOUT = -5
CSA2_ERR_NONFINITE = -6
CSA2_ERR_RANGE = -7
CSA2_F32, CSA2_BF16 = 0, 1
CSA2_MODE_FULL, CSA2_MODE_REINDEX, CSA2_MODE_REUSE = 0, 1, 2

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64


class csa2_query_batch(ctypes.Structure):
    _fields_ = [("n_seq", _i32), ("n_tok", _i32), ("max_seq_len", _i32), ("max_q_per_seq", _i32),
                ("seq_len", _vp), ("tok_start", _vp), ("tok_seq", _vp), ("tok_pos", _vp)]


class csa2_fp4_cache(ctypes.Structure):
    _fields_ = [("codes", _vp), ("scales", _vp), ("n_rows", _i64), ("dim", _i32), ("page_size", _i32),
                ("page_table", _vp), ("max_pages", _i32), ("seq_base", _vp)]


class csa2_swa_desc(ctypes.Structure):
    _fields_ = [("codes", _vp), ("scale", _vp), ("cap", _i32), ("window", _i32), ("dim", _i32)]


class csa2_layer_desc(ctypes.Structure):
    _fields_ = [("mode", _i32), ("iq", _vp), ("iw", _vp), ("q", _vp), ("swa", ctypes.POINTER(csa2_swa_desc)),
                ("out", _vp), ("lse", _vp), ("idx_out", _vp), ("pool_out", _vp)]


class csa2_stack_desc(ctypes.Structure):
    _fields_ = [("qb", csa2_query_batch), ("k_idx", csa2_fp4_cache), ("kv", csa2_fp4_cache), ("H_I", _i32),
                ("P", _i32), ("K", _i32), ("Hq", _i32), ("q_dtype", _i32), ("out_dtype", _i32),
                ("softmax_scale", ctypes.c_float), ("new_k_idx", _vp), ("new_kv", _vp), ("new_slot_k_idx", _vp),
                ("new_slot_kv", _vp), ("n_layers", _i32), ("layers", ctypes.POINTER(csa2_layer_desc)),
                ("attend_wait_event", _vp)]


_P = ctypes.POINTER
_SIGS = {
    "csa2_quantize_fp4": [_vp, _i64, _i32, _vp, _vp, _vp, _vp],
    "csa2_index_full": [_P(csa2_query_batch), _vp, _vp, _vp, _i32, _P(csa2_fp4_cache), _i32, _i32, _vp, _vp, _vp,
                        _vp, _vp, _vp, ctypes.c_size_t, _vp],
    "csa2_index_reindex": [_P(csa2_query_batch), _vp, _vp, _vp, _i32, _P(csa2_fp4_cache), _vp, _vp, _i32, _i32, _vp,
                           _vp, _vp, ctypes.c_size_t, _vp],
    "csa2_attend_reuse": [_P(csa2_query_batch), _vp, _i32, _i32, _P(csa2_fp4_cache), _vp, _vp, _i32,
                          _P(csa2_swa_desc), ctypes.c_float, _vp, _i32, _vp, _vp, ctypes.c_size_t, _vp],
    "csa2_decode_stack": [_P(csa2_stack_desc), _vp, ctypes.c_size_t, _vp],
    "csa2_index_reindex_noalloc": [_P(csa2_query_batch), _vp, _vp, _vp, _i32, _P(csa2_fp4_cache), _vp, _vp, _i32,
                                   _i32, _vp, _vp, _vp],
    "csa2_index_workspace_size": [_P(csa2_query_batch), _i32, _i32, _i32, _i32, _P(ctypes.c_size_t)],
    "csa2_attend_workspace_size": [_P(csa2_query_batch), _i32, _i32, _i32, _i32, _P(ctypes.c_size_t)],
    "csa2_stack_workspace_size": [_P(csa2_stack_desc), _P(ctypes.c_size_t)],
    "csa2_get_status": [_vp],
    "csa2_last_error": [],
    "csa2_version": [],
    "csa2_selftest_wait_timeout": [_i64, _vp],
    "csa2_profiler_enable": [ctypes.c_int],
    "csa2_profiler_read": [_vp, _i32, _vp],
    "csa2_launch_count": [],
    "csa2_tensor_peak": [_i32, _i32, ctypes.POINTER(ctypes.c_double), _vp],
    "csa2_cp_candidates": [_vp, _i64, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "csa2_cp_merge": [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp],
    "csa2_cp_localize": [_vp, _vp, _i32, _i32, _i64, _i64, _i32, _vp, _vp, _vp],
    "csa2_cp_pool_scores": [_P(csa2_query_batch), _vp, _vp, _vp, _i32, _i32, _P(csa2_fp4_cache), _vp, _vp, _i32,
                            _vp, _vp],
    "csa2_cp_select_positions": [_vp, _i32, _i32, _i32, _vp, _vp, _i32, _i32, _vp, _vp, _vp],
    "csa2_cp_attend_merge": [_vp, _vp, _i32, _i64, _i64, _i32, _i32, _i32, _vp, _i32, _vp, _vp],
}

_lib = None


def lib():
    """Load libcsa2.so (raises if it is missing: the product has no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libcsa2.so not built ({LIB_PATH}); run csa2_fp4_sparse_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = {"csa2_last_error": ctypes.c_char_p, "csa2_launch_count": ctypes.c_int64}.get(name, ctypes.c_int)
        _lib = L
    return _lib


class Csa2Error(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(f"csa2 error {code}: {msg}")
        self.code = code


def check(rc: int) -> int:
    if rc != CSA2_OK:
        raise Csa2Error(rc, lib().csa2_last_error().decode())
    return rc


def _wrap(name):
    def f(*args):
        return getattr(lib(), name)(*args)
    f.__name__ = name
    return f


csa2_quantize_fp4 = _wrap("csa2_quantize_fp4")
csa2_index_full = _wrap("csa2_index_full")
csa2_index_reindex = _wrap("csa2_index_reindex")
csa2_attend_reuse = _wrap("csa2_attend_reuse")
csa2_decode_stack = _wrap("csa2_decode_stack")
csa2_index_reindex_noalloc = _wrap("csa2_index_reindex_noalloc")
csa2_index_workspace_size = _wrap("csa2_index_workspace_size")
csa2_attend_workspace_size = _wrap("csa2_attend_workspace_size")
csa2_stack_workspace_size = _wrap("csa2_stack_workspace_size")
csa2_get_status = _wrap("csa2_get_status")
csa2_version = _wrap("csa2_version")
csa2_selftest_wait_timeout = _wrap("csa2_selftest_wait_timeout")
csa2_cp_candidates = _wrap("csa2_cp_candidates")
csa2_cp_merge = _wrap("csa2_cp_merge")
csa2_cp_localize = _wrap("csa2_cp_localize")
csa2_cp_pool_scores = _wrap("csa2_cp_pool_scores")
csa2_cp_select_positions = _wrap("csa2_cp_select_positions")
csa2_cp_attend_merge = _wrap("csa2_cp_attend_merge")


class csa2_kernel_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("launches", _i64), ("total_ms", ctypes.c_double)]


csa2_profiler_enable = _wrap("csa2_profiler_enable")
csa2_launch_count = _wrap("csa2_launch_count")


def csa2_profiler_read(cap: int = 64) -> dict:
    """{kernel name: (launches, total ms)} since the last read; synchronises"""
    arr = (csa2_kernel_stat * cap)()
    n = _i32(0)
    check(lib().csa2_profiler_read(arr, cap, ctypes.byref(n)))
    return {arr[i].name.decode(): (int(arr[i].launches), float(arr[i].total_ms)) for i in range(n.value)}


def csa2_tensor_peak(kind: int, iters: int, stream) -> float:
    """measured dense MMA rate (TFLOP/s) of kind 0 (fp16) or 1 (block-scaled FP4)"""
    v = ctypes.c_double(0.0)
    check(lib().csa2_tensor_peak(kind, iters, ctypes.byref(v), stream))
    return v.value


def csa2_last_error() -> str:
    return lib().csa2_last_error().decode()


EXPORTED = list(_SIGS)
