"""ctypes view of the C ABI in include/twilight.h (argument marshalling only).

Loading fails loudly when lib/libtwilight.so is missing: there is no fallback.
Build it with `python -m adaptive_top_sparse_quest_b200.build`.
"""
from __future__ import annotations

import ctypes
import os
import re

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libtwilight.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "twilight.h")

TW_OK = 0
TW_ERR_INVALID_ARG = 1
TW_ERR_UNSUPPORTED = 2
TW_ERR_CAPACITY = 3
TW_ERR_CUDA = 4
TW_ERR_TIMEOUT = 5

c_i32 = ctypes.c_int32
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t


class TwKv(ctypes.Structure):
    _fields_ = [
        ("k", c_vp), ("v", c_vp), ("batch", c_i32), ("num_kv_heads", c_i32),
        ("max_seq_len", c_i32), ("seq_lens", c_vp), ("page_table", c_vp),
        ("max_pages_per_seq", c_i32), ("num_pool_pages", c_i32), ("page_size", c_i32),
        ("head_dim", c_i32), ("key_bits", c_i32),
    ]


class TwStep(ctypes.Structure):
    _fields_ = [
        ("q", c_vp), ("num_q_heads", c_i32), ("kv", TwKv), ("codes", c_vp), ("scales", c_vp),
        ("zeros", c_vp), ("meta", c_vp), ("budget_tokens", c_i32), ("p", ctypes.c_double),
        ("group_mode", c_i32), ("cand_pages", c_vp), ("cand_stride", c_i32), ("ncand", c_vp),
        ("idx", c_vp), ("capacity", c_i32), ("count", c_vp), ("out", c_vp), ("lse", c_vp),
        ("ws", c_vp), ("ws_bytes", c_size), ("append_keys", c_i32),
    ]


_SIGS = {
    "tw_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tw_last_cuda_error": (ctypes.c_int, []),
    "tw_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "tw_version": (ctypes.c_int, []),
    "tw_quantize_keys": (ctypes.c_int, [ctypes.POINTER(TwKv), c_vp, c_vp, c_vp, c_vp]),
    "tw_page_meta": (ctypes.c_int, [ctypes.POINTER(TwKv), c_vp, c_vp]),
    "tw_append_keys": (ctypes.c_int, [ctypes.POINTER(TwKv), c_vp, c_vp, c_vp, c_vp, c_vp]),
    "tw_workspace_size": (ctypes.c_int, [c_i32, c_i32, c_i32, c_i32, c_i32,
                                         ctypes.POINTER(c_size)]),
    "tw_select_pages": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_i32, c_vp,
                                       c_i32, c_vp, c_vp, c_size, c_vp]),
    "tw_topp_prune": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_vp, c_vp, c_vp,
                                     c_i32, c_vp, ctypes.c_double, c_i32, c_vp, c_i32, c_vp, c_vp,
                                     c_size, c_vp]),
    "tw_sparse_decode": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_i32, c_vp,
                                        c_i32, c_vp, c_vp, c_vp, c_size, c_vp]),
    "tw_topp_prune_noalloc": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_vp, c_vp,
                                             c_vp, c_i32, c_vp, ctypes.c_double, c_i32, c_vp,
                                             c_i32, c_vp, c_vp]),
    "tw_label_cache": (ctypes.c_int, [ctypes.POINTER(TwKv), c_vp, c_i32, c_vp, c_vp]),
    "tw_token_workspace_size": (ctypes.c_int, [c_i32, c_i32, c_i32, c_i32, c_i32, c_i32, c_i32,
                                               ctypes.POINTER(c_size)]),
    "tw_select_tokens": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_vp, c_i32,
                                        c_i32, c_vp, c_i32, c_vp, c_vp, c_size, c_vp]),
    "tw_topp_prune_tokens": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(TwKv), c_vp, c_vp, c_vp,
                                            c_vp, c_i32, c_vp, ctypes.c_double, c_i32, c_vp,
                                            c_i32, c_vp, c_vp, c_size, c_vp]),
    "tw_decode_step": (ctypes.c_int, [ctypes.POINTER(TwStep), c_vp]),
    "tw_decode_step_host": (ctypes.c_int, [ctypes.POINTER(TwStep), c_vp, c_vp, c_vp]),
    "tw_decode_step_num_kernels": (ctypes.c_int, [ctypes.POINTER(TwStep)]),
    "tw_decode_step_kernel_name": (ctypes.c_char_p, [ctypes.POINTER(TwStep), c_i32]),
    "tw_decode_step_profiled": (ctypes.c_int, [ctypes.POINTER(TwStep), ctypes.POINTER(c_vp), c_i32,
                                               c_vp]),
}

_lib = None


def header_functions(path: str = HEADER):
    """Names of the functions include/twilight.h declares."""
    text = open(path).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(tw_[a-z0-9_]+)\s*\(", text)))


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libtwilight.so and declare every entry point's signature."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"Twilight CUDA library not found at {path}; build it with "
            "`python -m adaptive_top_sparse_quest_b200.build` (there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    if path == LIB_PATH:
        _lib = lib
    return lib


class TwError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_err: int = 0):
        lib = load()
        msg = lib.tw_status_string(status).decode()
        if status == TW_ERR_CUDA:
            msg += f" (cudaError {cuda_err})"
        super().__init__(f"{where}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != TW_OK:
        cuda_err = load().tw_last_cuda_error() if status == TW_ERR_CUDA else 0
        raise TwError(status, where, cuda_err)
