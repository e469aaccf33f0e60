"""ctypes binding of libhardkv.so: argument marshalling only.

Every function here forwards to the C entry point of the same name (declared in
include/hardkv.h); all computation happens in the library's CUDA kernels. Loading
fails loudly when the shared library is missing: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

HERE = os.path.dirname(os.path.abspath(__file__))
# HARDKV_CHECKED=1 selects the bounds-checked build (libhardkv_checked.so)
LIB_PATH = os.path.join(HERE, "libhardkv_checked.so" if os.environ.get("HARDKV_CHECKED") == "1"
                        else "libhardkv.so")
HEADER = os.path.join(HERE, "..", "include", "hardkv.h")

OK, EINVAL, EALIGN, EDTYPE, ECAP, ECUDA, ESCRATCH = 0, -1, -2, -3, -4, -5, -6
F32, BF16 = 0, 1
EVICT, MERGE = 0, 1
SELECT_ALL, SELECT_MOVED = 0, 1
RULE_TOPP, RULE_TOPK = 0, 1
LAYOUT_REWRITE, LAYOUT_SPARSE_LOAD, LAYOUT_MTI = 0, 1, 2
CAL_TAU, CAL_ENTROPY = 0, 1
STATUS_WORDS = 8
ST_FLAGS, ST_CLAMPS, ST_NEAR_TIES, ST_MERGED, ST_MOVES, ST_SELECTIONS = range(6)
DEV_RING_OVERFLOW, DEV_BAD_BOUNDS, DEV_SEGMENTS, DEV_WAIT_TIMEOUT = 1, 2, 4, 8
DEV_SELECT, DEV_POOL_SHORT, DEV_CHECK = 16, 32, 64
PAGE_ROWS = 16
POOL_FREE, POOL_RETURNED, POOL_CTL_WORDS = 0, 1, 4
STEP_EVENTS = 6

_i32 = ctypes.c_int32
_vp = ctypes.c_void_p


class Desc(ctypes.Structure):
    _fields_ = [(n, _i32) for n in (
        "batch", "n_q_heads", "n_kv_heads", "head_dim", "block", "dense_window",
        "condensed_slots", "n_sink", "sparse_cap", "ring_rows", "dtype", "condense_mode")]


class Cache(ctypes.Structure):
    _fields_ = [(n, _vp) for n in (
        "k_ring", "v_ring", "len", "d_lo", "s_lo", "moved", "k_sp", "v_sp", "sp_idx",
        "n_kept", "sp_mode", "k_cd", "v_cd", "w_cd", "status", "k_pool", "v_pool", "blk_tab",
        "blk_cnt", "free_list", "ret_list", "pool_ctl")] + [("pool_blocks", ctypes.c_int64)]


class LayoutPolicy(ctypes.Structure):
    _fields_ = [("mode", _i32), ("reuse_steps", _i32), ("l_lower", _i32), ("l_upper", _i32),
                ("gather_surcharge", ctypes.c_float)]


class StepArgs(ctypes.Structure):
    _fields_ = [("q", _vp), ("k_new", _vp), ("v_new", _vp), ("tau", _vp),
                ("p", ctypes.c_float), ("select_mode", _i32), ("mask", _vp), ("out", _vp),
                ("stage_events", _vp), ("rule", _i32), ("top_k", _i32), ("calibration", _i32),
                ("tau_out", _vp), ("layout", ctypes.POINTER(LayoutPolicy))]


class HardKVError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} returned {code}: {text}")
        self.code = code


_lib = None

_SIGS = {
    "hardkv_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(Desc)]),
    "hardkv_mask_words": (_i32, [ctypes.POINTER(Desc)]),
    "hardkv_validate": (ctypes.c_int, [ctypes.POINTER(Desc)]),
    "hardkv_append": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _vp, _vp, _vp]),
    "hardkv_condense": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _vp]),
    "hardkv_score_calibrate_topp": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp,
                                                   _vp, ctypes.c_float, _i32, _vp, _vp, _vp]),
    "hardkv_score_calibrate_entropy_topp": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache),
                                                           _vp, ctypes.c_float, _i32, _vp, _vp, _vp,
                                                           _vp]),
    "hardkv_score_topk": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _i32, _i32,
                                         _vp, _vp, _vp]),
    "hardkv_regularize": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _i32,
                                         _vp, _vp]),
    "hardkv_regularize_policy": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _i32,
                                                ctypes.POINTER(LayoutPolicy), _vp, _vp]),
    "hardkv_select_from_scores": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _vp,
                                                 ctypes.c_float, _i32, _i32, _i32, _vp, _vp, _vp]),
    "hardkv_flatten_sum": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _vp, _vp]),
    "hardkv_decode_attn": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache), _vp, _vp,
                                          _vp, _vp]),
    "hardkv_decode_step": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache),
                                          ctypes.POINTER(StepArgs), _vp, _vp]),
    "hardkv_decode_step_host": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache),
                                               ctypes.POINTER(StepArgs), _vp, _vp]),
    "hardkv_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "hardkv_selftest_wait_timeout": (ctypes.c_int, [_vp, ctypes.c_uint32, _vp]),
    "hardkv_score_calibrate_topp_static": (ctypes.c_int, [ctypes.POINTER(Desc), ctypes.POINTER(Cache),
                                                          _vp, _vp, ctypes.c_float, _i32, _vp, _vp]),
    "hardkv_static_scratch_bytes": (ctypes.c_size_t, []),
}


def load() -> ctypes.CDLL:
    """Load libhardkv.so (built by attention_kv_head_b200.build). Raises if missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m attention_kv_head_b200.build` (no CPU fallback)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/hardkv.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hardkv_[a-z0-9_]+)\s*\(", text)))


def strerror(code: int) -> str:
    return load().hardkv_strerror(code).decode()


def check(fn: str, code: int) -> None:
    if code != OK:
        raise HardKVError(fn, code, strerror(code))


def call(name: str, *args) -> int:
    """Call entry point `name`; raise HardKVError on a non-zero return."""
    rc = getattr(load(), name)(*args)
    check(name, rc)
    return rc
