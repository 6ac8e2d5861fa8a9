"""ctypes declarations of the C ABI in include/svg.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import threading

from .build import LIB_PATH

SVG_OK, SVG_ERR_INVALID_ARG, SVG_ERR_SHAPE, SVG_ERR_UNSUPPORTED = 0, 1, 2, 3
SVG_ERR_ALIGNMENT, SVG_ERR_CAPACITY, SVG_ERR_CUDA, SVG_ERR_TIMEOUT = 4, 5, 6, 7
SVG_HEAD_SPATIAL, SVG_HEAD_TEMPORAL, SVG_HEAD_DENSE = 0, 1, 2
SVG_STEP_DENSE, SVG_STEP_PROFILE, SVG_STEP_REUSE = 0, 1, 2
SVG_NORM_ROPE, SVG_LAYOUT = 1, 2


class SvgShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int), ("d", ctypes.c_int),
                ("F", ctypes.c_int), ("Hs", ctypes.c_int), ("Ws", ctypes.c_int), ("text_len", ctypes.c_int)]


class SvgParams(ctypes.Structure):
    _fields_ = [("spatial_frames", ctypes.c_int), ("temporal_radius", ctypes.c_int),
                ("block_q", ctypes.c_int), ("block_k", ctypes.c_int),
                ("eps", ctypes.c_float), ("rope_base", ctypes.c_float),
                ("rope_split", ctypes.c_int * 3), ("softmax_scale", ctypes.c_float)]


class SVGError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lock = threading.Lock()
_lib = None

# name -> (restype, argtypes)
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SP, _PP = ctypes.POINTER(SvgShape), ctypes.POINTER(SvgParams)
SIGNATURES = {
    "svg_qknorm_rope_layout": (_i32, [_SP, _PP, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svg_profile_heads": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp, _vp, _vp]),
    "svg_profile_heads_raw_q": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _sz, _vp, _vp, _vp]),
    "svg_profile_heads_noalloc": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp]),
    "svg_build_block_index": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _i64, _vp]),
    "svg_block_sparse_attn": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svg_block_sparse_attn_model_order": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svg_inverse_layout": (_i32, [_SP, _vp, _vp, _vp, _vp]),
    "svg_attention_step": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64,
                                  _vp, _sz, _vp]),
    "svg_attention_step_host_workspace_size": (_sz, [_SP, _PP, _i32, _i32]),
    "svg_attention_step_host": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _vp, _sz,
                                       _vp]),
    "svg_sample_queries": (_i32, [ctypes.c_uint64, _i64, _i32, _vp]),
    "svg_adaspa_block_mass": (_i32, [_SP, _PP, _vp, _vp, _vp, _vp, _vp]),
    "svg_adaspa_select": (_i32, [_SP, _PP, _vp, ctypes.c_double, _vp, _vp, _vp, _i64, _vp]),
    "svg2_kmeans_workspace_size": (_sz, [_SP, _i32]),
    "svg2_kmeans": (_i32, [_SP, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "svg2_permutation": (_i32, [_SP, _vp, _i32, _vp, _vp, _vp]),
    "svg2_select": (_i32, [_SP, _PP, _vp, _vp, _vp, _i32, _i32, ctypes.c_double, _vp, _vp]),
    "svg2_permute": (_i32, [_SP, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "svg2_build_block_index": (_i32, [_SP, _PP, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]),
    "svg2_attention": (_i32, [_SP, _PP, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                              _vp]),
    "svg_step_policy": (_i32, [_i32, _i32, ctypes.c_float, _i32, ctypes.POINTER(ctypes.c_int)]),
    "svg_rope_table_size": (_sz, [_SP, _PP]),
    "svg_rope_table_fill": (_i32, [_SP, _PP, _vp]),
    "svg_block_index_capacity": (_i64, [_SP, _PP]),
    "svg_profile_workspace_size": (_sz, [_SP, _i32]),
    "svg_workspace_size": (_sz, [_SP, _PP]),
    "svg_release": (_i32, []),
    "svg_sync_status": (_i32, [_vp]),
    "svg_selftest_wait_timeout": (_i32, [_vp]),
    "svg_status_string": (ctypes.c_char_p, [_i32]),
    "svg_version": (ctypes.c_char_p, []),
}


def lib():
    """The loaded library.  Raises if it has not been built: there is no
    fallback implementation."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library missing: {LIB_PATH}; build it with "
                                   "`python -m sparse_attention_video_qk_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().svg_status_string(status).decode()
    except Exception:  # library not loadable: still report the number
        return f"status {status}"


def check(status: int, where: str):
    if status != SVG_OK:
        raise SVGError(status, where)
