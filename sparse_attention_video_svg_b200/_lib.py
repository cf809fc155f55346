"""ctypes loader of libsvg_b200.so with the C ABI signatures of include/svg.h.

The library is built in-tree (``python sparse_attention_video_svg_b200/build.py``).
There is no fallback: if the shared library is missing, importing this module
raises."""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsvg_b200.so")

SVG_OK, SVG_ERR_INVALID_ARG, SVG_ERR_UNSUPPORTED, SVG_ERR_CUDA, SVG_ERR_TIMEOUT = range(5)
SVG_BF16, SVG_FP32 = 0, 1
SVG_MODE_SPATIAL, SVG_MODE_TEMPORAL, SVG_MODE_DENSE = 0, 1, 2
SVG_DEVICE_BAD_LIST_ID, SVG_DEVICE_BAD_INDEX, SVG_DEVICE_TIMEOUT, SVG_DEVICE_CAPACITY = 1, 2, 4, 8
SVG_DEVICE_RANGE = 16
SVG_FUSE_INPUT = 1
SVG_FUSE_OUTPUT = 2
SVG_QK_NORM = 1
SVG_QK_ROPE = 2
SVG_TILE = 128

_p = C.c_void_p
_i = C.c_int
_i64 = C.c_int64
_sz = C.c_size_t
_d = C.c_double
_f = C.c_float

# name -> (restype, argtypes); must match include/svg.h
SIGNATURES = {
    "svg_version": (C.c_char_p, []),
    "svg_last_error": (C.c_char_p, []),
    "svg_set_wait_limit": (_i, [C.c_uint32]),
    "svg_get_wait_limit": (C.c_uint32, []),
    "svg_profile_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "svg_profile_heads": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _i, _p, _p, _p, _sz,
                               _p]),
    "svg_profile_heads_noalloc": (_i, [_p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _i, _p, _p,
                                       _p]),
    "svg_permute_token_major": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "svg_permute_frame_major": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "svg_permute_temporal_heads": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _i, _p, _p]),
    "svg_pair_query_tiles_workspace_size": (_sz, [_i, _i, _i]),
    "svg_pair_query_tiles": (_i, [_p, _p, _i, _i, _i, _p, _p, _p, _sz, _p]),
    "svg_build_block_mask": (_i, [_i, _i, _i, _i, _i, _p, _p, _i64, _i64, _p, _p, _p]),
    "svg_block_energy_workspace_size": (_sz, [_i, _i, _i]),
    "svg_block_energy": (_i, [_p, _p, _i, _i, _i, _i, _i, _p, _p, _sz, _p]),
    "svg_calibrated_workspace_size": (_sz, [_i, _i, _i]),
    "svg_build_block_mask_calibrated": (_i, [_p, _i, _i, _i, _i, _d, _d, _p, _p, _i64, _p, _p, _p,
                                             _sz, _p]),
    "svg_sparse_attn": (_i, [_p, _p, _p, _p, _i, _i, _i, _i, _i, _p, _i, _i, _p, _p, _f, _p, _p,
                             _p]),
    "svg_epsilon_schedule": (_i, [_i, C.c_double, C.c_double, _p]),
    "svg_lists_to_intervals": (_i, [_i, _i, _p, _p, _p, _p, _p, C.c_int64, _p, _p, _p]),
    "svg_lists_to_bitmap": (_i, [_i, _i, _p, _p, _p, _p, _p]),
    "svg_sparse_attn_fused": (_i, [_p, _p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _p,
                                   _i, _i, _i, _p, _p, _p, _f, _p, _p, _p]),
    "svg_v_exponents": (_i, [_p, _i, _i, _i, _i, _i, _p, _p]),
    "svg_qk_norm_rope": (_i, [_p, _p, _p, _p, _p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _p, _f,
                              _p, _p, _p]),
    "svg_row_similarity_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "svg_row_similarity": (_i, [_p, _p, _i, _i, _i, _i, _i, _i, _i, _i, _p, _i, _p, _p, _sz, _p,
                                _p]),
    "svg_anchor_lists": (_i, [_i, _i, _p, _p, _i, _i, _i, _i, _i, _p, _p, _i, _i, _p, _p, _i64,
                              _p, _p, _p, _p]),
    "svg_anchor_list_ids": (_i, [_p, _p, _i, _i, _i, _p, _p]),
    "svg_row_broadcast": (_i, [_p, _i, _i, _i, _i, _i, _i, _i, _i, _i, _p, _i, _p]),
}


class SvgError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed with status {status}: {msg}")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with `python sparse_attention_video_svg_b200/build.py`"
            " (there is no CPU fallback)")
    lib = C.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


def call(name: str, *args) -> None:
    """Calls a status-returning entry point; raises SvgError on failure."""
    st = getattr(lib, name)(*args)
    if st != SVG_OK:
        raise SvgError(name, st, lib.svg_last_error().decode())
