"""ctypes declarations of the libzb C ABI (include/zb.h)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libzb.so")

c_i32, c_i64, c_f32, c_sz, c_vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p


class ZbShape(ctypes.Structure):
    _fields_ = [("heads", c_i32), ("n_tokens", c_i64), ("head_dim", c_i32), ("tile", c_i32)]


STATUS = {
    0: "ZB_OK", 1: "ZB_ERR_NULL", 2: "ZB_ERR_SHAPE", 3: "ZB_ERR_ALIGN", 4: "ZB_ERR_UNSUPPORTED",
    5: "ZB_ERR_WORKSPACE", 6: "ZB_ERR_CUDA", 7: "ZB_ERR_TIMEOUT", 8: "ZB_ERR_DEVICE",
    9: "ZB_ERR_INDEX", 10: "ZB_ERR_SINGULAR",
}

# name -> (restype, argtypes); every function declared in include/zb.h
PROTOTYPES = {
    "zb_abi_version": (c_i32, []),
    "zb_status_string": (ctypes.c_char_p, [c_i32]),
    "zb_landmark_build": (c_i32, [c_vp, c_vp, c_vp, ZbShape, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "zb_tile_score_topk_workspace_bytes": (c_sz, [ZbShape]),
    "zb_tile_score_topk": (c_i32, [c_vp, c_vp, ZbShape, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "zb_tile_sparse_attn_workspace_bytes": (c_sz, []),
    "zb_tile_sparse_attn": (c_i32, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_i32, c_f32, ZbShape,
                                    c_vp, c_vp, c_vp, c_sz, c_vp]),
    "zb_dense_attn": (c_i32, [c_vp, c_i64, c_vp, c_vp, c_i64, c_i32, c_i32, c_f32, c_vp, c_i32, c_vp, c_vp]),
    "zb_dense_attn_split_workspace_bytes": (c_sz, [c_i64, c_i32, c_i32, c_i32]),
    "zb_dense_attn_split": (c_i32, [c_vp, c_i64, c_vp, c_vp, c_i64, c_i32, c_i32, c_f32, c_i32, c_vp, c_i32, c_vp,
                                    c_vp, c_sz, c_vp]),
    "zb_linear_state_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32]),
    "zb_linear_state": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "zb_linear_state_static_scratch_bytes": (c_sz, []),
    "zb_linear_state_static": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp]),
    "zb_linear_apply": (c_i32, [c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp]),
    "zb_spatial_order": (c_i32, [c_i32, c_i32, c_i32, c_i32, c_i32, c_vp, c_vp]),
    "zb_gather_rows": (c_i32, [c_vp, c_i32, c_i64, c_i64, c_i32, c_vp, c_vp, c_vp]),
    "zb_linear_attn_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32]),
    "zb_linear_attn": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "zb_key_mean_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32]),
    "zb_key_mean": (c_i32, [c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_sz, c_vp]),
    "zb_linear_state_centered": (c_i32, [c_vp, c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "zb_block_mass": (c_i32, [c_vp, c_vp, c_vp, ZbShape, c_f32, c_vp, c_vp]),
    "zb_block_mass_top_fraction": (c_i32, [c_vp, c_i32, c_i32, c_i32, c_vp, c_vp]),
    "zb_block_mass_selected_fraction": (c_i32, [c_vp, c_i32, c_i32, c_vp, c_i32, c_vp, c_vp]),
    "zb_affine_fit_workspace_bytes": (c_sz, [c_i32, c_i64, c_i32]),
    "zb_affine_fit": (c_i32, [c_vp, c_vp, c_i32, c_i64, c_i32, c_vp, c_vp, c_vp, c_sz, c_vp]),
    "zb_gather_tiles": (c_i32, [c_vp, ZbShape, c_vp, c_i32, c_vp, c_vp]),
    "zb_last_device_status": (c_i32, [c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libzb.so (built in-tree); raises ImportError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m linear_hybrid_attention_b200.build` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
