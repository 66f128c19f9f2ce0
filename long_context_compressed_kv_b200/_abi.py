"""ctypes mirror of include/v4attn.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libv4attn.so")

# status codes
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE_CHECK = range(7)
# dtypes
F32, BF16, E4M3_BF16ROPE, MXFP4 = range(4)
NOALLOC_MAX_SCORES = 2097152   # V4A_NOALLOC_MAX_SCORES
NOALLOC_MAX_QUERIES = 1365     # V4A_NOALLOC_MAX_QUERIES
# layer kinds
CSA, HCA = 0, 1

c_i32, c_i64, c_f32, c_ptr, c_sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                    ctypes.c_void_p, ctypes.c_size_t)


class LayerDesc(ctypes.Structure):
    _fields_ = [("kind", c_i32), ("m", c_i32), ("n_win", c_i32), ("H", c_i32), ("d", c_i32),
                ("d_rope", c_i32), ("rope_theta", c_f32), ("softmax_scale", c_f32),
                ("H_I", c_i32), ("d_I", c_i32), ("top_k", c_i32), ("kv_dtype", c_i32),
                ("idx_dtype", c_i32), ("rms_eps", c_f32)]


class CompressArgs(ctypes.Structure):
    _fields_ = [("m", c_i32), ("overlap", c_i32), ("c", c_i32), ("B", c_i32),
                ("Ca", c_ptr), ("Za", c_ptr), ("Cb", c_ptr), ("Zb", c_ptr),
                ("in_dtype", c_i32), ("in_seq_stride", c_i64), ("in_row_stride", c_i64),
                ("in_rows", c_i64), ("bias", c_ptr), ("seq_len", c_ptr), ("entry_begin", c_ptr),
                ("n_entries", c_i32), ("complete_only", c_i32), ("apply_rmsnorm", c_i32),
                ("apply_rope", c_i32), ("out_dtype", c_i32), ("out", c_ptr), ("out_scale", c_ptr),
                ("out_rows", c_i64)]


class IndexArgs(ctypes.Structure):
    _fields_ = [("n_q", c_i32), ("B", c_i32), ("qI", c_ptr), ("qI_sf", c_ptr), ("w", c_ptr),
                ("q_seq", c_ptr), ("q_pos", c_ptr), ("keys", c_ptr), ("keys_sf", c_ptr),
                ("key_rows", c_i64), ("max_vis", c_i64), ("idx_out", c_ptr),
                ("scores_out", c_ptr), ("score_dtype", c_i32), ("block_table", c_ptr),
                ("blocks_per_seq", c_i32)]


class MqaArgs(ctypes.Structure):
    _fields_ = [("n_q", c_i32), ("B", c_i32), ("Q", c_ptr), ("q_dtype", c_i32),
                ("q_rmsnorm", c_i32), ("q_seq", c_ptr), ("q_pos", c_ptr), ("kv", c_ptr),
                ("kv_scale", c_ptr), ("kv_rows", c_i64), ("swa", c_ptr), ("swa_scale", c_ptr),
                ("swa_rows", c_i64), ("idx", c_ptr), ("n_sel", c_i32), ("max_vis", c_i64),
                ("sink", c_ptr), ("out", c_ptr), ("out_dtype", c_i32), ("lse", c_ptr),
                ("block_table", c_ptr), ("blocks_per_seq", c_i32)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("B", c_i32), ("pos", c_ptr), ("in_dtype", c_i32), ("x_main", c_ptr),
                ("tail", c_ptr), ("bias", c_ptr), ("x_idx", c_ptr), ("itail", c_ptr),
                ("ibias", c_ptr), ("kv", c_ptr), ("kv_scale", c_ptr), ("kv_rows", c_i64),
                ("keys", c_ptr), ("keys_sf", c_ptr), ("key_rows", c_i64), ("swa", c_ptr),
                ("swa_scale", c_ptr), ("swa_rows", c_i64), ("Q", c_ptr), ("q_dtype", c_i32),
                ("qI", c_ptr), ("qI_sf", c_ptr), ("w", c_ptr), ("sink", c_ptr), ("out", c_ptr),
                ("out_dtype", c_i32), ("lse", c_ptr), ("idx_out", c_ptr), ("max_vis", c_i64),
                ("block_table", c_ptr), ("blocks_per_seq", c_i32)]


class ProjectArgs(ctypes.Structure):
    _fields_ = [("M", c_i64), ("N", c_i64), ("K", c_i64), ("X", c_ptr), ("x_dtype", c_i32),
                ("ldx", c_i64), ("W", c_ptr), ("w_dtype", c_i32), ("ldw", c_i64), ("Y", c_ptr),
                ("y_dtype", c_i32), ("ldy", c_i64)]


STRUCTS = {"v4attn_layer_desc": LayerDesc, "v4attn_compress_args": CompressArgs,
           "v4attn_index_args": IndexArgs, "v4attn_mqa_args": MqaArgs,
           "v4attn_decode_args": DecodeArgs, "v4attn_project_args": ProjectArgs}

# entry point -> (restype, argtypes)
SIGNATURES = {
    "v4attn_workspace_size": (c_sz, [ctypes.POINTER(LayerDesc), c_i32, c_i64]),
    "v4attn_workspace_init": (ctypes.c_int, [c_ptr, c_sz, c_ptr]),
    "v4attn_compress": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(CompressArgs),
                                       c_ptr, c_sz, c_ptr]),
    "v4attn_index_topk": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(IndexArgs),
                                         c_ptr, c_sz, c_ptr]),
    "v4attn_sparse_mqa": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(MqaArgs),
                                         c_ptr, c_sz, c_ptr]),
    "v4attn_dense_mqa": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(MqaArgs),
                                        c_ptr, c_sz, c_ptr]),
    "v4attn_decode": (ctypes.c_int, [ctypes.POINTER(LayerDesc), ctypes.POINTER(DecodeArgs),
                                     c_ptr, c_sz, c_ptr]),
    "v4attn_project": (ctypes.c_int, [ctypes.POINTER(ProjectArgs), c_ptr]),
    "v4attn_index_topk_noalloc": (ctypes.c_int, [ctypes.POINTER(LayerDesc),
                                                 ctypes.POINTER(IndexArgs), c_ptr]),
    "v4attn_noalloc_device_status": (ctypes.c_int, [c_ptr, ctypes.POINTER(ctypes.c_uint32)]),
    "v4attn_debug_index_stall": (ctypes.c_int, [ctypes.POINTER(LayerDesc),
                                                ctypes.POINTER(IndexArgs), c_ptr, c_sz,
                                                ctypes.c_uint32, c_ptr]),
    "v4attn_tc_peak_probe": (ctypes.c_int, [c_i32, c_i32, c_i32, ctypes.POINTER(c_i32),
                                            ctypes.POINTER(ctypes.c_double), c_ptr, c_ptr]),
    "v4attn_device_status": (ctypes.c_int, [c_ptr, c_ptr, ctypes.POINTER(ctypes.c_uint32)]),
    "v4attn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "v4attn_build_info": (ctypes.c_char_p, []),
    "v4attn_last_cuda_error": (ctypes.c_char_p, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libv4attn.so; raises if it has not been built (no fallback exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python long_context_compressed_kv_b200/csrc/build.py` (there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
