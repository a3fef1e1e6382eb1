"""ctypes declarations of the C ABI in include/fkv.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfkv.so")

FKV_OK = 0
FKV_ERR_INVALID_ARG = 1
FKV_ERR_SHAPE = 2
FKV_ERR_UNSUPPORTED = 3
FKV_ERR_CUDA = 4
FKV_ERR_TIMEOUT = 5
FKV_ERR_WORKSPACE = 6
FKV_ERR_DEVICE_ARG = 7

FKV_DTYPE_BF16 = 0
FKV_DTYPE_FP32 = 1
FKV_GRAN_FRAME = 0
FKV_GRAN_TOKEN = 1
FKV_FLAG_SCORE_WITH_CHUNK = 1
FKV_FLAG_STATIC_TOKEN_MASK = 2
FKV_POLICY_UNIFORM = 0
FKV_POLICY_RANDOM = 1

c_i32, c_i64, c_f32, c_vp, c_sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t


class Params(ctypes.Structure):
    """fkv_params_t."""

    _fields_ = [
        ("num_layers", c_i32), ("num_heads", c_i32), ("head_dim", c_i32),
        ("frame_tokens", c_i32), ("hist_frames", c_i32), ("chunk_frames", c_i32),
        ("score_stride", c_i32), ("n_score_q", c_i32), ("sink_tokens", c_i32),
        ("recent_tokens", c_i32), ("comp_rows", c_i32), ("scale", c_f32),
        ("dtype", c_i32), ("granularity", c_i32), ("flags", c_i32),
    ]


STEP_IO_FIELDS = (
    "q_cur", "k_cur", "v_cur", "k_hist", "v_hist", "q_score", "head_role", "static_mask",
    "k_per_head", "seg_score", "kept_idx", "kept_cnt", "k_comp", "v_comp", "out",
)


class StepIO(ctypes.Structure):
    """fkv_step_io_t."""

    _fields_ = [(n, c_vp) for n in STEP_IO_FIELDS]


FP8_CACHE_FIELDS = (
    "k_comp", "v_comp", "k_comp_scale", "v_comp_scale", "k_cur", "v_cur", "k_cur_scale",
    "v_cur_scale", "q_cur", "q_scale",
)


class Fp8Cache(ctypes.Structure):
    """fkv_fp8_cache_t."""

    _fields_ = [(n, c_vp) for n in FP8_CACHE_FIELDS]


# name -> (restype, argtypes), exactly the declarations of include/fkv.h
SIGNATURES = {
    "fkv_status_string": (ctypes.c_char_p, [c_i32]),
    "fkv_abi_version": (c_i32, []),
    "fkv_check_params": (c_i32, [ctypes.POINTER(Params)]),
    "fkv_num_segments": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(c_i64)]),
    "fkv_max_kept": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(c_i64)]),
    "fkv_max_comp_rows": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(c_i64)]),
    "fkv_workspace_size": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(c_sz)]),
    "fkv_step_launches": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(c_i32)]),
    "fkv_exp2_emulated": (c_i32, [c_vp, c_vp, c_i64, c_vp]),
    "fkv_diag_attend_timeout": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp,
                                        c_vp, c_i64, c_vp, c_vp]),
    "fkv_diag_mma_rate": (c_i32, [c_i32, c_i32, c_i32, c_vp, c_vp, c_vp]),
    "fkv_diag_ex2_rate": (c_i32, [c_i32, c_i32, c_vp, c_vp]),
    "fkv_workspace_init": (c_i32, [c_vp, c_sz, c_vp]),
    "fkv_read_status": (c_i32, [c_vp, c_vp, ctypes.POINTER(c_i32), ctypes.POINTER(c_i32)]),
    "fkv_score_segments": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "fkv_score_segments_noalloc": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "fkv_select_topk": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "fkv_compact_gather": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "fkv_attend_compressed": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "fkv_compact_gather_rope": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, c_vp, c_vp]),
    "fkv_cache_advance": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp, c_vp, c_i64, c_vp, c_vp, c_vp, c_vp]),
    "fkv_step": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(StepIO), c_vp, c_vp]),
    "fkv_select_heuristic": (c_i32, [ctypes.POINTER(Params), c_i32, ctypes.c_uint64, c_vp, c_vp, c_vp,
                                     c_vp, c_vp, c_vp]),
    "fkv_compact_gather_fp8": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp, c_vp,
                                       ctypes.POINTER(Fp8Cache), c_vp, c_vp]),
    "fkv_quantize_chunk_fp8": (c_i32, [ctypes.POINTER(Params), c_vp, c_vp, c_vp,
                                       ctypes.POINTER(Fp8Cache), c_vp, c_vp]),
    "fkv_attend_compressed_fp8": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(Fp8Cache), c_vp,
                                          c_vp, c_vp, c_vp]),
    "fkv_step_fp8": (c_i32, [ctypes.POINTER(Params), ctypes.POINTER(StepIO), ctypes.POINTER(Fp8Cache),
                             c_vp, c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Loads the in-tree libfkv.so.  There is no fallback: a missing library is an error."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is not built; run `python -m kv_cache_compression_fkv_b200.build` "
            "(needs nvcc).  The package has no CPU fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
