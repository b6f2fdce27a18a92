"""ctypes loader for libswiglu_ffn.so and the C signatures of include/swiglu_ffn.h.

There is no fallback: if the shared library is missing or fails to load, importing the
binding raises, so that no caller can silently run anything else."""
from __future__ import annotations

import ctypes as C
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libswiglu_ffn.so")

SWF_OK = 0
STATUS_NAMES = {0: "SWF_OK", 1: "SWF_ERR_INVALID_ARG", 2: "SWF_ERR_UNSUPPORTED",
                3: "SWF_ERR_ALIGNMENT", 4: "SWF_ERR_WORKSPACE", 5: "SWF_ERR_LAUNCH",
                6: "SWF_ERR_TIMEOUT"}
SWF_F32, SWF_BF16 = 0, 1
OPS = {"fwd": 0, "fwd_infer": 1, "bwd": 2, "select": 3, "sparse_fwd": 4, "sparse_bwd": 5,
       "buckets": 6, "mlp2_fwd": 7, "mlp2_bwd": 8}


class swf_plan_info(C.Structure):
    _fields_ = [("path", C.c_int32), ("tile_m", C.c_int32), ("tile_n", C.c_int32),
                ("tile_k", C.c_int32), ("stages", C.c_int32), ("grid", C.c_int32),
                ("num_kernels", C.c_int32), ("deterministic", C.c_int32),
                ("gemm_tiles", C.c_int64), ("flops", C.c_int64),
                ("workspace_bytes", C.c_size_t), ("saved_bytes", C.c_size_t)]


P, I64, I32, SZ, U64 = C.c_void_p, C.c_int64, C.c_int32, C.c_size_t, C.c_uint64
IP = C.POINTER(C.c_int32)

SIGNATURES = {
    "swiglu_ffn_fwd": (I32, [P, P, P, P, P, P, P, P, I64, I64, I64, I32, P]),
    "swiglu_ffn_fwd_infer": (I32, [P, P, P, P, P, P, SZ, I64, I64, I64, I32, P]),
    "swiglu_ffn_fwd_infer_noalloc": (I32, [P, P, P, P, P, I64, I64, I64, I32, P]),
    "swiglu_ffn_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, P, SZ, I64, I64, I64, I32, P]),
    "leaky_relu_sq_mlp_fwd": (I32, [P, P, P, P, P, P, I64, I64, I64, I32, P]),
    "leaky_relu_sq_mlp_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, SZ, I64, I64, I64, I32, P]),
    "flash_mhffn_fwd": (I32, [P, P, P, P, P, P, I64, I32, I32, I32, I32, I32, P]),
    "flash_mhffn_prologue": (I32, [P, P, P, P, P, P, I64, I64, I32, I32, I32, C.c_float, I32, P]),
    "flash_mhffn_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, P, SZ, I64, I32, I32, I32, I32, I32, P]),
    "flash_mhffn_bwd_workspace_bytes": (SZ, [I64, I32, I32, I32, I32, I32]),
    "flash_mhffn_prologue_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, SZ, I64, I64, I32, I32, I32,
                                       C.c_float, I32, P]),
    "flash_mhffn_prologue_bwd_workspace_bytes": (SZ, [I64, I64, I32, I32, I32, I32]),
    "swf_make_subsample_index": (I32, [I64, I32, I32, U64, P]),
    "grouped_topk_select": (I32, [P, P, P, I32, P, I32, I32, P, P, P, SZ, I64, I64, I64, I32, P]),
    "swf_group_buckets": (I32, [P, I64, I32, I32, P, P, P, SZ, P]),
    "sparse_swiglu_ffn_fwd": (I32, [P, P, P, P, P, I32, I32, P, P, SZ, P, SZ, I64, I64, I64, I32, P]),
    "sparse_swiglu_ffn_bwd": (I32, [P, P, P, P, P, P, P, SZ, P, P, P, P, P, SZ, I64, I64, I64,
                                    I32, I32, I32, P]),
    "swf_group_frequency": (I32, [P, I64, I32, I32, P, P]),
    "update_load_balance_bias": (I32, [P, P, P, C.c_float, C.c_float, C.c_float, C.c_float, I32, P]),
    "swf_workspace_bytes": (SZ, [I32, I64, I64, I64, I32, I32, I32]),
    "swf_sparse_saved_bytes": (SZ, [I64, I64, I64, I32, I32, I32]),
    "swf_supported": (I32, [I32, I64, I64, I64, I32, I32, I32, I32]),
    "swf_plan": (I32, [I32, I64, I64, I64, I32, I32, I32, I32, C.POINTER(swf_plan_info)]),
    "swf_validate_group_idx": (I32, [P, I64, I32, I32, C.POINTER(C.c_int64), P]),
    "swf_set_debug": (I32, [I32]),
    "swf_get_debug": (I32, []),
    "swf_device_status": (I32, [P]),
    "swf_selftest_wait_timeout": (I32, [I32, P]),
    "swf_status_string": (C.c_char_p, [I32]),
    "swf_profile_enable": (I32, [I32]),
    "swf_profile_read": (I32, [I32, P, P]),
    "swf_kernel_name": (C.c_char_p, [I32]),
}


def load(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m swiglu_feed_forward_b200.build` "
            "(the library has no fallback path)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_LIB = None


def lib() -> C.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load()
    return _LIB
