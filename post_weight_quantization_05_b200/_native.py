"""ctypes loader for libgptq.so (the C ABI in include/gptq.h).

Loading needs no GPU: the library links the CUDA runtime statically and
reaches the driver only when a call is made.  There is no fallback: if the
library is missing, every entry point raises.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgptq.so")

c_i64 = ctypes.c_int64
c_int = ctypes.c_int
c_vp = ctypes.c_void_p
c_size = ctypes.c_size_t
c_float = ctypes.c_float

# name -> (restype, argtypes)
SIGNATURES = {
    "gptq_abi_version": (c_int, []),
    "gptq_launch_count": (ctypes.c_uint64, []),
    "gptq_status_string": (ctypes.c_char_p, [c_int]),
    "gptq_hessian_workspace_size": (c_size, [c_int, c_i64, c_i64]),
    "gptq_hessian_accumulate": (c_int, [c_vp, c_int, c_i64, c_i64, c_vp, c_vp, c_size, c_vp]),
    "gptq_hessian_accumulate_batches": (c_int, [c_vp, c_vp, c_int, c_int, c_i64, c_vp, c_vp, c_size, c_vp]),
    "gptq_prepare_hinv_workspace_size": (c_size, [c_i64]),
    "gptq_prepare_hinv": (c_int, [c_vp, c_i64, c_float, c_vp, c_vp, c_vp, c_size, c_vp]),
    "gptq_quantize_workspace_size": (c_size, [c_i64, c_i64, c_int]),
    "gptq_quantize_layer": (c_int, [c_vp, c_i64, c_i64, c_vp, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp,
                                    c_vp, c_size, c_vp]),
    "gptq_quantize_layer_noalloc": (c_int, [c_vp, c_i64, c_i64, c_vp, c_int, c_int, c_int, c_vp, c_vp, c_vp, c_vp,
                                            c_vp]),
    "gptq_rtn_layer": (c_int, [c_vp, c_i64, c_i64, c_int, c_int, c_vp, c_vp, c_vp, c_vp, c_vp]),
    "gptq_act_order_perm": (c_int, [c_vp, c_i64, c_vp, c_vp]),
    "gptq_permute_hessian": (c_int, [c_vp, c_i64, c_vp, c_vp, c_vp]),
    "gptq_permute_columns": (c_int, [c_vp, c_i64, c_i64, c_vp, c_int, c_vp, c_vp]),
    "gptq_dequant_gemv_workspace_size": (c_size, [c_i64, c_i64, c_int]),
    "gptq_dequant_gemv": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_int, c_int, c_vp, c_vp, c_i64, c_vp, c_vp,
                                  c_size, c_vp]),
    "gptq_dequantize": (c_int, [c_vp, c_vp, c_vp, c_i64, c_i64, c_int, c_int, c_vp, c_int, c_vp, c_vp]),
    "gptq_widen_bf16": (c_int, [c_vp, c_vp, c_i64, c_vp]),
    "gptq_fill_f32": (c_int, [c_vp, c_i64, c_float, c_vp]),
    "gptq_get_status": (c_int, [c_vp, ctypes.POINTER(c_int)]),
}

STATUS = {0: "GPTQ_OK", 1: "GPTQ_ERR_INVALID_ARG", 2: "GPTQ_ERR_UNSUPPORTED", 3: "GPTQ_ERR_NOT_PD",
          4: "GPTQ_ERR_NONFINITE", 5: "GPTQ_ERR_GRID", 6: "GPTQ_ERR_TIMEOUT", 7: "GPTQ_ERR_CUDA"}
GPTQ_F32, GPTQ_BF16 = 0, 1

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load (once) and type the library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libgptq.so not found at {path}; build it with "
                           "`python -m post_weight_quantization_05_b200.build_lib`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib
