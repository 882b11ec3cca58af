"""ctypes loader for ``_lib/libnvfp4moe.so``: the C ABI declared in ``include/nvfp4_moe.h``.

Loading fails loudly when the library is missing; there is no fallback implementation.
"""

import ctypes
import os

from .build import LIB

c_int = ctypes.c_int
c_i64 = ctypes.c_int64
c_size = ctypes.c_size_t
c_void = ctypes.c_void_p
c_char_p = ctypes.c_char_p
c_float = ctypes.c_float

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_UNSUPPORTED_SHAPE",
    3: "NVFP4_ERR_MISALIGNED", 4: "NVFP4_ERR_WORKSPACE_TOO_SMALL", 5: "NVFP4_ERR_CUDA",
    6: "NVFP4_ERR_TIMEOUT", 7: "NVFP4_ERR_BAD_INDEX",
}

# name -> (restype, argtypes), in header order
SIGNATURES = {
    "nvfp4_quantize_workspace_size": (c_size, []),
    "nvfp4_quantize": (c_int, [c_void, c_i64, c_i64, c_i64, c_void, c_int, c_i64, c_void, c_void,
                               c_void, c_int, c_void, c_size, c_void, c_void]),
    "mxfp4_quantize": (c_int, [c_void, c_i64, c_i64, c_i64, c_void, c_void, c_void, c_void]),
    "nvfp4_rmsnorm_quantize_workspace_size": (c_size, [c_i64]),
    "nvfp4_rmsnorm_quantize": (c_int, [c_void, c_i64, c_i64, c_i64, c_void, c_float, c_void, c_int,
                                       c_i64, c_void, c_void, c_void, c_int, c_void, c_size, c_void,
                                       c_void]),
    "moe_rows_max": (c_i64, [c_int, c_int, c_int]),
    "moe_permute_workspace_size": (c_size, [c_int, c_int, c_int]),
    "moe_permute": (c_int, [c_void, c_int, c_int, c_int, c_int, c_void, c_void, c_void, c_void,
                            c_void, c_void, c_void, c_size, c_void, c_void]),
    "nvfp4_grouped_gemm": (c_int, [c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_int,
                                   c_int, c_int, c_i64, c_void, c_int, c_void, c_void]),
    "mxfp4_grouped_gemm": (c_int, [c_void, c_void, c_void, c_void, c_void, c_int, c_int, c_int,
                                   c_i64, c_void, c_int, c_void, c_void]),
    "nvfp4_gemm_dense_workspace_size": (c_size, [c_i64, c_int, c_int]),
    "nvfp4_gemm_dense": (c_int, [c_void, c_void, c_void, c_i64, c_void, c_void, c_void, c_int, c_int,
                                 c_void, c_void, c_size, c_void, c_void]),
    "nvfp4_linear_workspace_size": (c_size, [c_i64, c_int, c_int]),
    "nvfp4_linear": (c_int, [c_void, c_i64, c_int, c_i64, c_void, c_float, c_void, c_void, c_void,
                             c_int, c_void, c_void, c_size, c_void, c_void]),
    "nvfp4_shared_expert_workspace_size": (c_size, [c_i64, c_int, c_int]),
    "nvfp4_shared_expert": (c_int, [c_void, c_i64, c_int, c_i64, c_void, c_float, c_void, c_void,
                                    c_void, c_void, c_void, c_void, c_int, c_void, c_void, c_void,
                                    c_size, c_void, c_void]),
    "moe_grouped_gemm_l1_swiglu_q": (c_int, [c_void, c_void, c_void, c_void, c_void, c_void,
                                             c_void, c_void, c_int, c_int, c_int, c_i64, c_void,
                                             c_void, c_void, c_void, c_void]),
    "moe_grouped_gemm_l1_swiglu_q_stats": (c_int, [c_void, c_void, c_void, c_void, c_void, c_void,
                                                   c_void, c_void, c_int, c_int, c_int, c_i64,
                                                   c_void, c_void, c_void, c_void, c_void, c_void,
                                                   c_void]),
    "nvfp4_scale_from_amax": (c_int, [c_void, c_void, c_void]),
    "moe_grouped_gemm_l2_scatter": (c_int, [c_void, c_void, c_void, c_void, c_void, c_void, c_void,
                                            c_void, c_void, c_void, c_int, c_int, c_int, c_int,
                                            c_int, c_i64, c_void, c_void, c_void, c_void, c_void]),
    "moe_grouped_gemm_l2_scatter_add": (c_int, [c_void, c_void, c_void, c_void, c_void, c_void,
                                                c_void, c_void, c_void, c_void, c_int, c_int,
                                                c_int, c_int, c_int, c_i64, c_void, c_void,
                                                c_void, c_void]),
    "moe_ffn_l2_form": (c_int, [c_int, c_int, c_int, c_int]),
    "moe_grouped_gemm_l2_scatter_noalloc": (c_int, [c_void, c_void, c_void, c_void, c_void,
                                                    c_void, c_void, c_void, c_void, c_void, c_int,
                                                    c_int, c_int, c_int, c_int, c_i64, c_void,
                                                    c_void, c_void]),
    "moe_w1_row_map": (c_int, [c_int, c_void]),
    "moe_ffn_workspace_size": (c_size, [c_int, c_int, c_int, c_int, c_int]),
    "moe_ffn_forward": (c_int, [c_void, c_void, c_int, c_int, c_int, c_int, c_int, c_void, c_void,
                                c_void, c_void, c_void, c_void, c_void, c_void, c_void, c_size,
                                c_void, c_void]),
    "moe_ffn_forward_ex": (c_int, [c_void, c_void, c_int, c_int, c_int, c_int, c_int, c_void,
                                   c_void, c_void, c_void, c_void, c_void, c_void, c_int, c_void,
                                   c_void, c_void, c_size, c_void, c_void]),
    "nvfp4_read_status": (c_int, [c_void, c_void, c_void]),
    "nvfp4_wait_selftest": (c_int, [c_i64, c_void, c_void, c_void]),
    "nvfp4_last_error": (c_char_p, []),
    "nvfp4_abi_version": (c_int, []),
}

_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(
                f"{LIB} is missing: build it with `python -m nvfp4_block_scaled_gsa_b200.build` "
                "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


class Nvfp4Error(RuntimeError):
    def __init__(self, fn, code):
        msg = STATUS.get(code, str(code))
        detail = lib().nvfp4_last_error()
        if code == 5 and detail:
            msg += f" ({detail.decode(errors='replace')})"
        super().__init__(f"{fn}: {msg}")
        self.code = code


def call(name, *args):
    """Call a status-returning entry point; raise Nvfp4Error unless it returns NVFP4_OK."""
    rc = getattr(lib(), name)(*args)
    if rc != 0:
        raise Nvfp4Error(name, rc)
    return rc
