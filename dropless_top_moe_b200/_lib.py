"""ctypes declarations of libmoe_b200.so (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Loading fails loudly when the library has not been built.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA = range(5)
MOE_F32, MOE_BF16 = 0, 1
MOE_DEVERR_EXPERT_ID, MOE_DEVERR_TIMEOUT, MOE_DEVERR_ROWS, MOE_DEVERR_MODE = 1, 2, 4, 8
MOE_LAYER_GATHER_ROWS = 4   # flag OR-ed into the layer's training mode
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_WORKSPACE", 4: "MOE_ERR_CUDA"}

P, I32, I64, SZ, FL = C.c_void_p, C.c_int32, C.c_int64, C.c_size_t, C.c_float

# name -> (restype, argtypes); mirrors include/moe.h one to one
SIGNATURES = {
    "moe_tile_rows": (I32, []),
    "moe_padded_rows_max": (I64, [I32, I32, I32]),
    "moe_route_workspace_size": (SZ, [I32, I32, I32, I32, I32]),
    "moe_dispatch_meta_workspace_size": (SZ, [I32, I32, I32]),
    "moe_grouped_workspace_size": (SZ, []),
    "moe_unpermute_router_bwd_workspace_size": (SZ, [I32, I32, I32, I64]),
    "moe_aux_loss_workspace_size": (SZ, [I32, I32]),
    "moe_workspace_size": (SZ, [I32, I32, I32, I32, I32, I32, I32]),
    "moe_workspace_init": (I32, [P, SZ, P]),
    "moe_get_device_status": (I32, [P, P, P]),
    "moe_route": (I32, [P, P, I32, I32, I32, I32, I32, P, P, P, P, P, SZ, P]),
    "moe_dispatch_meta": (I32, [P, I32, I32, I32, I32, P, P, P, P, P, P, SZ, P]),
    "moe_permute": (I32, [P, P, P, P, I32, I32, I32, I32, I32, P, P]),
    "moe_grouped_swiglu": (I32, [P, P, P, P, P, I32, I32, I32, I64, I32, P, P, P, P, SZ, P]),
    "moe_combine": (I32, [P, P, P, I32, I32, I32, I32, P, P]),
    "moe_combine_bwd": (I32, [P, P, P, P, P, P, I32, I32, I32, I32, I32, P, P, P, P]),
    "moe_grouped_swiglu_bwd": (I32, [P, P, P, P, P, P, P, P, I32, I32, I32, I64, I32,
                                     P, P, P, P, P, P, SZ, P]),
    "moe_unpermute_router_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, FL, FL, I32, I32, I32, I32, I64,
                                       I32, P, P, P, SZ, P]),
    "moe_aux_loss": (I32, [P, P, I32, I32, I32, FL, P, P, P, SZ, P]),
    "moe_layer_fwd": (I32, [P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I32, FL, P, P, P, P,
                            P, P, P, P, SZ, P]),
    "moe_layer_bwd": (I32, [P, P, P, P, P, P, P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32, I32,
                            FL, FL, P, P, P, P, P, P, SZ, P]),
    "moe_dispatch_meta_noalloc": (I32, [P, I32, I32, I32, P, P, P, P, P, P, P]),
    "moe_sum_rank_ordered": (I32, [P, I32, I64, I32, FL, P, P]),
    "moe_selftest_wait_timeout": (I32, [P, I64, P]),
    "moe_trace_attach": (I32, [P, I32, P, P]),
    "moe_trace_detach": (I32, []),
}

_lib = None


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS_NAMES.get(code, code)}")
        self.code = code


def load(path: str = LIB_PATH) -> C.CDLL:
    """Open the library (once) and declare every exported function."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m dropless_top_moe_b200.build`")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def call(name: str, *args) -> None:
    """Call a status-returning entry point and raise MoEError unless MOE_OK."""
    code = getattr(load(), name)(*args)
    if code != MOE_OK:
        raise MoEError(name, code)
