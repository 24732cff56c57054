"""B200-native dropless top-k Mixture-of-Experts layer (sm_100a CUDA kernels
behind a C ABI, include/moe.h).  Python here only marshals arguments."""
from ._lib import LIB_PATH, MOE_LAYER_GATHER_ROWS, MoEError, load
from .ops import (MoELayer, device_status, moe_aux_loss, moe_combine, moe_combine_bwd, moe_dispatch_meta,
                  moe_grouped_swiglu, moe_grouped_swiglu_bwd, moe_permute, moe_route,
                  moe_unpermute_router_bwd, padded_rows_max, selftest_wait_timeout, tile_rows, workspace)

__all__ = ["LIB_PATH", "MOE_LAYER_GATHER_ROWS", "MoEError", "load", "MoELayer", "device_status", "moe_aux_loss", "moe_combine",
           "moe_combine_bwd", "moe_dispatch_meta", "moe_grouped_swiglu", "moe_grouped_swiglu_bwd",
           "moe_permute", "moe_route", "moe_unpermute_router_bwd", "padded_rows_max", "selftest_wait_timeout",
           "tile_rows",
           "workspace"]
