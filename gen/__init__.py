"""Seeded input generators shared by the oracle-based tests and the CUDA path."""
from .moe_inputs import (MoEShape, WORKLOADS, WORKLOAD_ORDER, make_inputs, make_router,
                         token_rows, resample_rows, expert_bias, random_counts)

__all__ = ["MoEShape", "WORKLOADS", "WORKLOAD_ORDER", "make_inputs", "make_router",
           "token_rows", "resample_rows", "expert_bias", "random_counts"]
