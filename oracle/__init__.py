"""CPU oracle for the dropless top-k MoE layer.

Test infrastructure only: the tests, the smoke check and the benchmark's CPU
baseline import it; the library (dropless_top_moe_b200) never does, and the
two share no code.  float64 numpy throughout.
"""
from . import moe_oracle
from .moe_oracle import *  # noqa: F401,F403
