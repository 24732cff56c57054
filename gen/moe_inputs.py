"""Seeded synthetic inputs for the dropless top-k MoE layer.

This module only draws random numbers and lays them out; it computes nothing
of the layer itself (no matmul, softmax, top-k, sort or expert FFN).  Both the
CPU oracle and the CUDA path receive the tensors it returns.

Workload shapes follow the pages' problem statement: tokens x[N, H], router
W_r[H, E], per-expert SwiGLU weights W1, W3 [H, F] and W2 [F, H] stacked into
contiguous [E, ...] tensors ("MoE computation principle", section 2.1-2.3;
MoonEP "memory contract", section 03, one contiguous weight tensor indexed by
expert row).

Streams (one torch.Generator per tensor, so that any tensor can be regenerated
alone): x = seed, W_r = seed+1, W1 = seed+2, W3 = seed+3, W2 = seed+4,
dy = seed+5, expert bias = seed+6, row resampling = seed+7 (+round).

Distributions: x ~ N(0, 1); W_r ~ N(0, 0.02^2) (the pages' example draws the
router as randn * 0.02); W1, W3 ~ N(0, 1/H) and W2 ~ N(0, 1/F), i.e. standard
deviation 1/sqrt(fan_in); dy ~ N(0, 1).

Skewed routing is produced without a router bias term: column 0 of every token
is set to exactly 1 and row 0 of W_r holds the per-expert bias b_e, so that the
layer's own router GEMM adds b_e to every token's logit for expert e.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class MoEShape:
    """One workload: sizes, arithmetic type and routing-skew recipe."""
    name: str
    N: int
    H: int
    E: int
    K: int
    F: int
    dtype: str = "bf16"          # "f32" or "bf16"
    skew: Optional[str] = None   # None, "normal" (b_e ~ N(0, sigma^2)) or "zipf"
    skew_param: float = 0.0      # sigma for "normal", tau for "zipf"
    training: bool = False

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_(self, **kw) -> "MoEShape":
        return replace(self, **kw)


# The five workloads.  Sizes, dtype and the skew intent follow the layer's
# benchmark description; the bias scales below are input recipe constants:
#  * fine_grained: sigma = 0.75 makes per-expert counts span from a handful
#    (seed 0: 7) to several hundred tokens (median 163, a few above 1000), so
#    many groups are a single padded tile (MoonEP benchmark shapes, section
#    05, use the same H=7168, K=8, H'=2048 geometry).
#  * skewed_zipf: b_e = -tau * 1.2 * ln(rank_e), a Zipf(s=1.2) popularity
#    profile over a seeded random expert ranking (MoonEP maxvio, section 01).
WORKLOADS = {
    "tiny_fp32": MoEShape("tiny_fp32", N=256, H=128, E=4, K=2, F=256, dtype="f32"),
    "mixtral": MoEShape("mixtral", N=4096, H=4096, E=8, K=2, F=14336),
    "fine_grained": MoEShape("fine_grained", N=8192, H=7168, E=256, K=8, F=2048,
                             skew="normal", skew_param=0.75),
    "skewed_zipf": MoEShape("skewed_zipf", N=16384, H=2048, E=64, K=6, F=1408,
                            skew="zipf", skew_param=1.0),
    "train_step": MoEShape("train_step", N=16384, H=4096, E=64, K=4, F=2048,
                           training=True),
}
WORKLOAD_ORDER = ["tiny_fp32", "mixtral", "fine_grained", "skewed_zipf", "train_step"]


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal(shape, std, gen, device, dtype, chunk_dim0=False) -> torch.Tensor:
    """N(0, std^2) draws, materialised in float32 then cast once to dtype.

    With chunk_dim0 the leading dimension is drawn slice by slice from the same
    generator so that a multi-GB weight never needs a float32 twin in memory.
    """
    if not chunk_dim0:
        t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
        return t.mul_(std).to(dtype)
    out = torch.empty(shape, device=device, dtype=dtype)
    for i in range(shape[0]):
        t = torch.randn(shape[1:], generator=gen, device=device, dtype=torch.float32)
        out[i].copy_(t.mul_(std))
    return out


def expert_bias(shape: MoEShape, seed: int = 0) -> Optional[torch.Tensor]:
    """Per-expert logit offsets b[E] (float64, CPU) for the skewed workloads."""
    if shape.skew is None:
        return None
    g = _gen(seed + 6, "cpu")
    if shape.skew == "normal":
        return torch.randn(shape.E, generator=g, dtype=torch.float64) * shape.skew_param
    if shape.skew == "zipf":
        rank = torch.randperm(shape.E, generator=g) + 1          # 1..E, seeded
        return -shape.skew_param * 1.2 * torch.log(rank.to(torch.float64))
    raise ValueError(f"unknown skew {shape.skew!r}")


def token_rows(shape: MoEShape, n: int, gen: torch.Generator, device) -> torch.Tensor:
    """n fresh token rows x ~ N(0,1); column 0 pinned to 1 for skewed workloads."""
    x = _normal((n, shape.H), 1.0, gen, device, shape.torch_dtype)
    if shape.skew is not None and n > 0:
        x[:, 0] = 1.0
    return x


def make_router(shape: MoEShape, seed: int = 0, device="cpu") -> torch.Tensor:
    W_r = _normal((shape.H, shape.E), 0.02, _gen(seed + 1, device), device, shape.torch_dtype)
    b = expert_bias(shape, seed)
    if b is not None:
        W_r[0, :] = b.to(device=device, dtype=shape.torch_dtype)
    return W_r


def make_inputs(shape: MoEShape, seed: int = 0, device="cpu", with_dy: Optional[bool] = None,
                weights: bool = True) -> dict:
    """All layer inputs for one workload, deterministic in (shape, seed, device).

    Returns a dict with x, W_r, W1, W3, W2 (and dy when training or requested).
    """
    if with_dy is None:
        with_dy = shape.training
    dt = shape.torch_dtype
    big = shape.E * shape.H * shape.F > (1 << 26)
    out = {
        "x": token_rows(shape, shape.N, _gen(seed, device), device),
        "W_r": make_router(shape, seed, device),
    }
    if weights:
        out["W1"] = _normal((shape.E, shape.H, shape.F), 1.0 / math.sqrt(shape.H),
                            _gen(seed + 2, device), device, dt, chunk_dim0=big)
        out["W3"] = _normal((shape.E, shape.H, shape.F), 1.0 / math.sqrt(shape.H),
                            _gen(seed + 3, device), device, dt, chunk_dim0=big)
        out["W2"] = _normal((shape.E, shape.F, shape.H), 1.0 / math.sqrt(shape.F),
                            _gen(seed + 4, device), device, dt, chunk_dim0=big)
    if with_dy:
        out["dy"] = _normal((shape.N, shape.H), 1.0, _gen(seed + 5, device), device, dt)
    return out


def resample_rows(shape: MoEShape, x: torch.Tensor, rows, seed: int, round_: int) -> None:
    """Redraw the token rows `rows` of x in place from the resampling stream."""
    rows = torch.as_tensor(rows, dtype=torch.long)
    if rows.numel() == 0:
        return
    g = _gen(seed + 7 + 1000 * (round_ + 1), x.device)
    x[rows.to(x.device)] = token_rows(shape, int(rows.numel()), g, x.device)


def random_counts(E: int, total: int, seed: int, zero_frac: float = 0.0) -> torch.Tensor:
    """Random per-expert row counts summing to `total` (for grouped-GEMM cases).

    A seeded fraction of experts gets no rows at all, so that empty groups occur.
    """
    g = _gen(seed + 11, "cpu")
    w = torch.rand(E, generator=g, dtype=torch.float64) + 0.05
    if zero_frac > 0:
        w[torch.rand(E, generator=g, dtype=torch.float64) < zero_frac] = 0.0
    if w.sum() == 0:
        w[0] = 1.0
    c = torch.floor(w / w.sum() * total).to(torch.long)
    c[int(torch.argmax(w))] += total - int(c.sum())
    return c
