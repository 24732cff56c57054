"""Shared helpers for the tests: seeded cases with the logit-gap repair, and
the tolerance checks the layer's parity is held to.

Tolerances: y and gradients within max|err| <= 2e-2 * max|ref| for bf16 and
<= 1e-4 * max|ref| for fp32; routing weights and probabilities are fp32
outputs and take the fp32 bar (their logits accumulate H products in fp32,
e.g. ~1.3e-5 absolute on the weights at H = 7168); every integer output
bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

from gen import MoEShape, WORKLOADS, make_inputs, resample_rows
from oracle import moe_oracle as om

TOL = {"bf16": 2e-2, "f32": 1e-4}


def scaled_err(got, ref) -> float:
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    scale = np.max(np.abs(r)) if r.size else 0.0
    if scale == 0.0:
        return float(np.max(np.abs(g))) if g.size else 0.0
    return float(np.max(np.abs(g - r)) / scale)


def assert_scaled(got, ref, dtype: str, what: str = ""):
    e = scaled_err(got, ref)
    assert e <= TOL[dtype], f"{what}: max|err|/max|ref| = {e:.3e} > {TOL[dtype]}"
    return e


def make_case(shape: MoEShape, seed: int = 0, device="cuda", with_dy=None, repair: bool = True) -> dict:
    """Inputs of `shape`, generated on `device`, with rows re-drawn until every
    token's K+1 largest oracle logits are at least 1e-3 apart."""
    inp = make_inputs(shape, seed=seed, device=device, with_dy=with_dy)
    if repair and shape.N > 0:
        x_cpu = inp["x"].cpu()
        W_r_cpu = inp["W_r"].cpu()
        changed = []

        def resample(rows, r):
            resample_rows(shape, x_cpu, rows, seed, r)
            changed.append(np.asarray(rows))

        om.repair_logit_gaps(x_cpu, W_r_cpu, shape.K, resample)
        if changed:
            rows = torch.as_tensor(np.unique(np.concatenate(changed)), dtype=torch.long)
            inp["x"][rows.to(inp["x"].device)] = x_cpu[rows].to(inp["x"].device)
        inp["x_cpu"] = x_cpu
        inp["W_r_cpu"] = W_r_cpu
    return inp


def small_shape(name="s", N=300, H=128, E=8, K=2, F=256, dtype="bf16", skew=None, skew_param=0.0,
                training=False) -> MoEShape:
    return MoEShape(name, N=N, H=H, E=E, K=K, F=F, dtype=dtype, skew=skew, skew_param=skew_param,
                    training=training)
