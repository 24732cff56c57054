"""Shared helpers for the tests: seeded cases with the logit-gap repair, and
the tolerance checks the layer's parity is held to.

Tolerances: y and gradients within max|err| <= 2e-2 * max|ref| for bf16 and
<= 1e-4 * max|ref| for fp32; every integer output bit-exact.  Router logits,
probabilities and routing weights are fp32 outputs whose error comes from the
fp32 sum of H products (a bf16 x bf16 product is exact in fp32, so only the
summation rounds): routing_tol bounds it as a multiple of sqrt(H) rounding
steps of the running sum scaled by the logits' RMS (about 4e-5 on the
weights at H = 7168, 3e-6 at H = 128).
"""
from __future__ import annotations

import math

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


ROUND32 = 2.0 ** -24   # unit roundoff of fp32


def routing_tol(H: int, logit_rms: float) -> float:
    """Bound on the absolute error of a router logit.  The GPU sums H products
    in fp32 (exact for bf16 operands) in its own order, tensor-core k steps
    and H slices included.  Each addition rounds at the magnitude of the
    running sum, of the order of the logits' RMS, and with terms of random
    sign those roundings add like a random walk: about sqrt(H/2) * u * RMS
    for one logit, about 3.5 * sqrt(H) * u * RMS for the largest of a
    million.  The factor 8 leaves twice that.  The softmax and the
    renormalisation move a weight or a probability by at most half the
    largest logit error (p(1-p) <= 1/4 twice), so weights and probabilities
    take routing_tol / 2."""
    return 8.0 * math.sqrt(H) * ROUND32 * max(1.0, logit_rms)


def assert_routing(got, ref, H: int, logits_ref, what: str, half: bool = True):
    """Absolute check of a routing output (weights or probabilities when
    `half`, logits otherwise) against the bound of routing_tol."""
    g = got.detach().to("cpu", torch.float64).numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    r = np.asarray(ref, np.float64)
    assert g.shape == r.shape, (g.shape, r.shape)
    lr = np.asarray(logits_ref, np.float64)
    tol = routing_tol(H, float(np.sqrt(np.mean(lr * lr))) if lr.size else 1.0)
    if half:
        tol *= 0.5
    e = float(np.max(np.abs(g - r))) if r.size else 0.0
    assert e <= tol, f"{what}: max|err| = {e:.3e} > {tol:.3e} (H = {H})"
    return e, tol


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
