"""Pins for the CPU oracle: each check ties it to something other than itself
(library routines, closed forms, invariants, brute force, finite differences).
"""
import math
import os

import numpy as np
import pytest
import torch

from gen import WORKLOADS, make_inputs, resample_rows, MoEShape
from oracle import moe_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(N=48, H=16, E=4, K=2, F=24, seed=0, dtype="f32", skew=None, skew_param=0.0):
    shp = MoEShape("pin", N=N, H=H, E=E, K=K, F=F, dtype=dtype, skew=skew, skew_param=skew_param)
    inp = make_inputs(shp, seed=seed, with_dy=True)
    om.repair_logit_gaps(inp["x"], inp["W_r"], K,
                         lambda rows, r: resample_rows(shp, inp["x"], rows, seed, r))
    return shp, inp


# ------------------------------------------------------------- routing pins

def test_softmax_closed_form():
    p = om.softmax(np.array([[0.0, math.log(2.0), math.log(3.0)]]))
    np.testing.assert_allclose(p, [[1 / 6, 2 / 6, 3 / 6]], rtol=0, atol=1e-15)
    # shift invariance
    np.testing.assert_allclose(om.softmax(np.array([[1000.0, 1000.0 + math.log(3.0)]])),
                               [[0.25, 0.75]], atol=1e-15)


def test_topk_matches_torch_topk():
    g = torch.Generator().manual_seed(3)
    probs = torch.rand(200, 16, generator=g, dtype=torch.float64)
    vals, ids = om.top_k(probs.numpy(), 5)
    tv, ti = torch.topk(probs, 5, dim=-1, largest=True, sorted=True)
    np.testing.assert_array_equal(ids, ti.numpy())
    np.testing.assert_array_equal(vals, tv.numpy())


def test_topk_ties_go_to_lowest_id():
    vals, ids = om.top_k(np.array([[0.25, 0.25, 0.25, 0.25],
                                   [0.1, 0.3, 0.3, 0.3],
                                   [0.4, 0.1, 0.4, 0.1]]), 2)
    np.testing.assert_array_equal(ids, [[0, 1], [1, 2], [0, 2]])


def test_renormalised_weights_equal_softmax_over_kept_logits():
    """LLaMA MoE tutorial sec. 2.3 takes top-k of the logits first and a softmax
    over the K kept logits; that ordering must give the same experts and weights."""
    g = torch.Generator().manual_seed(5)
    logits = torch.randn(300, 8, generator=g, dtype=torch.float64) * 2
    r = om.route_from_logits(logits.numpy(), 3)
    tv, ti = torch.topk(logits, 3, dim=-1)
    w = torch.softmax(tv, dim=-1)
    np.testing.assert_array_equal(r["top_experts"], ti.numpy())
    np.testing.assert_allclose(r["weights"], w.numpy(), rtol=0, atol=1e-14)
    np.testing.assert_allclose(r["weights"].sum(1), 1.0, atol=1e-14)


def test_router_logits_match_library_matmul():
    _, inp = small()
    ref = torch.matmul(inp["x"].double(), inp["W_r"].double()).numpy()
    np.testing.assert_allclose(om.router_logits(inp["x"], inp["W_r"]), ref, rtol=1e-13, atol=1e-15)


def test_topk_gaps_match_brute_force():
    """Smallest gap among each row's K+1 largest logits (K when K = E), from
    torch.topk's sorted values and a plain double loop."""
    g = torch.Generator().manual_seed(9)
    for E, K in ((8, 2), (8, 8), (5, 1), (64, 6)):
        logits = torch.randn(50, E, generator=g, dtype=torch.float64)
        got = om.topk_gaps(logits.numpy(), K)
        m = min(K + 1, E)
        vals = torch.topk(logits, m, dim=-1, sorted=True).values.numpy()
        for t in range(50):
            want = min((vals[t, j] - vals[t, j + 1] for j in range(m - 1)), default=math.inf)
            assert got[t] == want


def test_gap_repair_enforces_margin():
    shp, inp = small(N=512, E=8, K=2, H=32)
    gaps = om.topk_gaps(om.router_logits(inp["x"], inp["W_r"]), 2)
    assert gaps.min() >= 1e-3


# ------------------------------------------------------------ metadata pins

def test_meta_golden_megablocks_counts():
    rows = {}
    with open(os.path.join(GOLDEN, "megablocks_counts.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            k, *v = line.split()
            rows[k] = [int(a) for a in v]
    hist = rows["hist"]
    te = np.concatenate([np.full(c, e) for e, c in enumerate(hist)])
    np.random.default_rng(0).shuffle(te)
    m = om.dispatch_meta(te.reshape(-1, 1), len(hist))
    np.testing.assert_array_equal(m["hist"], hist)
    np.testing.assert_array_equal(m["bins"], rows["bins"])
    np.testing.assert_array_equal(m["padded_bins"], rows["padded_bins"])


@pytest.mark.parametrize("E,K,N", [(4, 2, 256), (8, 2, 1000), (64, 6, 777), (256, 8, 300), (1, 1, 50)])
def test_meta_invariants_and_stable_sort(E, K, N):
    rng = np.random.default_rng(E * 1000 + K)
    te = np.stack([rng.permutation(E)[:K] for _ in range(N)]).astype(np.int32)
    m = om.dispatch_meta(te, E)
    flat = te.reshape(-1)
    assert m["hist"].sum() == N * K
    np.testing.assert_array_equal(m["hist"], np.bincount(flat, minlength=E))
    # library stable sort gives the same permutation
    np.testing.assert_array_equal(m["indices"], np.argsort(flat, kind="stable"))
    np.testing.assert_array_equal(m["bin_ids"], flat[m["indices"]])
    np.testing.assert_array_equal(m["bins"], np.cumsum(np.bincount(flat, minlength=E)))
    pb = np.concatenate([[0], m["padded_bins"]])
    d = np.diff(pb)
    assert np.all(d % 128 == 0) and np.all(d >= m["hist"]) and np.all(d - m["hist"] < 128)
    assert np.all((d == 0) == (m["hist"] == 0))
    # pos: unique, inside the owning expert's padded range, in sorted order
    pos = m["pos"]
    assert len(np.unique(pos)) == N * K
    for e in range(E):
        ids = np.nonzero(flat == e)[0]
        np.testing.assert_array_equal(pos[ids], pb[e] + np.arange(ids.size))
    assert pos.max(initial=-1) < om.padded_rows_max(N, E, K)


def test_maxvio_recomputed_from_counts():
    # uniform routing: maxvio 0; everything on K experts: E/K - 1
    N, E, K = 64, 8, 2
    te = np.stack([[(2 * t) % E, (2 * t + 1) % E] for t in range(N)])
    h = om.dispatch_meta(te, E)["hist"]
    assert om.maxvio(h, N, K, E) == 0.0
    te2 = np.tile([[3, 5]], (N, 1))
    h2 = om.dispatch_meta(te2, E)["hist"]
    assert om.maxvio(h2, N, K, E) == pytest.approx(E / K - 1)


def test_permute_then_combine_with_identity_experts_returns_x():
    """With O = x_perm (identity experts) the weighted K-sum returns x, since
    the renormalised weights sum to one: checks pos, permute and combine."""
    shp, inp = small(N=200, E=8, K=3, H=16)
    r = om.route(inp["x"], inp["W_r"], 3)
    m = om.dispatch_meta(r["top_experts"], 8)
    P = om.padded_rows_max(200, 8, 3)
    xp = om.permute(inp["x"], m["pos"], 3, P)
    y = om.combine(xp, r["weights"], m["pos"], 200, 3)
    np.testing.assert_allclose(y, om.f64(inp["x"]), rtol=0, atol=1e-13)
    # pad rows are zero
    used = np.zeros(P, bool)
    used[m["pos"]] = True
    assert np.all(xp[~used] == 0)


# ---------------------------------------------------------- expert-math pins

def test_single_expert_is_plain_swiglu_ffn():
    """E=1, K=1 reduces to one dense SwiGLU FFN, written with torch's own
    linear and silu (LLaMA MoE tutorial sec. 2.1)."""
    shp, inp = small(N=40, E=1, K=1, H=16, F=24)
    y = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 1)["y"]
    x = inp["x"].double()
    w1 = inp["W1"][0].double().T
    w3 = inp["W3"][0].double().T
    w2 = inp["W2"][0].double().T
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(x, w1)) * torch.nn.functional.linear(x, w3), w2)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_top_all_experts_equals_dense_softmax_mixture():
    shp, inp = small(N=64, E=4, K=4)
    y = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 4)["y"]
    yd = om.dense_mixture(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"])
    np.testing.assert_allclose(y, yd, rtol=1e-11, atol=1e-12)


def test_masked_dense_equals_sparse():
    """Every expert on every token, then keep only the routed (token, expert)
    pairs with their weights: same y as the sparse per-expert loop."""
    shp, inp = small(N=96, E=6, K=2)
    r = om.route(inp["x"], inp["W_r"], 2)
    y = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2, routing=r)["y"]
    x = torch.tensor(om.f64(inp["x"]))
    Wd = torch.zeros(96, 6, dtype=torch.float64)
    Wd.scatter_(1, torch.tensor(r["top_experts"], dtype=torch.long), torch.tensor(r["weights"]))
    ref = torch.zeros_like(x)
    for e in range(6):
        g = x @ inp["W1"][e].double()
        u = x @ inp["W3"][e].double()
        ref += Wd[:, e:e + 1] * ((torch.nn.functional.silu(g) * u) @ inp["W2"][e].double())
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-11, atol=1e-12)


def test_grouped_stages_compose_to_layer():
    """route -> meta -> permute -> grouped SwiGLU -> combine equals the
    per-expert loop form of the whole layer."""
    shp, inp = small(N=150, E=5, K=2, H=16, F=32)
    r = om.route(inp["x"], inp["W_r"], 2)
    m = om.dispatch_meta(r["top_experts"], 5)
    P = om.padded_rows_max(150, 5, 2)
    xp = om.permute(inp["x"], m["pos"], 2, P)
    A, O = om.grouped_swiglu(xp, inp["W1"], inp["W3"], inp["W2"], m["padded_bins"])
    y = om.combine(O, r["weights"], m["pos"], 150, 2)
    y2 = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2, routing=r)["y"]
    np.testing.assert_allclose(y, y2, rtol=1e-12, atol=1e-12)
    # pad rows of the grouped outputs stay zero
    used = np.zeros(P, bool)
    used[m["pos"]] = True
    assert np.all(O[~used] == 0) and np.all(A[~used] == 0)


def test_token_subset_matches_full_layer():
    shp, inp = small(N=80, E=4, K=2)
    full = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2)
    sub = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2,
                         routing=full["routing"], tokens=[3, 17, 40, 79])
    np.testing.assert_allclose(sub["y"], full["y"][[3, 17, 40, 79]], rtol=0, atol=1e-14)


# --------------------------------------------------------------- backward pins

def _fd(fun, arr, idx, h):
    old = arr[idx]
    arr[idx] = old + h
    fp = fun()
    arr[idx] = old - h
    fm = fun()
    arr[idx] = old
    return (fp - fm) / (2 * h)


@pytest.mark.parametrize("E,K", [(4, 2), (3, 3), (1, 1)])
def test_backward_matches_central_differences(E, K):
    shp, inp = small(N=6, H=8, E=E, K=K, F=12, seed=E + 10 * K)
    P = {k: om.f64(v).copy() for k, v in inp.items()}
    # keep routing strictly stable under the perturbation
    assert om.topk_gaps(om.router_logits(P["x"], P["W_r"]), K).min() > 1e-3
    grads = om.moe_backward(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], K, P["dy"])
    f = lambda: om.loss_sum(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], K, P["dy"])
    h = 1e-6
    for name, g in (("x", "dx"), ("W_r", "dW_r"), ("W1", "dW1"), ("W3", "dW3"), ("W2", "dW2")):
        arr = P[name]
        for idx in np.ndindex(arr.shape):
            num = _fd(f, arr, idx, h)
            assert abs(num - grads[g][idx]) <= 1e-6 * (1 + abs(num)), (name, idx, num, grads[g][idx])


def test_backward_token_subset_equals_sub_batch():
    shp, inp = small(N=30, E=4, K=2)
    full = om.route(inp["x"], inp["W_r"], 2)
    sub = om.moe_backward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2, inp["dy"],
                          routing=full, tokens=np.arange(10, 20))
    ref = om.moe_backward(inp["x"][10:20], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2,
                          inp["dy"][10:20])
    for k in ("dx", "dW_r", "dW1", "dW3", "dW2"):
        np.testing.assert_allclose(sub[k], ref[k], rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------- generator recipe

def test_workloads_match_stated_shapes():
    w = WORKLOADS
    assert (w["tiny_fp32"].N, w["tiny_fp32"].H, w["tiny_fp32"].E, w["tiny_fp32"].K, w["tiny_fp32"].F) == (256, 128, 4, 2, 256)
    assert (w["mixtral"].N, w["mixtral"].H, w["mixtral"].E, w["mixtral"].K, w["mixtral"].F) == (4096, 4096, 8, 2, 14336)
    assert (w["fine_grained"].N, w["fine_grained"].H, w["fine_grained"].E, w["fine_grained"].K, w["fine_grained"].F) == (8192, 7168, 256, 8, 2048)
    assert (w["skewed_zipf"].N, w["skewed_zipf"].H, w["skewed_zipf"].E, w["skewed_zipf"].K, w["skewed_zipf"].F) == (16384, 2048, 64, 6, 1408)
    assert (w["train_step"].N, w["train_step"].H, w["train_step"].E, w["train_step"].K, w["train_step"].F) == (16384, 4096, 64, 4, 2048)


def test_generator_is_deterministic_and_skew_column():
    shp = WORKLOADS["skewed_zipf"].with_(N=64, H=32, F=16)
    a = make_inputs(shp, seed=0)
    b = make_inputs(shp, seed=0)
    for k in a:
        assert torch.equal(a[k], b[k])
    assert torch.all(a["x"][:, 0] == 1)


# ----------------------------------------------------- load-balancing loss

def test_aux_loss_closed_forms():
    N, E, K = 64, 8, 2
    probs = np.full((N, E), 1.0 / E)
    te = np.stack([[(2 * t) % E, (2 * t + 1) % E] for t in range(N)])
    assert om.aux_loss(probs, te, 0.01) == pytest.approx(0.01, rel=1e-14)   # balanced: alpha
    # everything on experts 0 and 1 with certainty-like probabilities: alpha * E / 2 * (P0 + P1)
    p2 = np.zeros((N, E)); p2[:, 0] = 0.6; p2[:, 1] = 0.4
    te2 = np.tile([[0, 1]], (N, 1))
    assert om.aux_loss(p2, te2, 0.1) == pytest.approx(0.1 * E * (0.5 * 0.6 + 0.5 * 0.4), rel=1e-14)


@pytest.mark.parametrize("E,K", [(4, 2), (6, 3)])
def test_backward_with_aux_loss_matches_central_differences(E, K):
    shp, inp = small(N=7, H=8, E=E, K=K, F=12, seed=40 + E)
    P = {k: om.f64(v).copy() for k, v in inp.items()}
    alpha, g = 0.37, 1.7
    grads = om.moe_backward(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], K, P["dy"],
                            aux_alpha=alpha, aux_grad=g)
    f = lambda: om.loss_sum(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], K, P["dy"], alpha, g)
    for name, gk in (("x", "dx"), ("W_r", "dW_r")):
        arr = P[name]
        for idx in np.ndindex(arr.shape):
            num = _fd(f, arr, idx, 1e-6)
            assert abs(num - grads[gk][idx]) <= 1e-6 * (1 + abs(num)), (name, idx, num, grads[gk][idx])


# ------------------------------------------------------ token-dropping variant

def test_capacity_large_enough_equals_dropless():
    shp, inp = small(N=60, E=4, K=2)
    a = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2)["y"]
    b = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2, capacity=10 ** 6)["y"]
    np.testing.assert_array_equal(a, b)


def test_capacity_keeps_first_assignments_brute_force():
    te = np.array([[0, 1], [1, 0], [0, 2], [2, 0], [1, 2]])
    # expert 0 sees flat ids 0, 3, 4, 7; expert 1: 1, 2, 8; expert 2: 5, 6, 9
    keep = om.kept_mask(te, 3, 2)
    np.testing.assert_array_equal(keep, [[1, 1], [1, 1], [0, 1], [1, 0], [0, 0]])
    m = om.dispatch_meta(te, 3, capacity=2)
    np.testing.assert_array_equal(m["hist"], [2, 2, 2])
    np.testing.assert_array_equal(m["indices"], [0, 3, 1, 2, 5, 6])
    np.testing.assert_array_equal(m["pos"], [0, 128, 129, 1, -1, 256, 257, -1, -1, -1])
    assert om.capacity_from_factor(1000, 8, 1.25) == 157     # ceil(1000 / 8 * 1.25)
    assert om.capacity_from_factor(1000, 8, 1.0, K=2) == 250  # balanced top-2 load per expert


def test_capacity_layer_equals_masked_sum():
    """With dropping, y is the per-expert loop restricted to kept pairs."""
    shp, inp = small(N=90, E=4, K=2)
    r = om.route(inp["x"], inp["W_r"], 2)
    cap = 30
    y = om.moe_forward(inp["x"], inp["W_r"], inp["W1"], inp["W3"], inp["W2"], 2, routing=r, capacity=cap)["y"]
    keep = om.kept_mask(r["top_experts"], 4, cap)
    x = om.f64(inp["x"])
    ref = np.zeros_like(x)
    for t in range(90):
        for k in range(2):
            if keep[t, k]:
                e = r["top_experts"][t, k]
                ref[t] += r["weights"][t, k] * om.swiglu_ffn(x[t:t + 1], om.f64(inp["W1"][e]),
                                                             om.f64(inp["W3"][e]), om.f64(inp["W2"][e]))[0]
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-13)


def test_backward_with_capacity_matches_central_differences():
    shp, inp = small(N=8, H=8, E=3, K=2, F=12, seed=77)
    P = {k: om.f64(v).copy() for k, v in inp.items()}
    cap = 4       # 16 assignments over 3 experts: some experts overflow
    r = om.route(P["x"], P["W_r"], 2)
    assert not om.kept_mask(r["top_experts"], 3, cap).all()
    grads = om.moe_backward(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], 2, P["dy"], capacity=cap)
    f = lambda: om.loss_sum(P["x"], P["W_r"], P["W1"], P["W3"], P["W2"], 2, P["dy"], capacity=cap)
    for name, gk in (("x", "dx"), ("W_r", "dW_r"), ("W1", "dW1"), ("W2", "dW2")):
        arr = P[name]
        for idx in list(np.ndindex(arr.shape))[::3]:
            num = _fd(f, arr, idx, 1e-6)
            assert abs(num - grads[gk][idx]) <= 1e-6 * (1 + abs(num)), (name, idx, num, grads[gk][idx])
