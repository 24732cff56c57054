"""CPU oracle for the dropless top-k MoE layer (test infrastructure only).

Plain, slow and written to be checked by eye against the pages.  Everything
is float64 numpy; inputs given in bf16 or fp32 are widened exactly first.
Only tests, the smoke check and the benchmark's CPU-baseline leg use this
module; the library never does.

Sources (page title, section):
  * "MoE computation principle and execution" (icman), sec. 2.1 router
    logits = x W_r and softmax over experts; sec. 2.2 top-K of the softmax
    probabilities followed by renormalisation of the K kept values; sec. 2.3
    SwiGLU expert and output y = sum_i gate_i * expert_i(x).
  * "MegaBlocks - architecture" (ai-reference-codex), sec. 2.1/2.3: dispatch
    metadata = sort by expert, histogram, cumsum, round up to 128, cumsum;
    padded gather; scatter that multiplies by the routing weight and sums
    over the top-k; sec. 4: radix sort over ceil(log2 E) key bits, and the
    gather/scatter duality used by the backward pass.
  * "LLaMA MoE tutorial" (intelliparadigm), sec. 2.1 FeedForward
    w2(silu(w1 x) * w3 x); sec. 2.3 the per-expert loop that finds the
    (token, slot) pairs of each expert and index-adds weighted outputs.
  * MoonEP article (aikraft), sec. 01: maxvio = max_e(T_e / T_mean) - 1.

Readings where the pages are silent (each is listed in the design notes):
  * top-K order: descending probability; equal values go to the lower
    expert id (the pages only warn that library top-k may be unordered).
  * bins and padded_bins are inclusive cumulative sums; an expert with no
    tokens keeps zero padded rows; pad rows are zero.
  * the renormalisation clamp 1e-6 of the MoK demo never fires (the kept sum
    is at least K/E) and is omitted.
  * the backward pass is the chain rule of the forward definition; the
    router receives gradient only through the kept, renormalised weights
    (sec. 2.2 of the icman page).
"""
from __future__ import annotations

import numpy as np

TILE = 128   # MegaBlocks pads each expert's group to a multiple of 128 rows


def f64(a) -> np.ndarray:
    """Exact widening of a torch tensor (any float dtype) or array to float64."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            return a.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------- routing ---

def router_logits(x, W_r) -> np.ndarray:
    """logits[N, E] = x[N, H] @ W_r[H, E] (icman sec. 2.1)."""
    return f64(x) @ f64(W_r)


def softmax(logits) -> np.ndarray:
    """Row softmax over experts, max-subtracted (icman sec. 2.1)."""
    l = np.asarray(logits, dtype=np.float64)
    z = np.exp(l - l.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def top_k(probs, K: int):
    """K largest entries per row by repeated arg-max (icman sec. 2.2).

    Each pass takes the row's arg-max over the experts not yet taken; arg-max
    returns the first (lowest-id) position among equal maxima, so equal values
    resolve to the lower id.  Returns (values[N, K], ids[N, K] int32) in
    descending order.
    """
    p = np.array(probs, dtype=np.float64, copy=True)
    N, E = p.shape
    ids = np.zeros((N, K), dtype=np.int32)
    vals = np.zeros((N, K), dtype=np.float64)
    rows = np.arange(N)
    for k in range(K):
        best = np.argmax(p, axis=1)
        ids[:, k] = best
        vals[:, k] = p[rows, best]
        p[rows, best] = -np.inf
    return vals, ids


def renormalise(vals) -> np.ndarray:
    """Kept probabilities divided by their sum, so each row sums to 1 (sec. 2.2)."""
    v = np.asarray(vals, dtype=np.float64)
    return v / v.sum(axis=-1, keepdims=True)


def route(x, W_r, K: int) -> dict:
    """Router: logits, softmax, top-K, renormalisation (icman sec. 2.1-2.2)."""
    logits = router_logits(x, W_r)
    probs = softmax(logits)
    vals, ids = top_k(probs, K)
    return {"logits": logits, "probs": probs, "top_experts": ids,
            "weights": renormalise(vals)}


def route_from_logits(logits, K: int) -> dict:
    probs = softmax(logits)
    vals, ids = top_k(probs, K)
    return {"logits": np.asarray(logits, np.float64), "probs": probs,
            "top_experts": ids, "weights": renormalise(vals)}


def topk_gaps(logits, K: int) -> np.ndarray:
    """Smallest gap between consecutive entries among each row's K+1 largest
    logits (only the K ordered choices when K == E); used to keep generated
    inputs away from near-ties so that the selected set and its order do not
    depend on rounding."""
    l = -np.sort(-np.asarray(logits, np.float64), axis=-1)
    m = min(K + 1, l.shape[1])
    if m < 2:
        return np.full(l.shape[0], np.inf)
    return (l[:, :m - 1] - l[:, 1:m]).min(axis=-1)


def repair_logit_gaps(x, W_r, K: int, resample, min_gap: float = 1e-3, max_rounds: int = 50):
    """Redraw token rows whose top-K+1 logits are closer than min_gap.

    `resample(rows, round)` must overwrite those rows of x in place (the input
    generator supplies it).  Returns the number of rounds used.
    """
    for r in range(max_rounds):
        bad = np.nonzero(topk_gaps(router_logits(x, W_r), K) < min_gap)[0]
        if bad.size == 0:
            return r
        resample(bad, r)
    raise RuntimeError("logit-gap repair did not converge")


# ------------------------------------------------------ dispatch metadata ---

def round_up(n, m: int = TILE):
    return ((np.asarray(n, dtype=np.int64) + m - 1) // m) * m


def capacity_from_factor(N: int, E: int, capacity_factor: float, K: int = 1) -> int:
    """Per-expert capacity ceil(N*K / E * capacity_factor) (icman sec. 3.4
    writes ceil(N / E * cf) and says cf = 1 is the perfectly uniform case,
    which holds for top-K routing only when N counts the N*K assignments)."""
    import math
    return int(math.ceil(N * K / E * capacity_factor))


def kept_mask(top_experts, E: int, capacity: int) -> np.ndarray:
    """Token-dropping variant: each expert keeps its first `capacity`
    assignments in increasing flat id t*K + k and drops the rest
    (capacity 0 = dropless, everything kept)."""
    te = np.asarray(top_experts)
    flat = te.reshape(-1)
    keep = np.ones(flat.size, dtype=bool)
    if capacity > 0:
        seen = np.zeros(E, dtype=np.int64)
        for i, e in enumerate(flat):
            if seen[e] >= capacity:
                keep[i] = False
            seen[e] += 1
    return keep.reshape(te.shape)


def dispatch_meta(top_experts, E: int, capacity: int = 0) -> dict:
    """Sort / histogram / cumsum / round-up / cumsum (MegaBlocks sec. 2.1, 2.3).

    Flat assignment id i = t*K + k.  The sort is a counting sort that visits i
    in increasing order, so it is stable.  With capacity > 0 only the kept
    assignments (kept_mask) are counted and placed; dropped ones get pos -1.
      hist[e]        number of assignments to expert e
      bins[e]        inclusive cumsum of hist
      padded_bins[e] inclusive cumsum of round_up(hist, 128)
      indices[j]     flat id at sorted position j
      bin_ids[j]     expert of indices[j]
      pos[i]         padded row of assignment i
    """
    keep = kept_mask(top_experts, E, capacity).reshape(-1)
    te = np.asarray(top_experts, dtype=np.int64).reshape(-1)
    hist = np.zeros(E, dtype=np.int64)
    for e, kp in zip(te, keep):
        if kp:
            hist[e] += 1
    bins = np.cumsum(hist)
    padded_bins = np.cumsum(round_up(hist))
    sorted_start = bins - hist
    padded_start = padded_bins - round_up(hist)
    fill = np.zeros(E, dtype=np.int64)
    n_kept = int(hist.sum())
    indices = np.zeros(n_kept, dtype=np.int64)
    bin_ids = np.zeros(n_kept, dtype=np.int64)
    pos = np.full(te.size, -1, dtype=np.int64)
    for i, e in enumerate(te):
        if not keep[i]:
            continue
        r = fill[e]
        fill[e] += 1
        indices[sorted_start[e] + r] = i
        bin_ids[sorted_start[e] + r] = e
        pos[i] = padded_start[e] + r
    i32 = lambda a: a.astype(np.int32)
    return {"hist": i32(hist), "bins": i32(bins), "padded_bins": i32(padded_bins),
            "indices": i32(indices), "bin_ids": i32(bin_ids), "pos": i32(pos)}


def padded_rows_max(N: int, E: int, K: int) -> int:
    """Static upper bound on padded rows: N*K + E*127, rounded to 128."""
    return int(round_up(N * K + E * (TILE - 1)))


def maxvio(hist, N: int, K: int, E: int) -> float:
    """max_e(T_e / T_mean) - 1 with T_mean = N*K/E (MoonEP sec. 01)."""
    return float(np.max(hist) / (N * K / E) - 1.0)


def permute(x, pos, K: int, P: int) -> np.ndarray:
    """Padded gather: row pos[t*K+k] of the result is token t; pads stay 0.
    A dropped assignment (pos -1, token dropping) is not gathered."""
    xv = f64(x)
    out = np.zeros((P, xv.shape[1]), dtype=np.float64)
    for i, p in enumerate(np.asarray(pos).reshape(-1)):
        if p >= 0:
            out[p] = xv[i // K]
    return out


# ----------------------------------------------------------- expert math ---

def silu(g):
    return g / (1.0 + np.exp(-g))


def swiglu_ffn(X, W1e, W3e, W2e):
    """w2(silu(X w1) * (X w3)) for one expert (intelliparadigm sec. 2.1)."""
    G = X @ W1e
    U = X @ W3e
    return (silu(G) * U) @ W2e


def grouped_swiglu(x_perm, W1, W3, W2, padded_bins):
    """Per-expert SwiGLU over each expert's padded row range.

    Returns (A = silu(G)*U [P, F], O = A W2_e [P, H]); rows past the last
    group stay zero.
    """
    Xp, W1, W3, W2 = f64(x_perm), f64(W1), f64(W3), f64(W2)
    P = Xp.shape[0]
    E, H, F = W1.shape
    A = np.zeros((P, F))
    O = np.zeros((P, H))
    start = 0
    for e in range(E):
        end = int(padded_bins[e])
        if end > start:
            G = Xp[start:end] @ W1[e]
            U = Xp[start:end] @ W3[e]
            A[start:end] = silu(G) * U
            O[start:end] = A[start:end] @ W2[e]
        start = end
    return A, O


def combine(O, weights, pos, N: int, K: int):
    """y[t] = sum over k of weights[t,k] * O[pos[t*K+k]] (MegaBlocks sec. 2.1);
    a dropped assignment (pos -1) adds nothing (icman sec. 3.4)."""
    Ov = np.asarray(O, np.float64)
    w = np.asarray(weights, np.float64)
    p = np.asarray(pos).reshape(N, K)
    y = np.zeros((N, Ov.shape[1]))
    for t in range(N):
        for k in range(K):
            if p[t, k] >= 0:
                y[t] += w[t, k] * Ov[p[t, k]]
    return y


def moe_forward(x, W_r, W1, W3, W2, K: int, routing: dict | None = None,
                tokens=None, capacity: int = 0) -> dict:
    """Whole layer, written as the per-expert loop of the LLaMA MoE tutorial
    (sec. 2.3): for each expert find its (token, slot) pairs, run the expert
    on those tokens and index-add the weighted outputs.

    `routing` may carry a precomputed route(); `tokens` restricts y to a subset
    of token ids (y for token t depends only on x[t] once routing is fixed).
    capacity > 0 gives the token-dropping variant: dropped (token, expert)
    pairs contribute nothing (icman sec. 3.4; kept_mask for which are kept).
    """
    r = routing if routing is not None else route(x, W_r, K)
    te, w = r["top_experts"], r["weights"]
    if capacity > 0:
        w = np.where(kept_mask(te, W1.shape[0], capacity), w, 0.0)
    xv = f64(x)
    N = xv.shape[0]
    tok = np.arange(N) if tokens is None else np.asarray(tokens, dtype=np.int64)
    W1v, W3v, W2v = W1, W3, W2
    E = W1.shape[0]
    y = np.zeros((tok.size, xv.shape[1]))
    te_s, w_s = te[tok], w[tok]
    for e in range(E):
        rows, slots = np.nonzero(te_s == e)
        if rows.size == 0:
            continue
        out = swiglu_ffn(xv[tok[rows]], f64(W1v[e]), f64(W3v[e]), f64(W2v[e]))
        np.add.at(y, rows, out * w_s[rows, slots][:, None])
    return {"y": y, "routing": r, "tokens": tok}


def dense_mixture(x, W_r, W1, W3, W2) -> np.ndarray:
    """All experts on all tokens, weighted by the full softmax (no top-k)."""
    xv = f64(x)
    p = softmax(router_logits(x, W_r))
    y = np.zeros_like(xv)
    for e in range(W1.shape[0]):
        y += p[:, e:e + 1] * swiglu_ffn(xv, f64(W1[e]), f64(W3[e]), f64(W2[e]))
    return y


# ------------------------------------------------- load-balancing loss ---

def aux_loss(probs, top_experts, alpha: float, N_total: int | None = None) -> float:
    """Switch-style auxiliary load-balancing loss (icman sec. 4.2):
    alpha * E * sum_i f_i * P_i with f_i = share of the N*K assignments routed
    to expert i and P_i = mean over tokens of the router probability of i.
    With perfectly balanced routing and uniform probabilities it equals alpha."""
    p = np.asarray(probs, np.float64)
    te = np.asarray(top_experts)
    N, E = p.shape
    K = te.shape[1]
    f = np.bincount(te.reshape(-1), minlength=E) / (N * K)
    P = p.sum(axis=0) / N
    return float(alpha * E * np.sum(f * P))


# -------------------------------------------------------------- backward ---

def moe_backward(x, W_r, W1, W3, W2, K: int, dy, routing: dict | None = None,
                 tokens=None, aux_alpha: float = 0.0, aux_grad: float = 1.0,
                 capacity: int = 0) -> dict:
    """Gradients of sum(y * dy) by the chain rule of the forward definition.

    Per token t and slot k with expert e (forward g = x W1_e, u = x W3_e,
    a = silu(g) u, o = a W2_e, y = sum_k w_k o_k):
      dw_k = <dy, o_k>;  do_k = w_k dy
      da = do_k W2_e^T;  dW2_e += a^T do_k
      dg = da * u * silu'(g);  du = da * silu(g)
      dW1_e += x^T dg;  dW3_e += x^T du;  dx += dg W1_e^T + du W3_e^T
    Router (icman sec. 2.2: gradient flows through the kept softmax weights):
      w_k = p_{e_k} / S with S = sum of kept p  ->  dp_{e_k} = dw_k/S - <dw, p_kept>/S^2
      softmax: dlogits = p * (dp - <dp, p>);  dW_r += x^T dlogits;  dx += dlogits W_r^T
    `tokens` restricts every sum to a subset of tokens (the weight gradients
    are then those of the sub-batch).
    With aux_alpha != 0 the objective also carries aux_grad * aux_loss (of the
    whole batch): the counts f_i are piecewise constant, so the extra gradient
    flows through P_i = mean_t p_t,i only: dp_t,i += aux_grad*alpha*E*f_i/N.
    """
    xv, dyv = f64(x), f64(dy)
    r = routing if routing is not None else route(x, W_r, K)
    N, H = xv.shape
    tok = np.arange(N) if tokens is None else np.asarray(tokens, dtype=np.int64)
    E, _, F = W1.shape
    W_rv = f64(W_r)
    te, w, probs = r["top_experts"][tok], r["weights"][tok], r["probs"][tok]
    kept = kept_mask(r["top_experts"], E, capacity)[tok]   # all True when dropless
    xs, dys = xv[tok], dyv[tok]
    n = tok.size
    dx = np.zeros((n, H))
    dW1 = np.zeros((E, H, F))
    dW3 = np.zeros((E, H, F))
    dW2 = np.zeros((E, F, H))
    dw = np.zeros((n, K))
    for e in range(E):
        rows, slots = np.nonzero((te == e) & kept)
        if rows.size == 0:
            continue
        W1e, W3e, W2e = f64(W1[e]), f64(W3[e]), f64(W2[e])
        X = xs[rows]
        G = X @ W1e
        U = X @ W3e
        sig = 1.0 / (1.0 + np.exp(-G))
        A = G * sig * U
        O = A @ W2e
        dw[rows, slots] = np.sum(dys[rows] * O, axis=1)
        dO = w[rows, slots][:, None] * dys[rows]
        dA = dO @ W2e.T
        dW2[e] = A.T @ dO
        dG = dA * U * sig * (1.0 + G * (1.0 - sig))
        dU = dA * G * sig
        dW1[e] = X.T @ dG
        dW3[e] = X.T @ dU
        np.add.at(dx, rows, dG @ W1e.T + dU @ W3e.T)
    # renormalisation and softmax
    p_kept = np.take_along_axis(probs, te.astype(np.int64), axis=1)
    S = p_kept.sum(axis=1, keepdims=True)
    dp_kept = dw / S - np.sum(dw * p_kept, axis=1, keepdims=True) / S ** 2
    dp = np.zeros_like(probs)
    np.put_along_axis(dp, te.astype(np.int64), dp_kept, axis=1)
    if aux_alpha != 0.0:
        f_all = np.bincount(np.asarray(r["top_experts"]).reshape(-1), minlength=E) / (N * K)
        dp = dp + aux_grad * aux_alpha * E * f_all[None, :] / N
    dlogits = probs * (dp - np.sum(dp * probs, axis=1, keepdims=True))
    dW_r = xs.T @ dlogits
    dx += dlogits @ W_rv.T
    return {"dx": dx, "dW_r": dW_r, "dW1": dW1, "dW3": dW3, "dW2": dW2,
            "dw": dw, "dlogits": dlogits, "tokens": tok}


def loss_sum(x, W_r, W1, W3, W2, K, dy, aux_alpha: float = 0.0, aux_grad: float = 1.0,
             capacity: int = 0) -> float:
    """sum(y * dy) (+ aux_grad * aux_loss) with routing recomputed; used by the
    finite-difference pins."""
    out = moe_forward(x, W_r, W1, W3, W2, K, capacity=capacity)
    v = float(np.sum(out["y"] * f64(dy)))
    if aux_alpha != 0.0:
        r = out["routing"]
        v += aux_grad * aux_loss(r["probs"], r["top_experts"], aux_alpha)
    return v
