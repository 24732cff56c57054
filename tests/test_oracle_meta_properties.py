"""Property sweep of the oracle's dispatch metadata (MegaBlocks - architecture,
sec. 2.1 and 2.3; the token-dropping variant of "MoE computation principle and
execution", sec. 3.4) over random shapes, expert ids and capacities.

The expected values come from numpy's stable argsort and searchsorted: an
assignment's rank inside its expert is its position among that expert's flat
ids in increasing order, and with a capacity C an expert keeps ranks < C.
Nothing here restates the oracle's counting loop."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import moe_oracle as om


@st.composite
def routing(draw):
    E = draw(st.integers(1, 40))
    K = draw(st.integers(1, min(E, 6)))
    N = draw(st.integers(0, 300))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    skew = draw(st.booleans())
    rng = np.random.default_rng(seed)
    if skew:     # a few experts take most tokens: many empty experts
        p = rng.dirichlet(np.full(E, 0.2))
        rows = [rng.choice(E, K, replace=False, p=p if np.count_nonzero(p) >= K else None) for _ in range(N)]
    else:
        rows = [rng.permutation(E)[:K] for _ in range(N)]
    te = np.asarray(rows, dtype=np.int32).reshape(N, K)
    capacity = draw(st.sampled_from([0, 1, 2, 5, 17, 10 ** 6]))
    return te, E, K, N, capacity


@settings(max_examples=80, deadline=None)
@given(routing())
def test_dispatch_meta_matches_sort_primitives(case):
    te, E, K, N, capacity = case
    flat = te.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")
    sorted_e = flat[order]
    rank = np.empty(flat.size, dtype=np.int64)
    rank[order] = np.arange(flat.size) - np.searchsorted(sorted_e, sorted_e, side="left")
    kept = rank < capacity if capacity > 0 else np.ones(flat.size, dtype=bool)

    m = om.dispatch_meta(te, E, capacity=capacity)
    hist = np.bincount(flat[kept], minlength=E)
    np.testing.assert_array_equal(m["hist"], hist)
    np.testing.assert_array_equal(m["bins"], np.cumsum(hist))
    padded = -(-hist // 128) * 128
    np.testing.assert_array_equal(m["padded_bins"], np.cumsum(padded))
    np.testing.assert_array_equal(m["indices"], order[kept[order]])
    np.testing.assert_array_equal(m["bin_ids"], sorted_e[kept[order]])
    pstart = np.cumsum(padded) - padded
    expect_pos = np.where(kept, pstart[flat] + rank, -1)
    np.testing.assert_array_equal(m["pos"], expect_pos)
    # the static bound of the padded rows holds for every routing
    assert int(m["padded_bins"][-1]) <= om.padded_rows_max(N, E, K)
    # the kept mask is the same selection
    np.testing.assert_array_equal(om.kept_mask(te, E, capacity).reshape(-1), kept)


@settings(max_examples=60, deadline=None)
@given(routing(), st.integers(1, 5))
def test_permute_then_combine_with_identity_experts(case, H):
    """With every expert the identity, combine(permute(x)) gives each token
    x_t times the sum of its kept routing weights: the whole of x_t when
    nothing is dropped (the weights sum to 1), less when assignments are
    dropped; pad rows and dropped assignments carry nothing."""
    te, E, K, N, capacity = case
    rng = np.random.default_rng(N * 31 + E)
    x = rng.standard_normal((N, H))
    w = rng.random((N, K)) + 0.1
    w = w / w.sum(axis=1, keepdims=True)
    m = om.dispatch_meta(te, E, capacity=capacity)
    P = om.padded_rows_max(N, E, K)
    xp = om.permute(x, m["pos"], K, P)
    kept = om.kept_mask(te, E, capacity)
    # every gathered row is its token's row; pad rows are zero
    used = np.zeros(P, dtype=bool)
    pos = m["pos"].reshape(N, K)
    used[pos[kept]] = True
    assert not np.any(xp[~used])
    y = om.combine(xp, w, m["pos"], N, K)
    np.testing.assert_allclose(y, x * (w * kept).sum(axis=1, keepdims=True), rtol=1e-12, atol=1e-12)
