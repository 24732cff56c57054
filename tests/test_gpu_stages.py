"""Per-stage parity of the CUDA path against the CPU oracle (GPU only).

Every call goes through the C ABI (libmoe_b200.so) via the thin binding.
Integer outputs are compared bit for bit; floating-point outputs within the
tolerances of tests/_cases.py.
"""
import numpy as np
import pytest
import torch

import dropless_top_moe_b200 as moe
from gen import WORKLOADS, random_counts, MoEShape
from oracle import moe_oracle as om
from tests._cases import TOL, assert_routing, assert_scaled, make_case, scaled_err, small_shape

pytestmark = pytest.mark.gpu

ROUTE_SHAPES = [
    small_shape("r_f32", N=256, H=128, E=4, K=2, dtype="f32"),
    small_shape("r_bf16_e8", N=777, H=256, E=8, K=2),
    small_shape("r_bf16_e16", N=300, H=256, E=16, K=4),
    small_shape("r_bf16_e64", N=1000, H=512, E=64, K=6),
    small_shape("r_bf16_e256", N=515, H=384, E=256, K=8, skew="normal", skew_param=1.0),
    small_shape("r_bf16_e64_k1", N=260, H=128, E=64, K=1),
    small_shape("r_f32_k_eq_e", N=130, H=64, E=4, K=4, dtype="f32"),
    small_shape("r_bf16_zipf", N=640, H=256, E=64, K=6, skew="zipf", skew_param=1.0),
    small_shape("r_bf16_e4", N=300, H=128, E=4, K=2),
    small_shape("r_bf16_e100", N=333, H=256, E=100, K=5),
    # few row tiles and a long H: the router splits H over a cluster of S CTAs
    # (S = 8, 4 and 2 here) and sums the partial logits in slice order
    small_shape("r_split8_e8", N=300, H=2048, E=8, K=2),
    small_shape("r_split8_e64", N=1000, H=4096, E=64, K=6),
    small_shape("r_split4_e256", N=700, H=1024, E=256, K=8, skew="normal", skew_param=1.0),
    small_shape("r_split2_e40_k12", N=6000, H=1024, E=40, K=12),
    # the largest top-K lists (K up to 32), merged over 2 (S = 1), 8 (S = 4)
    # and 16 (S = 8) threads per row
    small_shape("r_bf16_e64_k32", N=500, H=256, E=64, K=32),
    small_shape("r_split4_e256_k20", N=600, H=1024, E=256, K=20, skew="normal", skew_param=1.0),
    small_shape("r_split8_e64_k32", N=300, H=4096, E=64, K=32),
]


@pytest.mark.parametrize("shape", ROUTE_SHAPES, ids=lambda s: s.name)
def test_route_matches_oracle(shape):
    c = make_case(shape, seed=1)
    r = moe.moe_route(c["x"], c["W_r"], shape.K, want_logits=True, want_probs=True)
    ref = om.route(c["x_cpu"], c["W_r_cpu"], shape.K)
    np.testing.assert_array_equal(r["top_experts"].cpu().numpy(), ref["top_experts"])
    assert_routing(r["weights"], ref["weights"], shape.H, ref["logits"], "routing weights")
    assert_routing(r["probs"], ref["probs"], shape.H, ref["logits"], "probs")
    lg = r["logits"].cpu().double().numpy()
    assert_routing(lg, ref["logits"], shape.H, ref["logits"], "logits", half=False)
    # the decision margin also holds on the GPU's own logits
    assert om.topk_gaps(lg, shape.K).min() >= 0.9e-3
    assert moe.device_status(r["ws"]) == 0


def test_route_ties_go_to_lowest_id():
    # all-zero tokens give identical logits for every expert
    for E, K, H, dt in ((8, 2, 128, torch.bfloat16), (64, 6, 256, torch.bfloat16),
                        (4, 3, 64, torch.float32), (256, 8, 128, torch.bfloat16)):
        x = torch.zeros(200, H, dtype=dt, device="cuda")
        W_r = torch.randn(H, E, device="cuda").to(dt)
        r = moe.moe_route(x, W_r, K)
        exp = np.tile(np.arange(K, dtype=np.int32), (200, 1))
        np.testing.assert_array_equal(r["top_experts"].cpu().numpy(), exp)
        np.testing.assert_allclose(r["weights"].cpu().numpy(), 1.0 / K, atol=1e-7)


def _routing(N, K, E, seed, mode="uniform"):
    g = torch.Generator().manual_seed(seed)
    if mode == "uniform":
        return torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(N)]).to(torch.int32)
    if mode == "one_expert":    # expert 3 (mod E) in every token's first slot
        te = torch.stack([torch.randperm(E, generator=g)[:K] for _ in range(N)])
        hot = 3 % E
        for t in range(N):
            row = te[t].tolist()
            if hot in row:
                row.remove(hot)
            te[t] = torch.tensor([hot] + row[:K - 1])
        return te.to(torch.int32)
    if mode == "few":           # only experts 0 and E-1 used (K = 1 or 2)
        te = torch.zeros(N, K, dtype=torch.int32)
        te[:, 0] = 0
        if K > 1:
            te[:, 1] = E - 1
        return te
    raise ValueError(mode)


META_CASES = [(256, 2, 4, "uniform"), (4096, 2, 8, "uniform"), (8192, 8, 256, "uniform"),
              (16384, 6, 64, "one_expert"), (1000, 1, 64, "few"), (333, 2, 256, "few"),
              (50, 1, 1, "uniform"), (2049, 3, 5, "uniform"), (1, 1, 3, "uniform")]


@pytest.mark.parametrize("N,K,E,mode", META_CASES)
def test_dispatch_meta_bit_exact(N, K, E, mode):
    te = _routing(N, K, E, seed=N + E, mode=mode)
    m = moe.moe_dispatch_meta(te.cuda(), E)
    ref = om.dispatch_meta(te.numpy(), E)
    for k in ("indices", "bin_ids", "bins", "padded_bins", "pos"):
        np.testing.assert_array_equal(m[k].cpu().numpy(), ref[k], err_msg=k)
    assert moe.device_status(m["ws"]) == 0


def test_dispatch_meta_flags_bad_expert_ids():
    te = _routing(100, 2, 8, seed=5)
    te[7, 1] = 8
    te[50, 0] = -1
    m = moe.moe_dispatch_meta(te.cuda(), 8)
    assert moe.device_status(m["ws"]) & 1
    pos = m["pos"].cpu().numpy()
    assert pos[7 * 2 + 1] == -1 and pos[50 * 2] == -1
    assert m["bins"][-1].item() == 198


@pytest.mark.parametrize("dtype,H,E,K,N", [("f32", 128, 4, 2, 256), ("bf16", 512, 8, 2, 333),
                                           ("bf16", 256, 64, 6, 700), ("bf16", 7168, 16, 4, 130)])
def test_permute_bit_exact_and_pads_zero(dtype, H, E, K, N):
    shp = small_shape("p", N=N, H=H, E=E, K=K, dtype=dtype)
    c = make_case(shp, seed=2, repair=False)
    te = _routing(N, K, E, seed=7)
    m = moe.moe_dispatch_meta(te.cuda(), E)
    xp = moe.moe_permute(c["x"], m["pos"], m["bins"], m["padded_bins"], K)
    ref_m = om.dispatch_meta(te.numpy(), E)
    P = xp.shape[0]
    used = int(ref_m["padded_bins"][-1])
    ref = om.permute(c["x"].cpu(), ref_m["pos"], K, P)
    got = xp.cpu().double().numpy()
    np.testing.assert_array_equal(got[:used], ref[:used])


@pytest.mark.parametrize("dtype,H,K,N", [("f32", 128, 2, 256), ("bf16", 4096, 2, 300),
                                         ("bf16", 256, 8, 513)])
def test_combine_matches_oracle(dtype, H, K, N):
    E = 16
    te = _routing(N, K, E, seed=11)
    m = moe.moe_dispatch_meta(te.cuda(), E)
    P = moe.padded_rows_max(N, E, K)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(3)
    O = torch.randn(P, H, generator=g, device="cuda").to(tdt)
    w = torch.rand(N, K, generator=g, device="cuda")
    w = (w / w.sum(1, keepdim=True)).contiguous()
    y = moe.moe_combine(O, w, m["pos"], N)
    ref = om.combine(om.f64(O.cpu()), w.cpu().double().numpy(), om.dispatch_meta(te.numpy(), E)["pos"], N, K)
    assert_scaled(y, ref, dtype, "combine")


GROUPED = [("f32", 128, 256, 4, [200, 0, 37, 300]),
           ("bf16", 128, 256, 4, [130, 0, 1, 400]),
           ("bf16", 256, 384, 8, [0, 0, 129, 255, 256, 1, 0, 700]),
           ("bf16", 384, 1408, 3, [257, 64, 640]),
           ("bf16", 512, 512, 2, [0, 1000]),
           # experts of more than 8 row units: several raster groups per expert
           ("bf16", 256, 256, 3, [2700, 0, 4500]),
           ("bf16", 384, 256, 2, [1300, 2100]),
           # mostly one-tile experts: GEMM1 splits into a pair launch and a
           # single-CTA launch for the one-tile experts
           ("bf16", 256, 256, 16, [100, 300, 5, 128, 129, 0, 60, 700, 1, 90, 256, 257, 40, 128, 77, 500])]


@pytest.mark.parametrize("dtype,H,F,E,counts", GROUPED)
def test_grouped_swiglu_matches_oracle(dtype, H, F, E, counts):
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(H + F)
    counts = np.asarray(counts)
    padded = om.round_up(counts)
    pb = np.cumsum(padded).astype(np.int32)
    P = int(om.round_up(int(pb[-1]) + 128))
    x_perm = torch.zeros(P, H, dtype=tdt, device="cuda")
    start = 0
    for c_, p_ in zip(counts, padded):
        x_perm[start:start + c_] = torch.randn(int(c_), H, generator=g, device="cuda").to(tdt)
        start += int(p_)
    W1 = (torch.randn(E, H, F, generator=g, device="cuda") / H ** 0.5).to(tdt)
    W3 = (torch.randn(E, H, F, generator=g, device="cuda") / H ** 0.5).to(tdt)
    W2 = (torch.randn(E, F, H, generator=g, device="cuda") / F ** 0.5).to(tdt)
    pbt = torch.as_tensor(pb, device="cuda")
    act, out, gu = moe.moe_grouped_swiglu(x_perm, W1, W3, W2, pbt, save_gate_up=True)
    A, O = om.grouped_swiglu(x_perm.cpu(), W1.cpu(), W3.cpu(), W2.cpu(), pb)
    used = int(pb[-1])
    assert_scaled(act[:used], A[:used], dtype, "act")
    assert_scaled(out[:used], O[:used], dtype, "out")
    Xd = om.f64(x_perm.cpu())
    start = 0
    for e in range(E):
        end = int(pb[e])
        if end > start:
            Gr = Xd[start:end] @ om.f64(W1[e].cpu())
            assert_scaled(gu[0, start:end], Gr, dtype, f"G[{e}]")
        start = end


@pytest.mark.parametrize("dt,n,numel", [(torch.bfloat16, 8, 1 << 20), (torch.float32, 3, 4096 * 3),
                                        (torch.bfloat16, 1, 64)])
def test_sum_rank_ordered_matches_ordered_fp32_sum(dt, n, numel):
    from dropless_top_moe_b200._lib import call, MOE_BF16, MOE_F32
    g = torch.Generator(device="cuda").manual_seed(n)
    shards = torch.randn(n, numel, generator=g, device="cuda").to(dt)
    out = torch.empty(numel, dtype=dt, device="cuda")
    call("moe_sum_rank_ordered", shards.data_ptr(), n, numel, MOE_BF16 if dt == torch.bfloat16 else MOE_F32,
         1.0 / n, out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    acc = torch.zeros(numel, dtype=torch.float32, device="cuda")
    for r in range(n):
        acc += shards[r].float()
    assert torch.equal(out, (acc * (1.0 / n)).to(dt))


COMBINE_BWD = [small_shape("cb_f32", N=256, H=128, E=4, K=2, F=256, dtype="f32", training=True),
               small_shape("cb_bf16", N=700, H=256, E=16, K=4, F=256, training=True),
               small_shape("cb_bf16_k8", N=333, H=512, E=64, K=8, F=128, skew="zipf", skew_param=1.0,
                           training=True)]


@pytest.mark.parametrize("shape", COMBINE_BWD, ids=lambda s: s.name)
def test_combine_bwd_dw_and_dlogit_match_oracle(shape):
    """moe_combine_bwd per stage (MegaBlocks sec. 4: the scatter's backward is
    a gather; icman sec. 2.2: the router's gradient flows through the kept,
    renormalised weights).  dw[t,k] against the oracle's dw, and dlogit[t,k]
    against the oracle's dense softmax-and-renormalisation gradient at the
    chosen expert, which must vanish at every other expert."""
    c = make_case(shape, seed=17, with_dy=True)
    N, E, K = shape.N, shape.E, shape.K
    r = moe.moe_route(c["x"], c["W_r"], K)
    m = moe.moe_dispatch_meta(r["top_experts"], E)
    xp = moe.moe_permute(c["x"], m["pos"], m["bins"], m["padded_bins"], K)
    _, out, _ = moe.moe_grouped_swiglu(xp, c["W1"], c["W3"], c["W2"], m["padded_bins"])
    dw, dlogit, d_out = moe.moe_combine_bwd(c["dy"], out, r["weights"], m["pos"], m["bins"], m["padded_bins"])
    torch.cuda.synchronize()
    ref = om.route(c["x_cpu"], c["W_r_cpu"], K)
    np.testing.assert_array_equal(r["top_experts"].cpu().numpy(), ref["top_experts"])
    gr = om.moe_backward(c["x_cpu"], c["W_r_cpu"], c["W1"].cpu(), c["W3"].cpu(), c["W2"].cpu(), K,
                         c["dy"].cpu(), routing=ref)
    assert_scaled(dw, gr["dw"], shape.dtype, "dw")
    te = ref["top_experts"].astype(np.int64)
    chosen = np.take_along_axis(gr["dlogits"], te, axis=1)
    assert_scaled(dlogit, chosen, shape.dtype, "dlogit")
    off = gr["dlogits"].copy()
    np.put_along_axis(off, te, 0.0, axis=1)
    assert np.max(np.abs(off)) <= 1e-12 * max(1.0, np.max(np.abs(gr["dlogits"])))
    # d_out rows: the routing weight times dy, pad rows zero
    ref_m = om.dispatch_meta(ref["top_experts"], E)
    dO = d_out.cpu().double().numpy()
    w = r["weights"].cpu().double().numpy()
    dy = om.f64(c["dy"].cpu())
    pos = ref_m["pos"].reshape(N, K)
    want = np.zeros_like(dO[: int(ref_m["padded_bins"][-1])])
    for t in range(N):
        for k in range(K):
            want[pos[t, k]] = w[t, k] * dy[t]
    assert_scaled(dO[: want.shape[0]], want, shape.dtype, "d_out")
