"""Pins of the CPU oracle against things other than itself: the paper's printed
closed forms, hand-derived values, library routines (numpy / scipy) on cases
that reduce to them, brute force on tiny inputs, and invariants of the layer
(LatentMoE, arXiv 2601.18089, Section 3, Eq. (1)/(2))."""
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import softmax as sp_softmax

import oracle
from mixture_experts_layer_64_b200 import costmodel, workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f64 = np.float64


def rnd(shape, std, seed, dtype="bf16"):
    g = torch.Generator().manual_seed(seed)
    t = torch.randn(shape, generator=g) * std
    return t.to(torch.bfloat16 if dtype == "bf16" else torch.float32)


def as64(t):
    return t.to(torch.float64).numpy()


def make_layer(d, l, N, k, m, act, shared_m=0, dtype="bf16", skip_proj=False,
               bias=False, seed=0, zero_shared=False):
    m_in = 2 * m if act == "swiglu" else m
    ms_in = 2 * shared_m if act == "swiglu" else shared_m
    W = dict(
        Wg=rnd((d, N), d ** -0.5, seed + 1, dtype),
        bias=(torch.randn(N, generator=torch.Generator().manual_seed(seed + 2)).float()
              if bias else None),
        Wdown=None if skip_proj else rnd((d, l), d ** -0.5, seed + 3, dtype),
        Wup=None if skip_proj else rnd((l, d), l ** -0.5, seed + 4, dtype),
        W1=rnd((N, l, m_in), l ** -0.5, seed + 5, dtype),
        W2=rnd((N, m, l), m ** -0.5, seed + 6, dtype),
        Ws1=rnd((d, ms_in), d ** -0.5, seed + 7, dtype) if shared_m else None,
        Ws2=rnd((shared_m, d), shared_m ** -0.5, seed + 8, dtype) if shared_m else None,
    )
    if zero_shared and shared_m:
        W["Ws1"] = torch.zeros_like(W["Ws1"])
    L = oracle.OracleLayer(d=d, l=l, N=N, k=k, m=m, act=act, shared_m=shared_m,
                           dtype=dtype, skip_proj=skip_proj, **W)
    return L, W


def np_act(act, a, m):
    silu = lambda v: v / (1.0 + np.exp(-v))
    if act == "swiglu":
        return silu(a[..., :m]) * a[..., m:]
    if act == "relu2":
        return np.maximum(a, 0.0) ** 2
    return silu(a)


# ---------------------------------------------------------------------------
# closed forms printed on the pages
# ---------------------------------------------------------------------------

def test_closed_forms_match_printed_values():
    g = json.load(open(os.path.join(GOLDEN, "closed_forms.json")))
    c = g["compute_bound_threshold"]
    assert costmodel.compute_bound_threshold(c["F"], c["bw_hbm"]) == c["printed"]
    t = g["threshold_tokens"]
    root = costmodel.threshold_tokens(t["I"], t["d"], t["m"])
    assert math.floor(root) == t["printed_floor"]
    # the printed bound is the integer part of the root: I crosses 1250 there
    assert costmodel.arithmetic_intensity(t["printed_floor"], t["d"], t["m"]) < t["I"]
    assert costmodel.arithmetic_intensity(t["printed_floor"] + 1, t["d"], t["m"]) >= t["I"]
    assert costmodel.arithmetic_intensity(root, t["d"], t["m"]) == pytest.approx(t["I"], rel=1e-12)
    r = g["comm_compute_ratio"]
    assert round(costmodel.comm_compute_ratio(r["F"], r["m"], r["bw_nvl"])) == r["printed_approx"]
    v = g["comm_volume"]
    assert 2.5 * v["N"] / v["EP"] == v["printed_coefficient"]
    tb = g["table1_weight_load"]
    ratio = (costmodel.weight_load_per_expert(tb["d"], 1536)
             / costmodel.weight_load_per_expert(tb["l"], 1536))
    assert ratio == tb["alpha"] == tb["d"] / tb["l"]


def test_intensity_limits():
    # I -> 2 t for t << d, m (memory bound) and -> 2 d m / (d + m) for t -> inf
    d, m = 4096, 1536
    assert costmodel.arithmetic_intensity(1, d, m) == pytest.approx(2.0, rel=1e-3)
    assert costmodel.arithmetic_intensity(1e12, d, m) == pytest.approx(2 * d * m / (d + m), rel=1e-6)


def test_layer_counts_table1_ratio():
    """Counted expert-weight bytes: standard-MoE shape over latent shape equals
    alpha = d / l for the same N, m (Table 1)."""
    std = costmodel.layer_counts(T=256, d=4096, l=4096, N=128, k=8, m=1536, act="swiglu",
                                 skip_proj=True)
    lat = costmodel.layer_counts(T=256, d=4096, l=1024, N=128, k=8, m=1536, act="swiglu")
    assert std.expert_weight_bytes / lat.expert_weight_bytes == 4.0


# ---------------------------------------------------------------------------
# routing: brute force and library routines
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,N,k,seed", [(1, 1, 1, 0), (7, 5, 2, 1), (64, 16, 4, 2),
                                        (33, 128, 8, 3), (40, 512, 32, 4), (17, 896, 16, 5),
                                        (9, 16, 16, 6)])
def test_route_brute_force(T, N, k, seed):
    lg = workloads.make_logits(T, N, seed, ties=True).numpy()
    idx, w, offsets, perm = oracle.route(lg, k)
    for t in range(T):
        # brute force: full sort of all (value, index) pairs
        order = sorted(range(N), key=lambda e: (-float(lg[t, e]), e))[:k]
        assert list(idx[t]) == order
        ref = sp_softmax(lg[t, order].astype(f64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-14, atol=1e-300)
    # grouping by expert: a stable argsort of the flattened expert ids
    ref_perm = np.argsort(idx.ravel(), kind="stable")
    np.testing.assert_array_equal(perm, ref_perm)
    counts = np.bincount(idx.ravel(), minlength=N)
    np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))


def test_route_invariants_and_special_cases():
    lg = workloads.make_logits(200, 64, 11, ties=True).numpy()
    idx, w, offsets, perm = oracle.route(lg, 6)
    assert offsets[-1] == 200 * 6
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    np.testing.assert_array_equal(perm[inv], np.arange(perm.size))
    for e in range(64):
        rows = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[rows] == e)
        assert np.all(np.diff(rows // 6) > 0)          # strictly ascending token
    np.testing.assert_allclose(w.sum(1), 1.0, rtol=0, atol=1e-15)
    assert np.all(np.diff(w, axis=1) <= 0)              # weights follow slot order
    # k = 1: a single weight of exactly one
    _, w1, _, _ = oracle.route(lg, 1)
    assert np.all(w1 == 1.0)
    # signed zeros compare equal: index order decides
    z = np.array([[-0.0, 0.0, -0.0, 0.0]], dtype=np.float32)
    assert list(oracle.route(z, 3)[0][0]) == [0, 1, 2]
    # all-equal row: the first k experts, uniform weights
    u = np.full((1, 8), 0.5, dtype=np.float32)
    i8, w8, _, _ = oracle.route(u, 4)
    assert list(i8[0]) == [0, 1, 2, 3] and np.all(w8 == 0.25)
    with pytest.raises(oracle.OracleError):
        oracle.route(np.array([[0.0, np.nan]], dtype=np.float32), 1)


@pytest.mark.parametrize("T,N,k,seed", [(9, 16, 4, 21), (33, 128, 8, 22), (17, 896, 16, 23),
                                        (5, 12, 12, 24)])
def test_route_full_softmax_is_softmax_over_all_experts(T, N, k, seed):
    """Eq. (1) read literally: the gate of a chosen expert is its entry of
    the softmax over all N logits (scipy), so the k gates sum to below one
    unless k = N, where the variant equals the renormalised default."""
    lg = workloads.make_logits(T, N, seed, ties=True).numpy()
    idx, w, offsets, perm = oracle.route(lg, k, full_softmax=True)
    idx0, w0, off0, perm0 = oracle.route(lg, k)
    np.testing.assert_array_equal(idx, idx0)          # the selection is unchanged
    np.testing.assert_array_equal(perm, perm0)
    np.testing.assert_array_equal(offsets, off0)
    p = sp_softmax(lg.astype(f64), axis=1)
    np.testing.assert_allclose(w, np.take_along_axis(p, idx.astype(np.int64), axis=1),
                               rtol=1e-13, atol=1e-300)
    if k < N:
        assert np.all(w.sum(1) < 1.0)
    else:
        np.testing.assert_allclose(w, w0, rtol=1e-14)


@pytest.mark.parametrize("full", [False, True])
def test_route_bias_selects_only(full):
    """Auxiliary-loss-free balancing (Section 4): the bias moves the choice,
    computed on the fp32 sum logit + bias (brute-force sort of numpy float32
    sums), while the gates come from the logits alone (scipy softmax)."""
    T, N, k = 40, 64, 6
    lg = workloads.make_logits(T, N, 31, ties=True).numpy()
    b = (np.random.default_rng(5).normal(size=N) * 2.0).astype(np.float32)
    idx, w, offsets, perm = oracle.route(lg, k, sel_bias=b, full_softmax=full)
    key = lg + b[None, :]                              # float32 + float32 -> float32
    assert key.dtype == np.float32
    for t in range(T):
        order = sorted(range(N), key=lambda e: (-float(key[t, e]), e))[:k]
        assert list(idx[t]) == order
        if full:
            ref = sp_softmax(lg[t].astype(f64))[order]
        else:
            ref = sp_softmax(lg[t, order].astype(f64))
        np.testing.assert_allclose(w[t], ref, rtol=1e-13, atol=1e-300)
    # the bias changed the selection of some tokens (it is large on purpose)
    assert not np.array_equal(idx, oracle.route(lg, k)[0])
    np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))


def test_layer_route_modes():
    """The layer-level route mode: with the bias selecting only, the router
    logits leave the bias out, and the whole layer equals the forward step
    fed by the variant routing."""
    L0, W = make_layer(64, 32, 12, 3, 24, "relu2", bias=True, seed=40)
    x = rnd((10, 64), 1.0, 41)
    for mode in (oracle.ROUTE_BIAS_SELECT, oracle.ROUTE_FULL_SOFTMAX,
                 oracle.ROUTE_BIAS_SELECT | oracle.ROUTE_FULL_SOFTMAX):
        L = oracle.OracleLayer(d=64, l=32, N=12, k=3, m=24, act="relu2", route_mode=mode, **W)
        lg = L.router_logits(x)
        plain = as64(x) @ as64(W["Wg"])
        if mode & oracle.ROUTE_BIAS_SELECT:
            np.testing.assert_allclose(lg, plain, rtol=1e-12, atol=1e-12)
        else:
            np.testing.assert_allclose(lg, plain + W["bias"].double().numpy(), rtol=1e-12,
                                       atol=1e-12)
        sb = W["bias"] if mode & oracle.ROUTE_BIAS_SELECT else None
        idx, w, _, _ = oracle.route(lg.astype(np.float32), 3, sel_bias=sb,
                                    full_softmax=bool(mode & oracle.ROUTE_FULL_SOFTMAX))
        res = L.layer(x)
        np.testing.assert_array_equal(res["idx"], idx)
        np.testing.assert_allclose(res["w"], w, rtol=1e-15)
        np.testing.assert_allclose(res["out"], L.forward(x, idx, w), rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------------
# router logits: a library matmul
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_router_logits_match_numpy(dtype):
    L, W = make_layer(96, 32, 24, 3, 40, "silu", dtype=dtype, bias=True)
    x = rnd((20, 96), 1.0, 99, dtype)
    got = L.router_logits(x)
    ref = as64(x) @ as64(W["Wg"]) + W["bias"].double().numpy()[None]
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# whole layer: hand-derived values and reductions to dense matmuls
# ---------------------------------------------------------------------------

def test_hand_worked_example_relu2_k2():
    """d=2, l=1, N=2, k=2, m=1, squared ReLU; every number chosen by hand.
    logits = [1.0, 0.5] -> slots (0, 1), w0 = 1/(1+e^-0.5); z = 3;
    y0 = relu2(3*1)*2 = 18, y1 = relu2(3*0.5)*4 = 9; comb = 18 w0 + 9 w1;
    out = x + comb * [1, -1]."""
    bf = torch.bfloat16
    x = torch.tensor([[1.0, 2.0]], dtype=bf)
    W = dict(Wg=torch.tensor([[0.0, 0.5], [0.5, 0.0]], dtype=bf),
             Wdown=torch.tensor([[1.0], [1.0]], dtype=bf),
             Wup=torch.tensor([[1.0, -1.0]], dtype=bf),
             W1=torch.tensor([[[1.0]], [[0.5]]], dtype=bf),
             W2=torch.tensor([[[2.0]], [[4.0]]], dtype=bf))
    L = oracle.OracleLayer(d=2, l=1, N=2, k=2, m=1, act="relu2", **W)
    r = L.layer(x)
    w0 = 1.0 / (1.0 + math.exp(-0.5))
    comb = 18.0 * w0 + 9.0 * (1.0 - w0)
    assert list(r["idx"][0]) == [0, 1]
    assert r["w"][0, 0] == pytest.approx(w0, rel=1e-15)
    np.testing.assert_allclose(r["out"][0], [1.0 + comb, 2.0 - comb], rtol=1e-14)


def test_hand_worked_example_swiglu_halves():
    """m=1 SwiGLU: FC1 columns are [gate | up]; h = silu(z g) * (z u).
    z = 2 (identity down-projection on d=l=1 via skip), g = 1, u = 3:
    h = silu(2) * 6, y = h * 0.5, out = x + y."""
    bf = torch.bfloat16
    x = torch.tensor([[2.0]], dtype=bf)
    W = dict(Wg=torch.tensor([[1.0]], dtype=bf),
             W1=torch.tensor([[[1.0, 3.0]]], dtype=bf),
             W2=torch.tensor([[[0.5]]], dtype=bf))
    L = oracle.OracleLayer(d=1, l=1, N=1, k=1, m=1, act="swiglu", skip_proj=True, **W)
    out = L.layer(x)["out"]
    silu2 = 2.0 / (1.0 + math.exp(-2.0))
    assert out[0, 0] == pytest.approx(2.0 + silu2 * 6.0 * 0.5, rel=1e-15)


@pytest.mark.parametrize("act", ["silu", "swiglu", "relu2"])
def test_single_expert_reduces_to_dense_ffn(act):
    """N = k = 1: w = 1 and the layer is x + act(x Wd W1) W2 Wu + act(x Ws1) Ws2,
    non-square everywhere so that a transposed operand cannot pass."""
    d, l, m, ms = 48, 16, 24, 40
    L, W = make_layer(d, l, 1, 1, m, act, shared_m=ms, seed=10)
    x = rnd((9, d), 1.0, 77)
    out = L.layer(x)["out"]
    X = as64(x)
    z = X @ as64(W["Wdown"])
    y = np_act(act, z @ as64(W["W1"][0]), m) @ as64(W["W2"][0])
    s = np_act(act, X @ as64(W["Ws1"]), ms) @ as64(W["Ws2"])
    ref = X + y @ as64(W["Wup"]) + s
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("act", ["silu", "swiglu", "relu2"])
def test_brute_force_per_token_mixture(act):
    """Per-token naive evaluation of Eq. (1) with the selection by full sort and
    the weights by scipy softmax, on a small layer with a bias."""
    d, l, N, k, m = 32, 8, 6, 3, 12
    L, W = make_layer(d, l, N, k, m, act, bias=True, seed=20)
    x = rnd((11, d), 1.0, 5)
    r = L.layer(x)
    X = as64(x)
    lg32 = (X @ as64(W["Wg"]) + W["bias"].double().numpy()).astype(np.float32)
    for t in range(11):
        sel = sorted(range(N), key=lambda e: (-float(lg32[t, e]), e))[:k]
        wt = sp_softmax(lg32[t, sel].astype(f64))
        z = X[t] @ as64(W["Wdown"])
        comb = sum(wt[j] * (np_act(act, z @ as64(W["W1"][e]), m) @ as64(W["W2"][e]))
                   for j, e in enumerate(sel))
        ref = X[t] + comb @ as64(W["Wup"])
        assert list(r["idx"][t]) == sel
        np.testing.assert_allclose(r["out"][t], ref, rtol=1e-11, atol=1e-11)


def test_uniform_routing_is_mean_of_all_experts():
    """k = N with W_g = 0 and no bias: all logits are 0, the weights are 1/N
    exactly and the routed output is the mean over all experts."""
    d, l, N, m = 24, 8, 4, 10
    L0, W = make_layer(d, l, N, N, m, "relu2", seed=30)
    W["Wg"] = torch.zeros_like(W["Wg"])
    L = oracle.OracleLayer(d=d, l=l, N=N, k=N, m=m, act="relu2", **W)
    x = rnd((5, d), 1.0, 6)
    r = L.layer(x)
    assert np.all(r["w"] == 0.25)
    assert np.all(r["idx"] == np.arange(N))
    X = as64(x)
    z = X @ as64(W["Wdown"])
    mean = sum(np_act("relu2", z @ as64(W["W1"][e]), m) @ as64(W["W2"][e]) for e in range(N)) / N
    np.testing.assert_allclose(r["out"], X + mean @ as64(W["Wup"]), rtol=1e-11, atol=1e-11)


def test_identity_projections_equal_projection_skip():
    """l = d with W_down = W_up = I is the standard MoE of Table 1's first row:
    identical (bit for bit) to the projection-skip path."""
    d, N, k, m = 32, 8, 2, 16
    L, W = make_layer(d, d, N, k, m, "swiglu", seed=40)
    eye = torch.eye(d, dtype=torch.bfloat16)
    Wi = dict(W, Wdown=eye, Wup=eye)
    Li = oracle.OracleLayer(d=d, l=d, N=N, k=k, m=m, act="swiglu", **Wi)
    Ws = dict(W, Wdown=None, Wup=None)
    Ls = oracle.OracleLayer(d=d, l=d, N=N, k=k, m=m, act="swiglu", skip_proj=True, **Ws)
    x = rnd((13, d), 1.0, 8)
    a, b = Li.layer(x), Ls.layer(x)
    np.testing.assert_array_equal(a["out"], b["out"])
    np.testing.assert_array_equal(a["idx"], b["idx"])


def test_token_independence_and_thread_count():
    L, W = make_layer(40, 12, 10, 3, 20, "swiglu", shared_m=16, bias=True, seed=50)
    x = rnd((31, 40), 1.0, 9)
    full = L.layer(x, nthreads=1)["out"]
    np.testing.assert_array_equal(full, L.layer(x, nthreads=7)["out"])
    sub = [30, 3, 17, 3, 0]
    np.testing.assert_array_equal(L.layer(x, tokens=sub)["out"], full[sub])
    np.testing.assert_array_equal(L.layer(x[sub])["out"], full[sub])


def test_expert_relabelling_invariance():
    d, l, N, k, m = 32, 8, 9, 3, 12
    L, W = make_layer(d, l, N, k, m, "silu", bias=True, seed=60)
    x = rnd((15, d), 1.0, 10)
    base = L.layer(x)
    p = np.random.default_rng(0).permutation(N)
    Wp = dict(W, Wg=W["Wg"][:, p], bias=W["bias"][p], W1=W["W1"][p], W2=W["W2"][p])
    Lp = oracle.OracleLayer(d=d, l=l, N=N, k=k, m=m, act="silu", **Wp)
    r = Lp.layer(x)
    np.testing.assert_array_equal(r["out"], base["out"])
    np.testing.assert_array_equal(p[r["idx"]], base["idx"])


def test_shared_expert_zero_and_split():
    d, l, N, k, m, ms = 32, 8, 6, 2, 12, 20
    L, W = make_layer(d, l, N, k, m, "relu2", shared_m=ms, seed=70)
    x = rnd((7, d), 1.0, 12)
    # a zero first matrix makes the shared expert vanish (relu2(0) = 0)
    Wz = dict(W, Ws1=torch.zeros_like(W["Ws1"]))
    Lz = oracle.OracleLayer(d=d, l=l, N=N, k=k, m=m, act="relu2", shared_m=ms, **Wz)
    Lr = oracle.OracleLayer(d=d, l=l, N=N, k=k, m=m, act="relu2",
                            **dict(W, Ws1=None, Ws2=None))
    np.testing.assert_array_equal(Lz.layer(x)["out"], Lr.layer(x)["out"])
    # two shared experts equal one of concatenated width (Table 2 has S = 2)
    full = L.layer(x)["out"] - Lr.layer(x)["out"]
    X = as64(x)
    half = ms // 2
    parts = sum(np_act("relu2", X @ as64(W["Ws1"][:, sl]), half) @ as64(W["Ws2"][sl])
                for sl in (slice(0, half), slice(half, ms)))
    np.testing.assert_allclose(full, parts, rtol=1e-9, atol=1e-10)


def test_missing_expert_is_reported():
    d, l, N, k, m = 16, 8, 4, 2, 8
    _, W = make_layer(d, l, N, k, m, "silu", seed=80)
    only = {0: W["W1"][0]}
    L = oracle.OracleLayer(d=d, l=l, N=N, k=k, m=m, act="silu",
                           **dict(W, W1=only, W2={0: W["W2"][0]}))
    x = rnd((4, d), 1.0, 13)
    with pytest.raises(oracle.OracleError):
        L.layer(x)


def test_workload_generator_is_deterministic_and_shaped():
    w = workloads.WORKLOADS["tiny-fp32"]
    a = workloads.make_weights(w)
    b = workloads.make_weights(w)
    for key in a:
        if a[key] is None:
            assert b[key] is None
        else:
            assert torch.equal(a[key], b[key])
    assert a["W1"].shape == (w.N, w.l, w.m_in) and a["W2"].shape == (w.N, w.m, w.l)
    assert a["W1"].dtype == torch.float32
    assert torch.equal(a["W1"][3], workloads.make_expert_W1(w, 3))
    zb = workloads.zipf_log_bias(896)
    assert zb.dtype == torch.float32 and bool(torch.all(zb[1:] < zb[:-1]))
    assert math.fsum(math.exp(v) for v in zb.double().tolist()) == pytest.approx(1.0, rel=1e-6)


def test_tiny_workload_end_to_end_runs():
    w = workloads.WORKLOADS["tiny-fp32"]
    W = workloads.make_weights(w)
    x = workloads.make_x(w)
    L = oracle.OracleLayer(d=w.d, l=w.l, N=w.N, k=w.k, m=w.m, act=w.act, dtype="f32", **W)
    r = L.layer(x)
    assert r["out"].shape == (w.T, w.d) and np.all(np.isfinite(r["out"]))
    np.testing.assert_allclose(r["w"].sum(1), 1.0, atol=1e-15)


# ---------------------------------------------------------------------------
# fp8 E4M3 expert weights with per-output-column scales
# ---------------------------------------------------------------------------

def test_e4m3_decode_matches_torch_for_every_code():
    """The oracle's E4M3 decoder against torch's float8_e4m3fn conversion (a
    library routine) for all 256 codes: 0x7F/0xFF are NaN, the rest exact."""
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).float().numpy().astype(f64)
    got = np.array([oracle.e4m3_value(c) for c in range(256)])
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_quantiser_round_trip():
    """Per-column scales map each column's largest magnitude to 448, and the
    decoded codes times the scales stay within half an E4M3 step of W."""
    W = rnd((3, 40, 24), 0.2, 51, "f32")
    codes, scale = workloads.quantize_e4m3(W)
    assert codes.dtype == torch.uint8 and scale.shape == (3, 24)
    dec = np.vectorize(oracle.e4m3_value)(codes.numpy())
    deq = dec * scale.numpy()[:, None, :]
    np.testing.assert_allclose(np.abs(dec).max(axis=1), 448.0)
    Wn = W.double().numpy()
    # relative half-step of E4M3 (3 mantissa bits) = 2^-4, or the subnormal step
    tol = np.maximum(np.abs(Wn) * 2.0 ** -4, scale.numpy()[:, None, :] * 2.0 ** -10)
    assert np.all(np.abs(deq - Wn) <= tol * 1.0000001)


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_fp8_single_expert_is_dense_chain(act):
    """N = k = 1 with fp8 experts: the layer is x + act(z (q1 s1)) (q2 s2) Wup
    with the dequantised matrices built in numpy (codes decoded, each output
    column times its scale)."""
    d, l, m = 48, 32, 40
    L0, W = make_layer(d, l, 1, 1, m, act, seed=60, dtype="f32")
    q1, s1 = workloads.quantize_e4m3(W["W1"])
    q2, s2 = workloads.quantize_e4m3(W["W2"])
    L = oracle.OracleLayer(d=d, l=l, N=1, k=1, m=m, act=act, dtype="f32", Wg=W["Wg"],
                           Wdown=W["Wdown"], Wup=W["Wup"], W1=q1, W2=q2, W1s=s1, W2s=s2)
    x = rnd((7, d), 1.0, 61, "f32")
    dec = np.vectorize(oracle.e4m3_value)
    W1d = dec(q1[0].numpy()) * s1[0].double().numpy()[None, :]
    W2d = dec(q2[0].numpy()) * s2[0].double().numpy()[None, :]
    z = as64(x) @ as64(W["Wdown"])
    h = np_act(act, z @ W1d, m)
    ref = as64(x) + (h @ W2d) @ as64(W["Wup"])
    res = L.layer(x)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def test_fp8_layer_equals_layer_with_dequantised_weights():
    """Many experts: the fp8 layer equals the f32 layer whose expert weights
    are the dequantised values (rounded to fp32, hence 1e-6); a scale applied
    per input row instead of per output column would miss by far."""
    d, l, N, k, m = 40, 24, 6, 2, 16
    L0, W = make_layer(d, l, N, k, m, "swiglu", dtype="f32", bias=True, seed=70)
    q1, s1 = workloads.quantize_e4m3(W["W1"])
    q2, s2 = workloads.quantize_e4m3(W["W2"])
    dec = np.vectorize(oracle.e4m3_value)
    W1d = torch.from_numpy((dec(q1.numpy()) * s1.double().numpy()[:, None, :]).astype(np.float32))
    W2d = torch.from_numpy((dec(q2.numpy()) * s2.double().numpy()[:, None, :]).astype(np.float32))
    common = dict(d=d, l=l, N=N, k=k, m=m, act="swiglu", dtype="f32", Wg=W["Wg"],
                  bias=W["bias"], Wdown=W["Wdown"], Wup=W["Wup"])
    L8 = oracle.OracleLayer(W1=q1, W2=q2, W1s=s1, W2s=s2, **common)
    Ld = oracle.OracleLayer(W1=W1d, W2=W2d, **common)
    x = rnd((30, d), 1.0, 71, "f32")
    a, b = L8.layer(x), Ld.layer(x)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-6, atol=1e-6)
    with pytest.raises(oracle.OracleError):
        oracle.OracleLayer(W1=q1, W2=q2, W1s=s1, **common)


# ---------------------------------------------------------------------------
# block-scaled FP4 (MXFP4) expert weights
# ---------------------------------------------------------------------------

# E2M1 (the OCP microscaling FP4 element): 1 sign, 2 exponent bits (bias 1),
# 1 mantissa bit, exponent 0 subnormal -- written out from that definition
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_is_the_format_table():
    got = [oracle.e2m1_value(c) for c in range(16)]
    assert got[:8] == E2M1_TABLE
    assert got[8:] == [-v for v in E2M1_TABLE]
    assert np.signbit(got[8])  # code 8 is -0


def _np_dequant_mxfp4(q, e):
    """numpy decode of output-major MXFP4 (codes [..., out, in/2], exponents
    [..., out, in/32]) back to the API layout [..., in, out]."""
    q = np.asarray(q, dtype=np.uint8)
    lo, hi = q & 15, q >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(*q.shape[:-1], q.shape[-1] * 2)
    mag = np.array(E2M1_TABLE)[codes & 7] * np.where(codes & 8, -1.0, 1.0)
    scale = np.exp2(np.asarray(e, dtype=np.float64) - 127.0)
    vals = mag * np.repeat(scale, 32, axis=-1)
    return np.swapaxes(vals, -1, -2)


def test_mxfp4_quantiser_round_trip():
    """Each block's scale maps its largest magnitude into [4, 8) (saturating
    at 6), the dequantised codes stay within half a grid step of W, values on
    the grid come back exactly and midpoints go to the even code."""
    W = rnd((3, 64, 24), 0.2, 81, "f32")
    q, e = workloads.quantize_mxfp4(W)
    assert q.shape == (3, 24, 32) and e.shape == (3, 24, 2) and q.dtype == torch.uint8
    deq = _np_dequant_mxfp4(q.numpy(), e.numpy())
    Wn = W.double().numpy()
    blk = np.abs(Wn).reshape(3, 2, 32, 24).max(axis=2)                 # [3, 2 blocks, 24]
    sc = np.exp2(np.swapaxes(e.numpy().astype(np.float64) - 127.0, -1, -2))  # [3, 2, 24]
    assert np.all((blk / sc >= 4.0) & (blk / sc < 8.0))
    # half the grid step at the value's magnitude; above 6 the code saturates
    X = np.repeat(sc, 32, axis=1)
    v = np.abs(Wn) / X
    step = np.where(v >= 4.0, 2.0, np.where(v >= 2.0, 1.0, 0.5))
    bound = np.where(v > 6.0, (v - 6.0) * X, step / 2 * X)
    assert np.all(np.abs(deq - Wn) <= bound * 1.0000001 + 1e-300)
    # grid values and midpoints (scale 1: the block's largest magnitude in [4, 8))
    vals = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 0.25, 0.75, 1.25, 1.75,
                         2.5, 3.5, 5.0, -0.75, -5.0, 7.9, -1.5, 0.5, 0.0, 1.0, 2.0, 3.0,
                         4.0, 6.0, -6.0, 0.1, 0.3, 2.9, 3.1, 5.1]).reshape(32, 1)
    q1, e1 = workloads.quantize_mxfp4(vals)
    assert int(e1[0, 0]) == 127
    got = _np_dequant_mxfp4(q1.numpy(), e1.numpy())[:, 0]
    want = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, -1.0,
            -4.0, 6.0, -1.5, 0.5, 0.0, 1.0, 2.0, 3.0, 4.0, 6.0, -6.0, 0.0, 0.5, 3.0, 3.0, 6.0]
    assert got.tolist() == want


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_fp4_single_expert_is_dense_chain(act):
    """N = k = 1 with MXFP4 experts: the layer is x + act(z W1d) W2d Wup with
    the matrices decoded in numpy (nibbles through the format table, each
    block of 32 inputs times its power of two)."""
    d, l, m = 48, 64, 96
    L0, W = make_layer(d, l, 1, 1, m, act, seed=82, dtype="f32")
    q1, e1 = workloads.quantize_mxfp4(W["W1"])
    q2, e2 = workloads.quantize_mxfp4(W["W2"])
    L = oracle.OracleLayer(d=d, l=l, N=1, k=1, m=m, act=act, dtype="f32", Wg=W["Wg"],
                           Wdown=W["Wdown"], Wup=W["Wup"], W1=q1, W2=q2, W1e=e1, W2e=e2)
    x = rnd((7, d), 1.0, 83, "f32")
    W1d = _np_dequant_mxfp4(q1[0].numpy(), e1[0].numpy())
    W2d = _np_dequant_mxfp4(q2[0].numpy(), e2[0].numpy())
    z = as64(x) @ as64(W["Wdown"])
    h = np_act(act, z @ W1d, m)
    ref = as64(x) + (h @ W2d) @ as64(W["Wup"])
    res = L.layer(x)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-12, atol=1e-12)


def test_fp4_layer_equals_layer_with_dequantised_weights():
    """Many experts: the MXFP4 layer equals the f32 layer whose expert weights
    are the decoded values (exact in fp32); exponents applied per output
    column instead of per block of inputs would miss."""
    d, l, N, k, m = 40, 64, 6, 2, 32
    L0, W = make_layer(d, l, N, k, m, "swiglu", dtype="f32", bias=True, seed=84)
    q1, e1 = workloads.quantize_mxfp4(W["W1"])
    q2, e2 = workloads.quantize_mxfp4(W["W2"])
    W1d = torch.from_numpy(_np_dequant_mxfp4(q1.numpy(), e1.numpy()).astype(np.float32))
    W2d = torch.from_numpy(_np_dequant_mxfp4(q2.numpy(), e2.numpy()).astype(np.float32))
    common = dict(d=d, l=l, N=N, k=k, m=m, act="swiglu", dtype="f32", Wg=W["Wg"],
                  bias=W["bias"], Wdown=W["Wdown"], Wup=W["Wup"])
    L4 = oracle.OracleLayer(W1=q1, W2=q2, W1e=e1, W2e=e2, **common)
    Ld = oracle.OracleLayer(W1=W1d, W2=W2d, **common)
    x = rnd((30, d), 1.0, 85, "f32")
    a, b = L4.layer(x), Ld.layer(x)
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-12, atol=1e-12)
    with pytest.raises(oracle.OracleError):
        oracle.OracleLayer(W1=q1, W2=q2, W1e=e1, **common)
