"""GPU parity of the CUDA library against the CPU oracle, through the C ABI.

Routing on shared fp32 logits is compared bit for bit (indices, offsets,
permutation); floating-point outputs within the stated tolerances on the five
workloads (bf16 storage with fp32 accumulation: max-abs <= 2e-2 and rel-L2 <=
5e-3; the fp32 layer: rel-L2 <= 1e-5) and within the arithmetic-derived bound
on the smaller test layers.  See tests/parity.py for how near-ties and the
bounds are handled.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_64_b200 import lmoe, workloads
from parity import check_forward, gpu_layer, sample_tokens

pytestmark = pytest.mark.gpu

W_ = workloads.Workload


# ---------------------------------------------------------------------------
# routing on shared logits: bit-exact
# ---------------------------------------------------------------------------

def _route_case(T, N, k, seed, bias=None):
    lg = workloads.make_logits(T, N, seed, bias=bias, ties=True)
    w = W_("route", T=max(T, 1), d=64, l=64, N=N, k=k, m=64, act="silu", dtype="bf16")
    L = lmoe.LatentMoELayer(w.d, w.l, N, k, w.m, act="silu", dtype="bf16")
    L.reserve(max(T, 1))
    r = L.route_only(lg.cuda())
    torch.cuda.synchronize()
    if T == 0:
        assert torch.all(r["offsets"] == 0)
        return
    o_idx, o_w, o_off, o_perm = oracle.route(lg.numpy(), k)
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), o_idx)
    np.testing.assert_array_equal(r["offsets"].cpu().numpy(), o_off)
    np.testing.assert_array_equal(r["perm"].cpu().numpy(), o_perm)
    np.testing.assert_allclose(r["w"].cpu().numpy(), o_w, rtol=2e-6, atol=1e-7)
    assert L.last_error() == (lmoe.OK, 0)


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_route_only_bit_exact_workload_shapes(name):
    w = workloads.WORKLOADS[name]
    _route_case(w.T, w.N, w.k, seed=w.seed + 10, bias=workloads.make_bias(w))


@pytest.mark.parametrize("T,N,k", [(1, 1, 1), (1, 16, 4), (33, 16, 16), (31, 7, 3), (32, 64, 1),
                                   (1000, 128, 8), (4097, 512, 22), (0, 16, 4), (65, 1024, 32),
                                   (300, 896, 16)])
def test_route_only_bit_exact_edges(T, N, k):
    _route_case(T, N, k, seed=T * 7 + N + k)


@pytest.mark.parametrize("T,N,k", [(200, 896, 16), (100, 512, 22), (64, 128, 8), (40, 1024, 32)])
def test_route_only_bit_exact_crowded_logits(T, N, k):
    """Logits on a coarse grid (six values, zeros of both signs): far more than
    k keys sit at or above the k-th largest lane maximum, so selection takes
    the exact radix-select branch, and ties decide most of the order."""
    g = torch.Generator().manual_seed(T + N + k)
    lg = (torch.randint(-3, 3, (T, N), generator=g).float() * 0.5)
    neg = torch.rand((T, N), generator=g) < 0.5
    lg = torch.where((lg == 0) & neg, torch.tensor(-0.0), lg)
    L = lmoe.LatentMoELayer(64, 64, N, k, 64, act="silu", dtype="bf16")
    L.reserve(T)
    r = L.route_only(lg.cuda())
    torch.cuda.synchronize()
    o_idx, o_w, o_off, o_perm = oracle.route(lg.numpy(), k)
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), o_idx)
    np.testing.assert_array_equal(r["offsets"].cpu().numpy(), o_off)
    np.testing.assert_array_equal(r["perm"].cpu().numpy(), o_perm)
    np.testing.assert_allclose(r["w"].cpu().numpy(), o_w, rtol=2e-6, atol=1e-7)


ROUTE_VARIANTS = [lmoe.ROUTE_FULL_SOFTMAX, lmoe.ROUTE_BIAS_SELECT,
                  lmoe.ROUTE_FULL_SOFTMAX | lmoe.ROUTE_BIAS_SELECT]


@pytest.mark.parametrize("flags", ROUTE_VARIANTS)
@pytest.mark.parametrize("T,N,k", [(300, 896, 16), (257, 512, 32), (100, 16, 4), (40, 128, 8)])
def test_route_only_variants_bit_exact(flags, T, N, k):
    """Routing variants on shared logits: the choice (on logit + bias in
    fp32 when the bias selects only) bit-exact; gates from the logits alone,
    renormalised or the softmax over all N (fp32 sum over N: 2e-5)."""
    w_ = W_("route-var", T=T, d=64, l=64, N=N, k=k, m=64, act="silu", bias="normal0.5",
            seed=T + N)
    W = workloads.make_weights(w_, device="cuda")
    W["bias"] = (torch.randn(N, generator=torch.Generator().manual_seed(N)) * 2.0).cuda()
    L, _ = gpu_layer(w_, flags, W)
    lg = workloads.make_logits(T, N, seed=T * 3 + k, ties=True)
    r = L.route_only(lg.cuda())
    torch.cuda.synchronize()
    sb = W["bias"].cpu().numpy() if flags & lmoe.ROUTE_BIAS_SELECT else None
    o_idx, o_w, o_off, o_perm = oracle.route(lg.numpy(), k, sel_bias=sb,
                                             full_softmax=bool(flags & lmoe.ROUTE_FULL_SOFTMAX))
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), o_idx)
    np.testing.assert_array_equal(r["offsets"].cpu().numpy(), o_off)
    np.testing.assert_array_equal(r["perm"].cpu().numpy(), o_perm)
    rtol = 2e-5 if flags & lmoe.ROUTE_FULL_SOFTMAX else 2e-6
    np.testing.assert_allclose(r["w"].cpu().numpy(), o_w, rtol=rtol, atol=1e-9)
    if flags & lmoe.ROUTE_BIAS_SELECT:  # the bias is large enough to move the choice
        assert not np.array_equal(o_idx, oracle.route(lg.numpy(), k)[0])


@pytest.mark.parametrize("flags", ROUTE_VARIANTS)
@pytest.mark.parametrize("name", ["silu-bias", "fp32"])
def test_forward_routing_variants(name, flags):
    w = SMALL[name]
    W = workloads.make_weights(w, device="cuda")
    W["bias"] = (torch.randn(w.N, generator=torch.Generator().manual_seed(7)) * 1.5).cuda()
    res = check_forward(w, flags=flags, W=W, fixture=True)
    assert res["unique"] >= 0.8 * res["tokens"]


def test_route_only_rejects_oversized_T():
    L = lmoe.LatentMoELayer(64, 64, 16, 4, 64, act="silu", dtype="bf16")
    L.reserve(8)
    with pytest.raises(lmoe.LmoeError):
        L.route_only(torch.zeros((9, 16), device="cuda"))


# ---------------------------------------------------------------------------
# small layers that span several tiles with ragged tails
# ---------------------------------------------------------------------------

SMALL = {
    # tcgen05 path: K multiples of 64, feature and row tiles with ragged tails
    "swiglu": W_("s-swiglu", T=300, d=256, l=128, N=8, k=3, m=192, act="swiglu", seed=11),
    "relu2-shared": W_("s-relu2", T=260, d=256, l=192, N=6, k=2, m=320, act="relu2",
                       shared_m=320, seed=12),
    "silu-bias": W_("s-silu", T=200, d=320, l=128, N=12, k=4, m=128, act="silu",
                    bias="normal0.5", seed=13),
    "swiglu-shared": W_("s-swiglu-sh", T=150, d=192, l=64, N=5, k=2, m=64, act="swiglu",
                        shared_m=192, seed=14),
    "skip": W_("s-skip", T=130, d=256, l=256, N=4, k=2, m=128, act="swiglu", skip_proj=True,
               seed=15),
    "skip-shared": W_("s-skip-sh", T=70, d=128, l=128, N=4, k=1, m=64, act="relu2",
                      skip_proj=True, shared_m=128, seed=16),
    # shapes the tcgen05 kernel does not take (K % 64 != 0): CUDA-core path
    "odd-K": W_("s-odd", T=90, d=200, l=72, N=6, k=2, m=40, act="swiglu", shared_m=24, seed=17),
    "fp32": W_("s-f32", T=100, d=96, l=32, N=8, k=3, m=48, act="relu2", shared_m=16, dtype="f32",
               seed=18),
}


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layer_default_path(name):
    res = check_forward(SMALL[name], fixture=True)
    assert res["unique"] >= res["tokens"] * 0.9


def paths(res):
    """(FC1, FC2) expert kernels of the last forward."""
    return res["expert_path"] & 7, res["expert_path"] >> 3


@pytest.mark.parametrize("name", ["swiglu", "relu2-shared", "skip"])
@pytest.mark.parametrize("flags", [0, lmoe.FORCE_SWAP, lmoe.FORCE_NOSWAP, lmoe.FORCE_WS_PAIR,
                                   lmoe.FORCE_NOPAIR, lmoe.FORCE_SIMT, lmoe.LOAD_SPLIT])
def test_small_layer_each_expert_kernel(name, flags):
    """Every expert kernel on the same layers (FC1, FC2): token-tiled with FC2
    on CTA pairs (1, 3, the default at these row counts), weight-stationary
    on single CTAs (2, 2), weight-stationary on CTA pairs (4, 4), token-tiled
    on single CTAs (1, 1), CUDA cores (0, 0), and split by load (5, 5: CTA
    pairs with FC1's rows gathered in both CTAs for the experts above 384
    rows, weight-stationary tiles of up to 128 / 256 rows for the rest)."""
    res = check_forward(SMALL[name], flags=flags, fixture=True)
    want = {0: (1, 3), lmoe.FORCE_SWAP: (2, 2), lmoe.FORCE_NOSWAP: (1, 3), lmoe.FORCE_WS_PAIR: (4, 4),
            lmoe.FORCE_NOPAIR: (1, 1), lmoe.FORCE_SIMT: (0, 0), lmoe.LOAD_SPLIT: (5, 5)}[flags]
    assert paths(res) == want


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_weight_stationary_pairs_on_skewed_loads(act):
    """Router bias that spreads the experts' loads from ~T/2 rows down to none:
    experts with one tile, several tiles of nearly equal size (including
    loads just past 128 and 256 rows), single rows and no rows; a feature
    count that ends inside a CTA's half of the 256-feature tile."""
    w = W_("ws-skew", T=1100, d=256, l=192, N=16, k=4, m=320, act=act, shared_m=0, seed=23)
    W = workloads.make_weights(w, device="cuda")
    b = torch.linspace(3.0, -3.0, w.N, device="cuda")
    b[-1] = -40.0  # never chosen
    W["bias"] = b
    res = check_forward(w, W=W, flags=lmoe.FORCE_WS_PAIR, fixture=True,
                        tokens=sample_tokens(w.T, 300, seed=2))
    assert paths(res) == (4, 4)
    L, _ = gpu_layer(w, lmoe.FORCE_WS_PAIR, W)
    x = workloads.make_x(w, device="cuda")
    L.forward(x)
    torch.cuda.synchronize()
    off = L.debug_dump("offsets", w.T).cpu().numpy()
    loads = np.diff(off)
    assert loads[-1] == 0 and loads.max() > 256 and ((loads > 128) & (loads < 256)).any()


@pytest.mark.parametrize("name", ["swiglu", "relu2-shared", "skip"])
@pytest.mark.parametrize("flags", [lmoe.SORTED_ROWS, lmoe.SORTED_ROWS | lmoe.LOAD_SPLIT,
                                   lmoe.SORTED_ROWS | lmoe.FORCE_SWAP,
                                   lmoe.SORTED_ROWS | lmoe.FORCE_WS_PAIR])
def test_sorted_fc1_rows_each_expert_kernel(name, flags):
    """LMOE_SORTED_ROWS: the FC1 input rows copied into expert order, FC1 on
    the TMA-fed variants of every expert kernel."""
    res = check_forward(SMALL[name], flags=flags, fixture=True)
    want = {lmoe.SORTED_ROWS: (1, 3), lmoe.SORTED_ROWS | lmoe.LOAD_SPLIT: (5, 5),
            lmoe.SORTED_ROWS | lmoe.FORCE_SWAP: (2, 2),
            lmoe.SORTED_ROWS | lmoe.FORCE_WS_PAIR: (4, 4)}[flags]
    assert paths(res) == want


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
@pytest.mark.parametrize("sorted_rows", [False, True])
def test_load_split_on_skewed_loads(act, sorted_rows):
    """The token-tiled expert GEMMs split by load (LMOE_LOAD_SPLIT) on loads
    from ~T/2 rows down to none: experts above 384 rows on CTA pairs (several 256-row tiles, a ragged
    last tile, FC1 rows gathered by token in both CTAs), the others on
    weight-stationary tiles of their rows (several tiles past 128 / 256
    rows); an expert with no rows in either kernel."""
    w = W_("split-skew", T=1100, d=256, l=192, N=16, k=4, m=320, act=act, shared_m=0, seed=24)
    W = workloads.make_weights(w, device="cuda")
    b = torch.linspace(3.0, -3.0, w.N, device="cuda")
    b[-1] = -40.0  # never chosen
    W["bias"] = b
    L, _ = gpu_layer(w, lmoe.LOAD_SPLIT | (lmoe.SORTED_ROWS if sorted_rows else 0), W)
    x = workloads.make_x(w, device="cuda")
    res = check_forward(w, W=W, layer=L, x=x, fixture=True, tokens=sample_tokens(w.T, 300, seed=3))
    assert paths(res) == (5, 5)
    loads = np.diff(L.debug_dump("offsets", w.T).cpu().numpy())
    print("loads", loads.tolist())
    assert loads[-1] == 0 and loads.max() > 512
    assert ((loads > 0) & (loads <= 128)).any() and ((loads > 128) & (loads <= 384)).any()


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_fc2_split_on_skewed_loads(act):
    """LMOE_FC2_SPLIT: an expert's rows past its whole 256-row tiles of the
    expert FC2, when at most 128, on one 128-row single-CTA tile, the rest on
    CTA pairs (loads from ~T/2 rows down to none: several whole tiles,
    remainders on either side of 128, experts below 256 rows)."""
    w = W_("fc2-split", T=1100, d=256, l=192, N=16, k=4, m=320, act=act, shared_m=0, seed=26)
    W = workloads.make_weights(w, device="cuda")
    b = torch.linspace(3.0, -3.0, w.N, device="cuda")
    b[-1] = -40.0  # never chosen
    W["bias"] = b
    L, _ = gpu_layer(w, lmoe.FC2_SPLIT, W)
    x = workloads.make_x(w, device="cuda")
    res = check_forward(w, W=W, layer=L, x=x, fixture=True, tokens=sample_tokens(w.T, 300, seed=4))
    assert paths(res) == (1, 3)
    loads = np.diff(L.debug_dump("offsets", w.T).cpu().numpy())
    assert loads[-1] == 0 and loads.max() > 512
    assert ((loads > 0) & (loads < 256)).any() and (loads % 256 != 0).any()
    # the same layer without the split: the same routing, outputs within the
    # bf16 tolerance (the remainder rows run through other MMA shapes)
    L2, _ = gpu_layer(w, 0, W)
    a, b2 = L.forward(x), L2.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(L.debug_dump("idx", w.T), L2.debug_dump("idx", w.T))
    err = (a.double() - b2.double()).abs()
    assert float(err.max()) <= 2e-2 + float(b2.double().abs().max()) * 2 ** -7


def test_fc2_split_full_size_skewed():
    """LMOE_FC2_SPLIT on latent-prefill-skewed at full size, sampled tokens
    plus the first and last tokens of the most loaded experts."""
    w = workloads.WORKLOADS["latent-prefill-skewed"]
    L, W = gpu_layer(w, lmoe.FC2_SPLIT)
    x = workloads.make_x(w, device="cuda")
    L.forward(x)
    torch.cuda.synchronize()
    toks = np.unique(np.concatenate([sample_tokens(w.T, 32, seed=w.seed + 1),
                                     edge_tokens_of_largest_experts(L, w.T)])).astype(np.int32)
    res = check_forward(w, tokens=toks, layer=L, W=W, x=x)
    assert res["unique"] >= 0.8 * res["tokens"]
    assert paths(res) == (1, 3)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("act", ["swiglu", "relu2"])
def test_stream_k_decode_tiles(act):
    """The weight-stationary decode FC1 with 2 to 16 tiles per CTA takes the
    stream-K split (tiles straddling two CTAs' ranges summed from two fp32
    parts): parity with the oracle, bitwise the same over repeated forwards,
    and within the tolerance of the whole-tile path (LMOE_NO_STREAM_K)."""
    w = W_("streamk", T=256, d=256, l=512, N=80, k=4, m=512, act=act, seed=25)
    W = workloads.make_weights(w, device="cuda")
    L, _ = gpu_layer(w, 0, W)
    x = workloads.make_x(w, device="cuda")
    res = check_forward(w, W=W, layer=L, x=x, fixture=True)
    assert paths(res) == (2, 2)
    a = L.forward(x).clone()
    b = L.forward(x).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    L2, _ = gpu_layer(w, lmoe.NO_STREAM_K, W)
    res2 = check_forward(w, W=W, layer=L2, x=x, fixture=True)
    assert paths(res2) == (2, 2)
    c = L2.forward(x)
    torch.cuda.synchronize()
    # the two paths split some tiles' K sums differently: within the stated
    # tolerance plus one bf16 step of the output
    ad, cd = a.double().cpu(), c.double().cpu()
    step = torch.exp2(torch.floor(torch.log2(cd.abs().clamp_min(2.0 ** -100))) - 7)
    assert bool(((ad - cd).abs() <= 2e-2 + step).all())
    assert L.last_error() == (lmoe.OK, 0) and L2.last_error() == (lmoe.OK, 0)


def test_pair_kernels_on_dense_prefill_shapes():
    """T >= 1024 puts the dense GEMMs (router, down-projection, shared FC1,
    up-projection) on CTA pairs as well as the expert GEMMs; ragged last row
    tile."""
    w = W_("pair-dense", T=1100, d=256, l=192, N=16, k=4, m=320, act="swiglu", shared_m=256,
           seed=22)
    res = check_forward(w, fixture=True, tokens=sample_tokens(w.T, 200, seed=1))
    assert paths(res) == (1, 3)
    res = check_forward(w, flags=lmoe.LOAD_SPLIT, fixture=True,
                        tokens=sample_tokens(w.T, 200, seed=1))
    assert paths(res) == (5, 5)
    res = check_forward(w, flags=lmoe.FORCE_WS_PAIR, fixture=True,
                        tokens=sample_tokens(w.T, 200, seed=1))
    assert paths(res) == (4, 4)
    res = check_forward(w, flags=lmoe.FORCE_NOPAIR, fixture=True,
                        tokens=sample_tokens(w.T, 200, seed=1))
    assert paths(res) == (1, 1)


@pytest.mark.parametrize("skip", [False, True])
def test_split_k_dense_gemms_at_decode_size(skip):
    """Few tokens and long K: the router, down-projection, gated shared FC1
    (with its hi/lo split) and up-projection run as split-K GEMMs whose fp32
    partial slices are summed in a fixed order; the projection-skip layer
    also sends its fp32 shared-expert output through the split."""
    w = W_("split", T=40, d=1024, l=1024 if skip else 512, N=16, k=4, m=128, act="swiglu",
           shared_m=256, skip_proj=skip, bias="normal0.5", seed=31)
    res = check_forward(w, fixture=True)
    assert res["unique"] >= 0.9 * res["tokens"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    a = L.forward(x)
    b = L.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# the x-only stages on a second stream
# ---------------------------------------------------------------------------

SIDE = {
    # split-K dense GEMMs on both streams at once (router on the caller's
    # stream; down-projection and gated shared FC1 on the side stream)
    "split": W_("side-split", T=40, d=1024, l=512, N=16, k=4, m=128, act="swiglu",
                shared_m=256, bias="normal0.5", seed=31),
    # projection-skip layer: the side stream carries the shared FC1 and its
    # fp32 FC2, which the combine adds
    "skip": W_("side-skip", T=40, d=1024, l=1024, N=16, k=4, m=128, act="swiglu",
               shared_m=256, skip_proj=True, seed=32),
    # CTA-pair dense GEMMs on both streams, ragged last row tile
    "pairs": W_("side-pairs", T=1100, d=256, l=192, N=16, k=4, m=320, act="relu2",
                shared_m=256, seed=33),
    # no shared expert: only the down-projection moves
    "no-shared": W_("side-noshared", T=300, d=256, l=128, N=8, k=3, m=192, act="swiglu",
                    seed=34),
}


@pytest.mark.parametrize("name", list(SIDE))
def test_side_stream_matches_single_stream(name):
    """By default the down-projection and the shared FC1 run on a second
    stream beside the router and routing steps; LMOE_SINGLE_STREAM keeps
    every stage on the caller's stream.  The two orders give bitwise the same
    output, also over back-to-back forwards with no synchronisation between
    them, and the default order matches the oracle."""
    w = SIDE[name]
    res = check_forward(w, fixture=True, tokens=sample_tokens(w.T, 200, seed=3))
    assert res["unique"] >= 0.9 * res["tokens"]
    W = workloads.make_weights(w, device="cuda")
    A, _ = gpu_layer(w, 0, W)
    B, _ = gpu_layer(w, lmoe.SINGLE_STREAM, W)
    x0 = workloads.make_x(w, device="cuda").float()
    xs = [(x0 * (1.0 + 0.5 * i)).roll(3 * i, dims=0).to(torch.bfloat16).contiguous()
          for i in range(3)]
    outs_a = [A.forward(x) for x in xs]  # enqueued back to back
    outs_b = [B.forward(x) for x in xs]
    torch.cuda.synchronize()
    for a, b in zip(outs_a, outs_b):
        assert torch.equal(a, b)
    assert A.last_error() == (lmoe.OK, 0) and B.last_error() == (lmoe.OK, 0)


@pytest.mark.parametrize("name", ["split", "pairs"])
def test_programmatic_launch_matches_plain_launches(name):
    """Kernels launched with programmatic dependent launch (the default)
    start while their predecessor drains and wait for its writes before
    touching global memory; LMOE_NO_PDL launches each after its predecessor
    has finished.  Back-to-back forwards give bitwise the same outputs."""
    w = SIDE[name]
    W = workloads.make_weights(w, device="cuda")
    A, _ = gpu_layer(w, 0, W)
    B, _ = gpu_layer(w, lmoe.NO_PDL | lmoe.SINGLE_STREAM, W)
    x0 = workloads.make_x(w, device="cuda").float()
    xs = [(x0 * (1.0 - 0.3 * i)).roll(5 * i, dims=0).to(torch.bfloat16).contiguous()
          for i in range(3)]
    outs_a = [A.forward(x) for x in xs]
    outs_b = [B.forward(x) for x in xs]
    torch.cuda.synchronize()
    for a, b in zip(outs_a, outs_b):
        assert torch.equal(a, b)
    assert A.last_error() == (lmoe.OK, 0) and B.last_error() == (lmoe.OK, 0)


@pytest.mark.parametrize("stage", ["expert_fc1", "down_proj", "group"])
def test_profile_selected_stages(stage):
    """Profiling one stage records only its two boundaries (a side-stream
    stage's on the side stream); the forward's output is unchanged."""
    w = SIDE["pairs"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    ref = L.forward(x)
    L.profile_begin(3, stages=[stage])
    outs = [L.forward(x) for _ in range(3)]
    prof = L.profile_end()
    assert len(prof) == 3
    for p, o in zip(prof, outs):
        assert list(p) == [stage] and p[stage] > 0
        assert torch.equal(o, ref)
    assert L.last_error() == (lmoe.OK, 0)


def test_profile_stage_mask_errors():
    """A stage mask without a stage bit, or no forwards, is rejected before
    anything is recorded; an unknown stage name is rejected by the binding."""
    w = SIDE["no-shared"]
    L, W = gpu_layer(w)
    lib = lmoe.lib()
    assert lib.lmoe_profile_begin_stages(L._h, 2, 0) == lmoe.ERR_INVALID_ARG
    assert lib.lmoe_profile_begin_stages(L._h, 2, 1 << 12) == lmoe.ERR_INVALID_ARG
    assert lib.lmoe_profile_begin_stages(L._h, 0, 1) == lmoe.ERR_INVALID_ARG
    with pytest.raises(ValueError):
        L.profile_begin(2, stages=["no_such_stage"])
    x = workloads.make_x(w, device="cuda")
    L.forward(x)
    torch.cuda.synchronize()
    assert L.last_error() == (lmoe.OK, 0)


def test_side_stream_profile_stages():
    """Profiled forwards time the side stream's two stages on that stream:
    every stage time is non-negative and the down-projection and shared FC1
    are not empty."""
    w = SIDE["pairs"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    L.profile_begin(2)
    for _ in range(2):
        L.forward(x)
    prof = L.profile_end()
    assert len(prof) == 2
    for p in prof:
        assert all(v >= 0 for v in p.values())
        assert p["down_proj"] > 0 and p["shared_fc1"] > 0


# ---------------------------------------------------------------------------
# fp8 E4M3 expert weights (codes + per-output-channel scales)
# ---------------------------------------------------------------------------

FP8 = {
    "swiglu": W_("f8-swiglu", T=300, d=256, l=128, N=8, k=3, m=192, act="swiglu", seed=41,
                 expert_fp8=True),
    "relu2-shared": W_("f8-relu2", T=260, d=256, l=192, N=6, k=2, m=320, act="relu2",
                       shared_m=320, bias="normal0.5", seed=42, expert_fp8=True),
    "silu-skip": W_("f8-silu-skip", T=90, d=128, l=128, N=12, k=4, m=64, act="silu",
                    skip_proj=True, seed=43, expert_fp8=True),
}


@pytest.mark.parametrize("name", list(FP8))
@pytest.mark.parametrize("flags", [0, lmoe.FORCE_SWAP, lmoe.FORCE_NOSWAP])
def test_fp8_experts(name, flags):
    """E4M3 expert weights widened to f16 inside the tensor-core kernels and
    scaled per output channel in the epilogue, against the oracle reading
    the same codes: FC1 weight-stationary or token-tiled by size with FC2 on
    token tiles (default), both weight-stationary (2, 2), both token-tiled
    (1, 1)."""
    res = check_forward(FP8[name], flags=flags, fixture=True)
    assert res["unique"] >= 0.9 * res["tokens"]
    fc1, fc2 = paths(res)
    assert fc1 in (1, 2)
    want = {0: (fc1, 1), lmoe.FORCE_SWAP: (2, 2), lmoe.FORCE_NOSWAP: (1, 1)}[flags]
    assert (fc1, fc2) == want


def test_fp8_experts_prefill_sized():
    """fp8 weights on the token-tiled kernel over many waves of tiles (256
    rows per expert, several feature tiles), the E4M3 slot ring cycling."""
    w = W_("f8-prefill", T=2048, d=1024, l=512, N=32, k=4, m=512, act="swiglu",
           shared_m=512, seed=44, expert_fp8=True)
    res = check_forward(w, tokens=sample_tokens(w.T, 160, seed=3))
    assert paths(res) == (1, 1)
    assert res["unique"] >= 0.8 * res["tokens"]


def test_ws_pair_prefill_sized():
    """The opt-in weight-stationary CTA-pair kernel at ~500 rows per expert
    (several nearly equal N tiles per expert, every K block, full feature
    tiles)."""
    w = W_("wsp-prefill", T=2048, d=512, l=512, N=16, k=4, m=512, act="swiglu", seed=45)
    res = check_forward(w, flags=lmoe.FORCE_WS_PAIR, tokens=sample_tokens(w.T, 160, seed=4))
    assert paths(res) == (4, 4)


def test_fp8_expert_api_errors():
    w = FP8["swiglu"]
    with pytest.raises(lmoe.LmoeError):  # fp8 experts need a bf16 layer
        lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="f32",
                            flags=lmoe.EXPERTS_FP8)
    with pytest.raises(lmoe.LmoeError):  # K of the expert GEMMs a multiple of 64
        lmoe.LatentMoELayer(w.d, 96, w.N, w.k, w.m, act=w.act, dtype="bf16",
                            flags=lmoe.EXPERTS_FP8)
    W = workloads.make_weights(w, device="cuda")
    L = lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="bf16",
                            flags=lmoe.EXPERTS_FP8)
    L.set_weights(W["Wg"], W["bias"], W["Wdown"], W["Wup"], None, None, None, None)
    L.reserve(w.T)
    x = workloads.make_x(w, device="cuda")
    with pytest.raises(lmoe.LmoeError):  # not ready before the fp8 experts are set
        L.forward(x)
    L.set_expert_weights_fp8(W["W1q"], W["W1s"], W["W2q"], W["W2s"])
    L.forward(x)
    torch.cuda.synchronize()
    plain = lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="bf16")
    with pytest.raises(lmoe.LmoeError):  # the layer was not created for fp8 experts
        plain.set_expert_weights_fp8(W["W1q"], W["W1s"], W["W2q"], W["W2s"])


FP4 = {
    "swiglu": W_("f4-swiglu", T=300, d=256, l=512, N=8, k=3, m=512, act="swiglu", seed=51,
                 expert_fp4=True),
    "relu2-shared": W_("f4-relu2", T=200, d=512, l=512, N=6, k=2, m=1024, act="relu2",
                       shared_m=256, bias="normal0.5", seed=52, expert_fp4=True),
    "silu-skip": W_("f4-silu-skip", T=90, d=512, l=512, N=12, k=4, m=512, act="silu",
                    skip_proj=True, seed=53, expert_fp4=True),
    # decode-like: 64 experts x 8 weight tiles of FC1, 2 to 16 tiles per CTA
    # (stream-K), K = 1024 (exponent boxes at two offsets)
    "decode-like": W_("f4-decode", T=64, d=1024, l=1024, N=64, k=8, m=512, act="swiglu",
                      bias="normal0.5", seed=54, expert_fp4=True),
}


@pytest.mark.parametrize("name", list(FP4))
@pytest.mark.parametrize("flags", [0, lmoe.FORCE_SWAP])
def test_fp4_experts(name, flags):
    """MXFP4 expert weights (E2M1 codes, one power-of-two scale per 32
    inputs), against the oracle on the same codes and exponents: FC1 widened
    in tensor memory on the weight-stationary kernel, FC2 widened in shared
    memory on token tiles (default) or in tensor memory (FORCE_SWAP)."""
    res = check_forward(FP4[name], flags=flags, fixture=True)
    assert res["unique"] >= 0.9 * res["tokens"]
    assert paths(res) == ((2, 2) if flags else (2, 1))


def test_fp4_experts_prefill_sized():
    """fp4 weights at prefill size (the weight-stationary kernels tile up to
    64 rows of an expert at a time: several row tiles per expert)."""
    w = W_("f4-prefill", T=1024, d=512, l=512, N=16, k=4, m=512, act="swiglu",
           shared_m=512, seed=55, expert_fp4=True)
    res = check_forward(w, tokens=sample_tokens(w.T, 160, seed=5))
    assert paths(res) == (2, 1)
    assert res["unique"] >= 0.8 * res["tokens"]


@pytest.mark.parametrize("low", [True, False])
def test_fp4_extreme_block_exponents(low):
    """FC2 blocks at one end of the accepted exponent range: scales 2^-23 ..
    2^-21 (codes x scale are f16 subnormals) or 2^11 .. 2^13 (up to 6 x 2^13
    = 49152), and all-zero blocks in both matrices.  The combined rows are
    compared relatively (rel-L2 of the comb stage), so a widening that
    flushed or clipped these values fails even where the residual hides them
    in the output.  FC1 keeps its quantised exponents: its output is stored
    in f16, so scales that overflow f16 there are outside the layer's range
    whatever the widening does."""
    w = W_("f4-extreme", T=200, d=512, l=512, N=8, k=2, m=512, act="silu", seed=56,
           expert_fp4=True)
    W = workloads.make_weights(w, device="cuda")
    g = torch.Generator(device="cpu").manual_seed(7)
    base = 127 - 23 if low else 127 + 11
    W["W2e"] = (base + torch.randint(0, 3, W["W2e"].shape, generator=g)).to(torch.uint8).cuda()
    for key in ("W1q", "W2q"):  # all-zero blocks: 32 codes = 16 bytes of a row
        q = W[key].cpu()
        q[:, :3, 16:32] = 0
        W[key] = q.to("cuda")
    res = check_forward(w, W=W, fixture=True)
    assert res["unique"] >= 0.9 * res["tokens"]
    assert "comb_rel_l2" in res


def test_fp4_expert_api_errors():
    w = FP4["swiglu"]
    for kw in (dict(dtype="f32"), dict(l=384), dict(m=256)):  # bf16, l and m multiples of 512
        a = dict(d=w.d, l=w.l, m=w.m, dtype="bf16")
        a.update(kw)
        with pytest.raises(lmoe.LmoeError):
            lmoe.LatentMoELayer(a["d"], a["l"], w.N, w.k, a["m"], act=w.act, dtype=a["dtype"],
                                flags=lmoe.EXPERTS_FP4)
    with pytest.raises(lmoe.LmoeError):  # not with fp8
        lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="bf16",
                            flags=lmoe.EXPERTS_FP4 | lmoe.EXPERTS_FP8)
    W = workloads.make_weights(w, device="cuda")
    L = lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="bf16",
                            flags=lmoe.EXPERTS_FP4)
    L.set_weights(W["Wg"], W["bias"], W["Wdown"], W["Wup"], None, None, None, None)
    L.reserve(w.T)
    x = workloads.make_x(w, device="cuda")
    with pytest.raises(lmoe.LmoeError):  # not ready before the fp4 experts are set
        L.forward(x)
    bad = W["W1e"].clone()
    bad[0, 0, 0] = 127 + 14  # a scale of 2^14: 6 x 2^14 is no f16 value
    with pytest.raises(lmoe.LmoeError):
        L.set_expert_weights_fp4(W["W1q"], bad, W["W2q"], W["W2e"])
    L.set_expert_weights_fp4(W["W1q"], W["W1e"], W["W2q"], W["W2e"])
    L.forward(x)
    torch.cuda.synchronize()
    assert L.last_error() == (lmoe.OK, 0)
    L.ep_reserve(w.T * w.k)
    with pytest.raises(lmoe.LmoeError):  # no expert parallelism for fp4 layers
        L.ep_dispatch(x)
    plain = lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, dtype="bf16")
    with pytest.raises(lmoe.LmoeError):  # the layer was not created for fp4 experts
        plain.set_expert_weights_fp4(W["W1q"], W["W1e"], W["W2q"], W["W2e"])


def test_tcgen05_path_is_taken_for_bf16():
    res = check_forward(SMALL["swiglu"], fixture=True)
    assert paths(res)[0] in (1, 2, 4, 5)
    res = check_forward(SMALL["odd-K"], fixture=True)
    assert res["expert_path"] == 0


def test_single_token_and_empty_batch():
    w = SMALL["relu2-shared"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    check_forward(w, layer=L, W=W, x=x[:1].contiguous(), fixture=True)
    out = torch.empty((0, w.d), dtype=torch.bfloat16, device="cuda")
    L.forward(x[:0], out)  # T = 0 enqueues nothing
    with pytest.raises(lmoe.LmoeError):
        L.forward(workloads.make_x(w.with_T(w.T + 1), device="cuda"))


def test_forward_is_deterministic_and_host_entry_matches():
    w = SMALL["swiglu-shared"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    a = L.forward(x)
    b = L.forward(x)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    L.forward_host(xh, oh)
    torch.cuda.synchronize()
    assert torch.equal(oh, a.cpu())


def test_host_entry_back_to_back_calls():
    """Consecutive host-buffer calls alternate two staging slots and upload on
    a copy stream while the previous forward runs: four calls with different
    inputs and no synchronisation in between must each equal the device-buffer
    forward of their own input."""
    w = SMALL["relu2-shared"]
    L, W = gpu_layer(w)
    x0 = workloads.make_x(w, device="cuda").float()
    xs = [(x0 * (1.0 + 0.25 * i)).roll(i, dims=0).to(torch.bfloat16).contiguous()
          for i in range(4)]
    ref = [L.forward(x).cpu() for x in xs]
    torch.cuda.synchronize()
    xh = [x.cpu().pin_memory() for x in xs]
    oh = [torch.empty_like(h).pin_memory() for h in xh]
    for a, b in zip(xh, oh):
        L.forward_host(a, b)
    torch.cuda.synchronize()
    for i in range(4):
        assert torch.equal(oh[i], ref[i]), i
    assert L.last_error() == (lmoe.OK, 0)


def test_bounded_wait_gives_up_and_reports():
    """A device wait that nothing completes gives up after its limit, the
    error word reads LMOE_DEVERR_WAIT_TIMEOUT (status TIMEOUT), the word is
    cleared by reading it, and the context stays usable for a forward."""
    w = SMALL["swiglu"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    L.selftest_wait_timeout(50_000)  # 50 ms
    assert L.last_error() == (lmoe.ERR_TIMEOUT, lmoe.DEVERR_WAIT_TIMEOUT)
    assert L.last_error() == (lmoe.OK, 0)
    check_forward(w, layer=L, W=W, x=x, fixture=True)
    with pytest.raises(lmoe.LmoeError):
        L.selftest_wait_timeout(0)


def test_debug_checks_flag_non_finite_logits():
    """LMOE_DEBUG_CHECKS: a NaN or an infinite router logit fed to
    lmoe_route_only sets LMOE_DEVERR_NONFINITE in the device error word
    (status DEVICE), with every index still in range; the word is cleared by
    reading it, and finite logits leave it at 0.  Without the flag the same
    logits set nothing."""
    T, N, k = 96, 128, 8
    lg = workloads.make_logits(T, N, seed=31, ties=False)
    bad = lg.clone()
    bad[3, 7] = float("nan")
    bad[50, 0] = float("inf")
    L = lmoe.LatentMoELayer(64, 64, N, k, 64, act="silu", dtype="bf16", flags=lmoe.DEBUG_CHECKS)
    L.reserve(T)
    L.route_only(lg.cuda())
    assert L.last_error() == (lmoe.OK, 0)
    r = L.route_only(bad.cuda())
    assert L.last_error() == (lmoe.ERR_DEVICE, lmoe.DEVERR_NONFINITE)
    idx = r["idx"].cpu().numpy()
    assert idx.min() >= 0 and idx.max() < N
    assert L.last_error() == (lmoe.OK, 0)
    r = L.route_only(lg.cuda())  # finite again: the routing is the oracle's
    o_idx = oracle.route(lg.numpy(), k)[0]
    np.testing.assert_array_equal(r["idx"].cpu().numpy(), o_idx)
    assert L.last_error() == (lmoe.OK, 0)
    L2 = lmoe.LatentMoELayer(64, 64, N, k, 64, act="silu", dtype="bf16")
    L2.reserve(T)
    L2.route_only(bad.cuda())
    assert L2.last_error() == (lmoe.OK, 0)


def test_uniform_router_is_mean_of_experts():
    """W_g = 0, k = N: every token uses every expert with weight 1/N."""
    w = W_("uniform", T=64, d=128, l=64, N=4, k=4, m=64, act="relu2", seed=19)
    W = workloads.make_weights(w, device="cuda")
    W["Wg"] = torch.zeros_like(W["Wg"])
    res = check_forward(w, W=W, fixture=True)
    assert res["unique"] == res["tokens"]


def test_device_error_word_clean_and_profile():
    w = SMALL["swiglu"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    L.profile_begin(3)
    for _ in range(3):
        L.forward(x)
    prof = L.profile_end()
    assert len(prof) == 3 and all(v >= 0 for p in prof for v in p.values())
    assert L.last_error() == (lmoe.OK, 0)
    # router, top-k, grouping count and rank, down-projection, expert FC1,
    # expert FC2, combine, up-projection
    assert L.last_launch_count >= 8


# ---------------------------------------------------------------------------
# the five workloads at full size (sampled tokens for the large ones)
# ---------------------------------------------------------------------------

FULL_SAMPLES = {"tiny-fp32": 64, "std-moe-decode": 96, "latent-decode": 96,
                "latent-prefill-shared": 64, "latent-prefill-skewed": 48,
                "std-moe-decode-fp8": 96, "latent-decode-fp8": 96,
                "std-moe-decode-fp4": 96, "latent-decode-fp4": 96,
                "l-moe-eff-decode": 64, "l-moe-acc-decode": 64, "std-moe-prefill": 48,
                "l-moe-eff-prefill": 48, "l-moe-acc-prefill": 48, "std-moe-latency": 8,
                "l-moe-eff-latency": 8, "l-moe-acc-latency": 8}


def edge_tokens_of_largest_experts(L, T: int, n_experts: int = 2, per_end: int = 3):
    """Tokens in the first and last row tiles of the most loaded experts (rows
    within an expert are in ascending token order): the lowest and highest
    token indices routed to each of them."""
    idx = L.debug_dump("idx", T).cpu().numpy()
    loads = np.bincount(idx.ravel(), minlength=L.N)
    out = []
    for e in np.argsort(-loads, kind="stable")[:n_experts]:
        toks = np.nonzero((idx == e).any(axis=1))[0]
        out += toks[:per_end].tolist() + toks[-per_end:].tolist()
    return out


@pytest.mark.parametrize("name", workloads.WORKLOAD_ORDER)
def test_workload_full_size(name):
    w = workloads.WORKLOADS[name]
    toks = sample_tokens(w.T, FULL_SAMPLES[name], seed=w.seed)
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    L.forward(x)
    torch.cuda.synchronize()
    toks = np.unique(np.concatenate([toks, edge_tokens_of_largest_experts(L, w.T)])).astype(np.int32)
    res = check_forward(w, tokens=toks, layer=L, W=W, x=x)
    print(name, res)
    assert res["unique"] >= 0.8 * res["tokens"]
    if w.dtype == "bf16":
        assert paths(res)[0] in (1, 2, 4, 5)
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["swiglu-shared", "decode-like"])
def test_forward_captures_into_a_cuda_graph(name):
    """lmoe_forward enqueues only kernels, copies and cross-stream events (no
    allocation, no synchronisation), so a caller can capture it into a CUDA
    graph (side stream, programmatic dependent launch and split-K / stream-K
    included) and replay it: each replay equals the eager forward bit for
    bit, also on new inputs written into the captured input buffer."""
    w = SMALL["swiglu-shared"] if name == "swiglu-shared" else W_(
        "graph-decode", T=64, d=1024, l=512, N=64, k=8, m=512, act="swiglu",
        bias="normal0.5", seed=57)
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    x2 = workloads.make_x(W_(**{**w.__dict__, "seed": w.seed + 99}), device="cuda")
    ref1 = L.forward(x).clone()
    ref2 = L.forward(x2).clone()
    xin, out = x.clone(), torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on a side stream, as torch asks before capture
        L.forward(xin, out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        L.forward(xin, out)
    for src, ref in ((x, ref1), (x2, ref2), (x, ref1)):
        xin.copy_(src)
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert L.last_error() == (lmoe.OK, 0)
    del g
