"""Expert parallelism on one GPU: `world` ranks emulated in one process (each
with its own handle and tokens; the all-to-alls replaced by copies between
their buffers, so no kernel waits for another rank).  Each rank's output
through dispatch -> exchange -> experts -> return -> combine must match
lmoe_forward on the same tokens (which the other tests check against the
CPU oracle), within the bf16 tolerance, and its own routing bit for bit.
(LatentMoE, Section 2.2 and the paragraph after Eq. (1): dispatch and
combine in the latent width.)"""
import numpy as np
import pytest
import torch

from mixture_experts_layer_64_b200 import lmoe, workloads
from parity import gpu_layer

pytestmark = pytest.mark.gpu

W_ = workloads.Workload


def _emulated_ep(w, world, flags=0):
    W = workloads.make_weights(w, device="cuda")
    n = w.N // world
    layers, xs, refs = [], [], []
    for r in range(world):
        L, _ = gpu_layer(w, flags, W)
        L.ep_reserve(world * w.T * w.k)
        x = workloads.make_x(workloads.Workload(**{**w.__dict__, "seed": w.seed + 17 * r}),
                             device="cuda")
        refs.append(L.forward(x).clone())
        ref_idx = L.debug_dump("idx", w.T).clone()
        layers.append((L, ref_idx))
        xs.append(x)
    # 1: dispatch on every rank
    sends = [L.ep_dispatch(x) for (L, _), x in zip(layers, xs)]
    torch.cuda.synchronize()
    counts = [c.cpu().numpy() for _, _, c in sends]
    # 2: the exchange (sources in rank order)
    recv = []
    for q in range(world):
        rows, gates, rc = [], [], []
        for s in range(world):
            srows, sgates, _ = sends[s]
            start = int(counts[s][:q * n].sum())
            cnt = int(counts[s][q * n:(q + 1) * n].sum())
            rows.append(srows[start:start + cnt])
            gates.append(sgates[start:start + cnt])
            rc.append(counts[s][q * n:(q + 1) * n])
        recv.append((torch.cat(rows), torch.cat(gates), np.stack(rc)))
    # 3: the experts on every rank
    outs = [layers[q][0].ep_experts(rr, rg, rc, q, world) for q, (rr, rg, rc) in enumerate(recv)]
    # 4: the return trip, each source's rows in its send order
    backs = []
    for s in range(world):
        parts = []
        for q in range(world):
            before = int(sum(recv[q][2][s2].sum() for s2 in range(s)))
            cnt = int(recv[q][2][s].sum())
            parts.append(outs[q][before:before + cnt])
        backs.append(torch.cat(parts))
    # 5: combine
    results = [L.ep_combine(x, b) for (L, _), x, b in zip(layers, xs, backs)]
    torch.cuda.synchronize()
    for (L, ref_idx), res, ref in zip(layers, results, refs):
        assert torch.equal(L.debug_dump("idx", w.T), ref_idx)  # the same routing
        assert L.last_error() == (lmoe.OK, 0)
    return results, refs


def _close(res, ref, tol=2e-2):
    """Within the stated bf16 tolerance of lmoe_forward's output, plus one
    bf16 step of the output (2^(floor(log2|ref|) - 7)): the expert GEMMs of
    the two paths may split a tile's K sum differently, and a last-bit
    difference in a bf16 intermediate can move the stored output by one
    step (0.03125 in [4, 8))."""
    a, b = res.double().cpu(), ref.double().cpu()
    err = (a - b).abs()
    step = torch.exp2(torch.floor(torch.log2(b.abs().clamp_min(2.0 ** -100))) - 7)
    assert bool((err <= tol + step).all()), float((err - step).max())
    assert float(torch.linalg.norm(a - b) / torch.linalg.norm(b)) <= 5e-3


EP = {
    "latent-swiglu": W_("ep-swiglu", T=200, d=256, l=128, N=16, k=4, m=192, act="swiglu",
                        seed=41),
    "latent-relu2-shared": W_("ep-relu2", T=150, d=256, l=192, N=12, k=3, m=256, act="relu2",
                              shared_m=256, seed=42),
    "skip": W_("ep-skip", T=120, d=256, l=256, N=8, k=2, m=128, act="swiglu", skip_proj=True,
               seed=43),
    "decode-like": W_("ep-decode", T=64, d=512, l=256, N=64, k=8, m=256, act="swiglu",
                      bias="normal0.5", seed=44),
}


@pytest.mark.parametrize("world", [1, 2, 4])
@pytest.mark.parametrize("name", list(EP))
def test_expert_parallel_matches_forward(name, world):
    w = EP[name]
    if w.N % world:
        pytest.skip("experts do not split")
    results, refs = _emulated_ep(w, world)
    for res, ref in zip(results, refs):
        _close(res, ref)


def test_expert_parallel_prefill_kernels():
    """Enough received rows per local expert for the token-tiled kernels
    (and the load split) on the expert side."""
    w = W_("ep-prefill", T=1100, d=256, l=192, N=8, k=4, m=320, act="swiglu", seed=45)
    for flags in (0, lmoe.LOAD_SPLIT):
        results, refs = _emulated_ep(w, 2, flags)
        for res, ref in zip(results, refs):
            _close(res, ref)


def test_expert_parallel_errors():
    w = EP["latent-swiglu"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    with pytest.raises(lmoe.LmoeError):  # no ep_reserve yet
        L.ep_experts(torch.zeros((16, w.l), dtype=torch.bfloat16, device="cuda"),
                     torch.zeros(16, device="cuda"), np.ones((1, w.N), dtype=np.int32), 0, 1)
    L.ep_reserve(8)
    with pytest.raises(lmoe.LmoeError):  # over the reserved rows
        L.ep_experts(torch.zeros((16, w.l), dtype=torch.bfloat16, device="cuda"),
                     torch.zeros(16, device="cuda"), np.ones((1, w.N), dtype=np.int32), 0, 1)
    with pytest.raises(lmoe.LmoeError):  # N % world != 0
        L.ep_experts(None, None, np.zeros((3, 5), dtype=np.int32), 0, 3)
    with pytest.raises(lmoe.LmoeError):  # combine without a dispatch
        L.ep_combine(x, torch.zeros((w.T * w.k, w.l), dtype=torch.bfloat16, device="cuda"))


def test_expert_parallel_layer_over_nccl_world_one():
    """ExpertParallelLayer through a real NCCL process group of one rank (the
    only size a one-GPU run can form; the gloo tests cover the exchange plan
    at world sizes 2 and 4): dispatch, the count and row all-to-alls, the
    experts and the combine equal lmoe_forward on the same tokens."""
    import os
    import socket
    import torch.distributed as dist
    from mixture_experts_layer_64_b200.ep import ExpertParallelLayer

    w = EP["latent-relu2-shared"]
    L, W = gpu_layer(w)
    x = workloads.make_x(w, device="cuda")
    ref = L.forward(x).clone()
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", torch.cuda.current_device()))
    try:
        ep_layer = ExpertParallelLayer(L, max_recv_rows=w.T * w.k)
        out = ep_layer(x)
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()
    _close(out, ref)
    assert L.last_error() == (lmoe.OK, 0)
