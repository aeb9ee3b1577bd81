"""lmoe_route_only_noalloc: the routing entry point for callers that cannot
allocate device memory (an inference server that owns all of HBM through its
own pool, or code where cudaMalloc's implicit synchronisation is not allowed).

It must give what lmoe_route_only gives (bit-exact indices, offsets and
permutation; gates within the routing tolerance), and what the CPU oracle's
routing gives, call after call, with its scratch in the library's fixed
device array: a second call must see no stale state from the first, and must
not change the device's free memory.  With an error word it runs the device
checks and reports a non-finite logit there.  The file is named to be
collected last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_64_b200 import lmoe, workloads

pytestmark = pytest.mark.gpu


def _outputs(T: int, N: int, k: int, dev):
    return {"idx": torch.full((T, k), -1, dtype=torch.int32, device=dev),
            "w": torch.full((T, k), -1.0, dtype=torch.float32, device=dev),
            "offsets": torch.full((N + 1,), -1, dtype=torch.int32, device=dev),
            "perm": torch.full((T * k,), -1, dtype=torch.int32, device=dev)}


def _noalloc_via_cabi(logits: torch.Tensor, k: int, out=None, word=None):
    """Calls the entry point through the C ABI on caller-owned outputs."""
    T, N = logits.shape
    if out is None:
        out = _outputs(T, N, k, logits.device)
    p = lambda t: ctypes.c_void_p(None if t is None else t.data_ptr())
    st = lmoe.lib().lmoe_route_only_noalloc(p(logits), T, N, k, p(out["idx"]), p(out["w"]),
                                            p(out["offsets"]), p(out["perm"]), p(word),
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, out


def _with_handle(logits: torch.Tensor, k: int):
    T, N = logits.shape
    L = lmoe.LatentMoELayer(64, 64, N, k, 64, act="silu", dtype="bf16")
    L.reserve(T)
    r = L.route_only(logits)
    torch.cuda.synchronize()
    return L, r


def _same(a, b):
    for key in ("idx", "offsets", "perm"):
        np.testing.assert_array_equal(a[key].cpu().numpy(), b[key].cpu().numpy(), err_msg=key)
    np.testing.assert_allclose(a["w"].cpu().numpy(), b["w"].cpu().numpy(), rtol=2e-6, atol=1e-7)


def test_noalloc_matches_route_only_on_two_calls_in_a_row():
    torch.cuda.set_device(0)
    # two different problems back to back: the second call must not see the
    # first call's bits, counters or offsets in the shared scratch array
    cases = [(300, 896, 16, 1), (1000, 128, 8, 2)]
    handles = []
    refs = []
    for T, N, k, seed in cases:
        lg = workloads.make_logits(T, N, seed, ties=True).cuda()
        L, r = _with_handle(lg, k)
        handles.append(L)
        refs.append((lg, k, r))
    torch.cuda.synchronize()
    for i, (lg, k, ref) in enumerate(refs):
        out = _outputs(lg.shape[0], lg.shape[1], k, lg.device)  # the caller's memory, first
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        st, got = _noalloc_via_cabi(lg, k, out)
        free_after = torch.cuda.mem_get_info()[0]
        torch.cuda.synchronize()
        assert st == lmoe.OK, lmoe.status_string(st)
        _same(got, ref)
        if i > 0:  # set-up (symbol lookup, module load) happened on the first call
            assert free_after == free_before
    # and once more with the first problem again, after the second
    lg, k, ref = refs[0]
    st, got = _noalloc_via_cabi(lg, k)
    torch.cuda.synchronize()
    assert st == lmoe.OK
    _same(got, ref)


def test_noalloc_matches_the_oracle_routing():
    torch.cuda.set_device(0)
    T, N, k = 257, 512, 22
    lg = workloads.make_logits(T, N, seed=5, ties=True)
    st, got = _noalloc_via_cabi(lg.cuda(), k)
    torch.cuda.synchronize()
    assert st == lmoe.OK
    o_idx, o_w, o_off, o_perm = oracle.route(lg.numpy(), k)
    np.testing.assert_array_equal(got["idx"].cpu().numpy(), o_idx)
    np.testing.assert_array_equal(got["offsets"].cpu().numpy(), o_off)
    np.testing.assert_array_equal(got["perm"].cpu().numpy(), o_perm)
    np.testing.assert_allclose(got["w"].cpu().numpy(), o_w, rtol=2e-6, atol=1e-7)


def test_noalloc_error_word_reports_a_non_finite_logit():
    torch.cuda.set_device(0)
    T, N, k = 64, 128, 8
    lg = workloads.make_logits(T, N, seed=9, ties=False).cuda()
    word = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st, got = _noalloc_via_cabi(lg, k, word=word)
    torch.cuda.synchronize()
    assert st == lmoe.OK and int(word.item()) == 0  # cleared by the call, nothing flagged
    bad = lg.clone()
    bad[5, 17] = float("nan")
    st, got = _noalloc_via_cabi(bad, k, word=word)
    torch.cuda.synchronize()
    assert st == lmoe.OK
    assert int(word.item()) & lmoe.DEVERR_NONFINITE
    idx = got["idx"].cpu().numpy()
    assert idx.min() >= 0 and idx.max() < N  # indices stay in range
    # the next clean call clears the word again
    st, _ = _noalloc_via_cabi(lg, k, word=word)
    torch.cuda.synchronize()
    assert st == lmoe.OK and int(word.item()) == 0


def test_noalloc_rejects_sizes_beyond_its_scratch():
    torch.cuda.set_device(0)
    N = 1024
    T = 32 * (lmoe.NOALLOC_MAX_WORDS // N) + 1  # one word per expert too many
    lg = torch.zeros((T, N), dtype=torch.float32, device="cuda")
    st, out = _noalloc_via_cabi(lg, 4)
    torch.cuda.synchronize()
    assert st == lmoe.ERR_UNSUPPORTED
    assert torch.all(out["offsets"] == -1)  # nothing was enqueued
    st, _ = _noalloc_via_cabi(torch.zeros((8, 16), device="cuda"), 17)  # k > N
    assert st == lmoe.ERR_INVALID_ARG
