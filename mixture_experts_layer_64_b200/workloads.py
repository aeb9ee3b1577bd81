"""Seeded synthetic workloads for the LatentMoE layer.

This module holds the five workload shapes and the seeded generator of their
inputs (token activations, router / projection / expert weights, router bias).
It contains none of the layer's arithmetic: both the CUDA library (through the
tests and the benchmark) and the CPU oracle consume the exact bytes it
produces, so the generator never affects parity.

Input recipe
------------
* ``x ~ N(0, 1)``.
* Every weight ``~ N(0, 1/fan_in)``, fan_in being the input width of the
  matrix: d for the router, the down-projection and the shared expert's first
  matrix; the latent width l for the expert FC1 and the up-projection; the
  expert width m for FC2; the shared width for the shared expert's second
  matrix.  In the standard-MoE shape (l = d, projections skipped) FC1 has
  fan_in d.
* Router bias (only where a workload asks for one): ``N(0, variance 0.5)`` for
  the latent decode shape; for the skewed prefill shape the log of a
  Zipf(s=1.1) law over experts ranked by index,
  ``b[e] = ln((e+1)^-1.1 / H_{N,1.1})``, computed in float64 and stored fp32.
* Storage: fp32 for the tiny shape, bf16 (round-to-nearest-even of the fp32
  draw) for the others; the bias is always fp32.
* Weights use the API layout ``[in, out]`` row-major (``y = x @ W``).  The
  SwiGLU FC1 matrix is ``[l, 2m]``: columns ``[0, m)`` feed the SiLU gate and
  columns ``[m, 2m)`` are the linear ("up") half.

Every tensor (and, for the expert stacks, every expert) draws from its own
``torch.Generator`` seeded by ``(workload seed, tensor id, expert)``, so a
tensor can be produced in pieces, on the CPU or on a CUDA device, and a subset
of experts can be regenerated without the rest.  Values drawn on different
device types differ (different Philox streams); any single run draws each
tensor once and hands the same bytes to both sides.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

ACTS = ("silu", "swiglu", "relu2")


@dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    l: int
    N: int
    k: int
    m: int
    act: str
    shared_m: int = 0
    dtype: str = "bf16"          # "f32" or "bf16"
    skip_proj: bool = False      # l == d and the two projections are identities
    bias: Optional[str] = None   # None, "normal0.5" or "zipf1.1"
    seed: int = 0
    expert_fp8: bool = False     # expert weights as E4M3 codes + per-channel scales
    expert_fp4: bool = False     # expert weights as MXFP4 (E2M1 codes + block exponents)

    @property
    def m_in(self) -> int:
        return 2 * self.m if self.act == "swiglu" else self.m

    @property
    def expert_format(self) -> Optional[str]:
        """The expert weights' low-precision format (costmodel.EXPERT_FORMATS)."""
        return "e4m3" if self.expert_fp8 else "mxfp4" if self.expert_fp4 else None

    @property
    def ms_in(self) -> int:
        return 2 * self.shared_m if self.act == "swiglu" else self.shared_m

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def with_T(self, T: int) -> "Workload":
        return replace(self, T=T)


# The five workloads: a tiny fp32 layer, the standard-MoE decode shape
# (projections skipped), the latent decode shape, latent prefill with a
# full-width shared expert, and high-sparsity skewed prefill.
WORKLOADS: Dict[str, Workload] = {
    "tiny-fp32": Workload("tiny-fp32", T=64, d=256, l=64, N=16, k=4, m=128,
                          act="silu", dtype="f32", seed=0),
    "std-moe-decode": Workload("std-moe-decode", T=256, d=4096, l=4096, N=128,
                               k=8, m=1536, act="swiglu", skip_proj=True,
                               seed=1),
    "latent-decode": Workload("latent-decode", T=256, d=4096, l=1024, N=512,
                              k=32, m=1536, act="swiglu", bias="normal0.5",
                              seed=2),
    "latent-prefill-shared": Workload("latent-prefill-shared", T=4096, d=4096,
                                      l=1024, N=512, k=22, m=2048,
                                      act="relu2", shared_m=3072, seed=3),
    "latent-prefill-skewed": Workload("latent-prefill-skewed", T=16384,
                                      d=7168, l=1792, N=896, k=16, m=1024,
                                      act="swiglu", bias="zipf1.1", seed=4),
}
# Low-precision expert weights (the paper's deployment lever at decode, where
# the expert weights are the traffic): the two decode shapes with E4M3 expert
# weights and per-channel scales, everything else as above.
WORKLOADS["std-moe-decode-fp8"] = replace(WORKLOADS["std-moe-decode"], name="std-moe-decode-fp8",
                                          expert_fp8=True)
WORKLOADS["latent-decode-fp8"] = replace(WORKLOADS["latent-decode"], name="latent-decode-fp8",
                                         expert_fp8=True)
# ... and with block-scaled FP4 expert weights (the precision of the paper's
# GB200 roofline analysis)
WORKLOADS["std-moe-decode-fp4"] = replace(WORKLOADS["std-moe-decode"], name="std-moe-decode-fp4",
                                          expert_fp4=True)
WORKLOADS["latent-decode-fp4"] = replace(WORKLOADS["latent-decode"], name="latent-decode-fp4",
                                         expert_fp4=True)
# The paper's two LatentMoE variants against the standard MoE they derive from
# (LatentMoE, Section 3, Eq. (1) and Eq. (2); Table 1): the standard layer
# (d = 4096, N = 128 experts, top-8, m = 1536, no projections), l-MoE_eff
# (latent l = d / 4, N' = 4 N, k' = k) and l-MoE_acc (l = d / 4, N' = 4 N,
# k' = 4 k), on the same kernels, at decode and prefill batches.  No router
# bias, so all three see the same routing statistics.  The standard decode
# point is std-moe-decode itself.
_SWEEP = dict(d=4096, m=1536, act="swiglu")
WORKLOADS["l-moe-eff-decode"] = Workload("l-moe-eff-decode", T=256, l=1024, N=512, k=8,
                                         seed=11, **_SWEEP)
WORKLOADS["l-moe-acc-decode"] = Workload("l-moe-acc-decode", T=256, l=1024, N=512, k=32,
                                         seed=12, **_SWEEP)
WORKLOADS["std-moe-prefill"] = Workload("std-moe-prefill", T=4096, l=4096, N=128, k=8,
                                        skip_proj=True, seed=13, **_SWEEP)
WORKLOADS["l-moe-eff-prefill"] = Workload("l-moe-eff-prefill", T=4096, l=1024, N=512, k=8,
                                          seed=14, **_SWEEP)
WORKLOADS["l-moe-acc-prefill"] = Workload("l-moe-acc-prefill", T=4096, l=1024, N=512, k=32,
                                          seed=15, **_SWEEP)
# ... and at a latency-bound batch of 8 tokens, where a step touches fewer
# experts than there are (the regime of the paper's per-token memory cost)
WORKLOADS["std-moe-latency"] = Workload("std-moe-latency", T=8, l=4096, N=128, k=8,
                                        skip_proj=True, seed=16, **_SWEEP)
WORKLOADS["l-moe-eff-latency"] = Workload("l-moe-eff-latency", T=8, l=1024, N=512, k=8,
                                          seed=17, **_SWEEP)
WORKLOADS["l-moe-acc-latency"] = Workload("l-moe-acc-latency", T=8, l=1024, N=512, k=32,
                                          seed=18, **_SWEEP)
# (batch, standard point, l-MoE_eff point, l-MoE_acc point) per batch size
VARIANT_SWEEP = (("latency", "std-moe-latency", "l-moe-eff-latency", "l-moe-acc-latency"),
                 ("decode", "std-moe-decode", "l-moe-eff-decode", "l-moe-acc-decode"),
                 ("prefill", "std-moe-prefill", "l-moe-eff-prefill", "l-moe-acc-prefill"))
WORKLOAD_ORDER = list(WORKLOADS)


def quantize_e4m3(W: torch.Tensor):
    """Per-output-column fp8 E4M3 quantisation of a weight stack in the API
    layout [..., in, out]: scale[..., o] = max_i |W[..., i, o]| / 448 (fp32,
    1 for an all-zero column) and codes = W / scale rounded to E4M3 by
    torch's float8_e4m3fn conversion.  Returns (codes uint8 [..., in, out],
    scales float32 [..., out]).  Inputs for the fp8 expert weights: the
    library and the oracle both read these codes and scales."""
    Wf = W.float()
    amax = Wf.abs().amax(dim=-2)
    scale = torch.where(amax > 0, amax / 448.0, torch.ones_like(amax))
    codes = (Wf / scale.unsqueeze(-2)).to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.contiguous()

# MXFP4: the eight magnitudes of an E2M1 code, and the midpoints between
# neighbours (a value on a midpoint goes to the neighbour whose code is even,
# i.e. whose mantissa bit is 0)
_E2M1_MIDPOINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)


def quantize_mxfp4(W: torch.Tensor):
    """Block-scaled FP4 (OCP MX: E2M1 elements, one E8M0 scale per 32
    elements) of a weight stack in the API layout [..., in, out], blocks of
    32 consecutive inputs of each output column.  Per block: scale exponent
    e = floor(log2(amax)) - 2 (2 = the largest E2M1 exponent; e = -23 for an
    all-zero block), clamped to [-23, 13] so that every scaled code is an f16
    value; elements round to nearest on the E2M1 grid, ties to the even code,
    saturating at 6.  Returns (codes uint8 [..., out, in / 2], element 2j in
    the low nibble of byte j; exponents uint8 [..., out, in / 32] = e + 127),
    output-major as the kernels read them.  Inputs for the fp4 expert
    weights: the library and the oracle both read these codes."""
    Wt = W.float().transpose(-1, -2)
    *lead, O, I = Wt.shape
    if I % 32:
        raise ValueError("the input width must be a multiple of 32")
    blk = Wt.reshape(*lead, O, I // 32, 32)
    amax = blk.abs().amax(dim=-1)
    e = torch.where(amax > 0, torch.floor(torch.log2(amax)) - 2, torch.full_like(amax, -23.0))
    e = e.clamp(-23.0, 13.0)
    v = blk / torch.exp2(e).unsqueeze(-1)
    a = v.abs()
    mids = torch.tensor(_E2M1_MIDPOINTS, dtype=torch.float32, device=W.device)
    idx = torch.searchsorted(mids, a.contiguous(), right=False)  # midpoints strictly below a
    tie = (idx < 7) & (a == mids[idx.clamp(max=6)])
    idx = torch.where(tie & (idx % 2 == 1), idx + 1, idx)
    code = (idx | torch.where(v < 0, 8, 0)).to(torch.uint8).reshape(*lead, O, I)
    packed = (code[..., 0::2] | (code[..., 1::2] << 4)).contiguous()
    return packed, (e + 127).to(torch.uint8).contiguous()


_TID = {"x": 1, "Wg": 2, "bias": 3, "Wdown": 4, "Wup": 5, "W1": 6, "W2": 7,
        "Ws1": 8, "Ws2": 9}


def _gen(seed: int, tid: int, sub: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(((seed * 1_000_003 + tid) * 65_537 + sub) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, std: float, seed: int, tid: int, sub: int, device,
            dtype: torch.dtype) -> torch.Tensor:
    g = _gen(seed, tid, sub, device)
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def zipf_log_bias(N: int, s: float = 1.1) -> torch.Tensor:
    """ln of a Zipf(s) probability law over N experts ranked by index."""
    H = math.fsum((r + 1) ** -s for r in range(N))
    return torch.tensor([math.log(((e + 1) ** -s) / H) for e in range(N)],
                        dtype=torch.float64).to(torch.float32)


def make_bias(w: Workload, device="cpu") -> Optional[torch.Tensor]:
    if w.bias is None:
        return None
    if w.bias == "normal0.5":
        return _normal((w.N,), math.sqrt(0.5), w.seed, _TID["bias"], 0, device,
                       torch.float32)
    if w.bias == "zipf1.1":
        return zipf_log_bias(w.N, 1.1).to(device)
    raise ValueError(f"unknown bias recipe {w.bias!r}")


def make_x(w: Workload, device="cpu", T: Optional[int] = None) -> torch.Tensor:
    T = w.T if T is None else T
    return _normal((T, w.d), 1.0, w.seed, _TID["x"], 0, device, w.torch_dtype)


def make_expert_W1(w: Workload, e: int, device="cpu") -> torch.Tensor:
    return _normal((w.l, w.m_in), 1.0 / math.sqrt(w.l), w.seed, _TID["W1"], e,
                   device, w.torch_dtype)


def make_expert_W2(w: Workload, e: int, device="cpu") -> torch.Tensor:
    return _normal((w.m, w.l), 1.0 / math.sqrt(w.m), w.seed, _TID["W2"], e,
                   device, w.torch_dtype)


def make_weights(w: Workload, device="cpu", experts: bool = True) -> Dict[str, Optional[torch.Tensor]]:
    """All weights of one layer, API layout.  With ``experts=False`` the expert
    stacks W1/W2 are left out (use make_expert_W1/W2 per expert)."""
    dt = w.torch_dtype
    out: Dict[str, Optional[torch.Tensor]] = {}
    out["Wg"] = _normal((w.d, w.N), 1.0 / math.sqrt(w.d), w.seed, _TID["Wg"], 0,
                        device, dt)
    out["bias"] = make_bias(w, device)
    if w.skip_proj:
        out["Wdown"] = None
        out["Wup"] = None
    else:
        out["Wdown"] = _normal((w.d, w.l), 1.0 / math.sqrt(w.d), w.seed,
                               _TID["Wdown"], 0, device, dt)
        out["Wup"] = _normal((w.l, w.d), 1.0 / math.sqrt(w.l), w.seed,
                             _TID["Wup"], 0, device, dt)
    if experts and w.expert_fp4:
        # the same bf16 draws, as MXFP4 per expert, output-major: W1q [N, m_in,
        # l / 2] and W1e [N, m_in, l / 32], W2q [N, l, m / 2] and W2e [N, l, m / 32]
        W1q = torch.empty((w.N, w.m_in, w.l // 2), dtype=torch.uint8, device=device)
        W2q = torch.empty((w.N, w.l, w.m // 2), dtype=torch.uint8, device=device)
        W1e = torch.empty((w.N, w.m_in, w.l // 32), dtype=torch.uint8, device=device)
        W2e = torch.empty((w.N, w.l, w.m // 32), dtype=torch.uint8, device=device)
        for e in range(w.N):
            W1q[e], W1e[e] = quantize_mxfp4(make_expert_W1(w, e, device))
            W2q[e], W2e[e] = quantize_mxfp4(make_expert_W2(w, e, device))
        out.update(W1=None, W2=None, W1q=W1q, W1e=W1e, W2q=W2q, W2e=W2e)
    elif experts and w.expert_fp8:
        # the same bf16 draws, quantised per expert (W1q/W2q codes, W1s/W2s
        # scales); W1/W2 stay None
        W1q = torch.empty((w.N, w.l, w.m_in), dtype=torch.uint8, device=device)
        W2q = torch.empty((w.N, w.m, w.l), dtype=torch.uint8, device=device)
        W1s = torch.empty((w.N, w.m_in), dtype=torch.float32, device=device)
        W2s = torch.empty((w.N, w.l), dtype=torch.float32, device=device)
        for e in range(w.N):
            W1q[e], W1s[e] = quantize_e4m3(make_expert_W1(w, e, device))
            W2q[e], W2s[e] = quantize_e4m3(make_expert_W2(w, e, device))
        out.update(W1=None, W2=None, W1q=W1q, W1s=W1s, W2q=W2q, W2s=W2s)
    elif experts:
        W1 = torch.empty((w.N, w.l, w.m_in), dtype=dt, device=device)
        W2 = torch.empty((w.N, w.m, w.l), dtype=dt, device=device)
        for e in range(w.N):
            W1[e] = make_expert_W1(w, e, device)
            W2[e] = make_expert_W2(w, e, device)
        out["W1"] = W1
        out["W2"] = W2
    if w.shared_m:
        out["Ws1"] = _normal((w.d, w.ms_in), 1.0 / math.sqrt(w.d), w.seed,
                             _TID["Ws1"], 0, device, dt)
        out["Ws2"] = _normal((w.shared_m, w.d), 1.0 / math.sqrt(w.shared_m),
                             w.seed, _TID["Ws2"], 0, device, dt)
    else:
        out["Ws1"] = None
        out["Ws2"] = None
    return out


def make_logits(T: int, N: int, seed: int, bias: Optional[torch.Tensor] = None,
                ties: bool = True, device="cpu") -> torch.Tensor:
    """fp32 router logits for routing-only tests: N(0,1) plus an optional bias,
    with exact ties, signed zeros and repeated values planted in some rows."""
    g = _gen(seed, 100, 0, "cpu")
    lg = torch.randn((T, N), generator=g, dtype=torch.float32)
    if bias is not None:
        lg += bias.to("cpu", torch.float32)[None, :]
    if ties and T > 0:
        r = torch.randint(0, 4, (T,), generator=g)
        for t in range(T):
            if r[t] == 0:      # a block of identical values
                c = torch.randint(0, N, (max(2, N // 4),), generator=g)
                lg[t, c] = lg[t, c[0]].item()
            elif r[t] == 1:    # +0.0 and -0.0 mixed with exact zeros
                c = torch.randint(0, N, (max(2, N // 3),), generator=g)
                sign = torch.randint(0, 2, (c.numel(),), generator=g)
                lg[t, c] = torch.where(sign == 0, torch.tensor(0.0), torch.tensor(-0.0))
            elif r[t] == 2:    # an entire row of one value
                lg[t, :] = 0.25
    return lg.to(device)
