"""Analytic cost model of the LatentMoE layer: the paper's roofline formulas
and the algorithmic FLOP / byte counts the benchmark divides by.

Paper formulas (LatentMoE, arXiv 2601.18089):
* Section 2.1: the compute-bound threshold F / BW_HBM, the per-expert cost
  C_exp = 2 t d m and traffic M_exp = d m + t (d + m), and the arithmetic
  intensity I = 2 t d m / (d m + t (d + m)) (also the Figure 2 caption).
* Section 2.2: the communication / compute time ratio 5 F / (4 m BW_NVL).
* Table 1: the per-expert weight-loading cost d m (standard MoE) versus
  l m (LatentMoE).

Algorithmic counts (what the layer must compute and move at minimum, used for
the achieved-throughput figures): only the experts that at least one token
reaches have their weights read; every other tensor is read or written once;
the intermediates (latent rows, expert hidden rows, expert outputs, the
combined rows) are excluded and reported separately as overhead.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Sequence


# ---- the paper's closed forms ------------------------------------------------

def compute_bound_threshold(F: float, bw_hbm: float) -> float:
    """FLOPs per byte above which a kernel is compute bound (Section 2.1)."""
    return F / bw_hbm


def expert_cost(t_exp: float, d: float, m: float):
    """(C_exp, M_exp) for one expert fed t_exp tokens (Section 2.1)."""
    return 2.0 * t_exp * d * m, d * m + t_exp * (d + m)


def arithmetic_intensity(t_exp: float, d: float, m: float) -> float:
    """I = 2 t d m / (d m + t (d + m)) (Section 2.1, Figure 2)."""
    c, mem = expert_cost(t_exp, d, m)
    return c / mem


def threshold_tokens(I: float, d: float, m: float) -> float:
    """Smallest t_exp with arithmetic_intensity(t_exp, d, m) >= I; the root of
    2 t d m = I (d m + t (d + m))."""
    den = 2.0 * d * m - I * (d + m)
    if den <= 0:
        return float("inf")
    return I * d * m / den


def comm_compute_ratio(F: float, m: float, bw_nvl: float) -> float:
    """All-to-all time over expert compute time under expert parallelism with
    FP4 dispatch and BF16 combine (Section 2.2): 5 F / (4 m BW_NVL)."""
    return 5.0 * F / (4.0 * m * bw_nvl)


def weight_load_per_expert(width: float, m: float) -> float:
    """Weight-loading memory cost per expert (Table 1): d m for a standard
    MoE, l m for LatentMoE."""
    return width * m


# ---- algorithmic counts of one forward pass ----------------------------------

@dataclass
class LayerCounts:
    flops: float            # whole layer
    bytes: float            # whole layer, algorithmic
    expert_flops: float     # the two expert GEMMs
    fc1_flops: float
    fc1_bytes: float        # FC1 kernel: touched W1 + latent rows in + hidden rows out
    fc2_flops: float
    fc2_bytes: float        # FC2 kernel: touched W2 + hidden rows in + expert rows out
    expert_weight_bytes: float
    intermediate_bytes: float
    touched: int
    t_exp_mean: float


# Low-precision expert weight formats: (bytes per weight, scale bytes per
# output channel, scale bytes per weight).  e4m3: one byte per code and an fp32
# scale per output channel; mxfp4: half a byte per E2M1 code and one E8M0 byte
# per 32 weights.
EXPERT_FORMATS = {"e4m3": (1.0, 4.0, 0.0), "mxfp4": (0.5, 0.0, 1.0 / 32)}


def expert_matrix_bytes(touched: int, K: int, O: int, elem_bytes: float,
                        expert_format: Optional[str] = None) -> float:
    """Bytes of `touched` expert matrices of K inputs x O outputs."""
    if expert_format is None:
        return touched * K * O * float(elem_bytes)
    per_w, per_ch, scale_per_w = EXPERT_FORMATS[expert_format]
    return touched * (K * O * (per_w + scale_per_w) + O * per_ch)


def layer_counts(*, T: int, d: int, l: int, N: int, k: int, m: int, act: str,
                 shared_m: int = 0, skip_proj: bool = False, elem_bytes: int = 2,
                 loads: Optional[Sequence[int]] = None,
                 expert_format: Optional[str] = None) -> LayerCounts:
    """Counts for one pass over T tokens.  ``loads`` are the per-expert row
    counts (default: every expert touched).  ``expert_format``: the expert
    weights' low-precision format (a key of EXPERT_FORMATS, scales counted
    too), else elem_bytes per weight."""
    m_in = 2 * m if act == "swiglu" else m
    ms_in = 2 * shared_m if act == "swiglu" else shared_m
    R = T * k
    touched = N if loads is None else sum(1 for c in loads if c > 0)
    eb = elem_bytes
    fc1_flops = 2.0 * R * l * m_in
    fc2_flops = 2.0 * R * m * l
    router_flops = 2.0 * T * d * N
    proj_flops = 0.0 if skip_proj else 2.0 * (2.0 * T * d * l)
    shared_flops = 2.0 * T * (d * ms_in + shared_m * d)
    flops = router_flops + proj_flops + fc1_flops + fc2_flops + shared_flops
    w1 = expert_matrix_bytes(touched, l, m_in, eb, expert_format)
    w2 = expert_matrix_bytes(touched, m, l, eb, expert_format)
    other_w = d * N * eb + (0 if skip_proj else 2 * d * l * eb) + (d * ms_in + shared_m * d) * eb
    io = 2.0 * T * d * eb
    byts = w1 + w2 + other_w + io
    fc1_bytes = w1 + T * l * eb + R * m * eb
    fc2_bytes = w2 + R * m * eb + R * l * eb
    inter = 2.0 * eb * (R * l + R * m + R * l + T * l)
    return LayerCounts(flops=flops, bytes=byts, expert_flops=fc1_flops + fc2_flops,
                       fc1_flops=fc1_flops, fc1_bytes=fc1_bytes, fc2_flops=fc2_flops,
                       fc2_bytes=fc2_bytes, expert_weight_bytes=w1 + w2,
                       intermediate_bytes=inter, touched=touched,
                       t_exp_mean=(R / touched) if touched else 0.0)


def stage_counts(*, T: int, d: int, l: int, N: int, k: int, m: int, act: str,
                 shared_m: int = 0, skip_proj: bool = False, elem_bytes: int = 2,
                 loads: Optional[Sequence[int]] = None,
                 expert_format: Optional[str] = None):
    """Algorithmic (flops, bytes) of each launch stage of one forward pass:
    every operand read once and every result written once; expert weights
    only for touched experts (in ``expert_format`` with its scales when
    given).  Keys follow the library's stage names."""
    m_in = 2 * m if act == "swiglu" else m
    ms_in = 2 * shared_m if act == "swiglu" else shared_m
    R = T * k
    eb = elem_bytes
    touched = N if loads is None else sum(1 for c in loads if c > 0)
    kup = (0 if skip_proj else l) + shared_m
    w1 = expert_matrix_bytes(touched, l, m_in, eb, expert_format)
    w2 = expert_matrix_bytes(touched, m, l, eb, expert_format)
    s = {
        "router": (2.0 * T * d * N, T * d * eb + N * d * eb + T * N * 4.0),
        "topk": (0.0, T * N * 4.0 + R * 8.0),
        "group": (0.0, R * 4.0 * 4),
        "down_proj": ((0.0, 0.0) if skip_proj else
                      (2.0 * T * d * l, T * d * eb + d * l * eb + T * l * eb)),
        "shared_fc1": ((0.0, 0.0) if not shared_m else
                       (2.0 * T * d * ms_in, T * d * eb + d * ms_in * eb + T * shared_m * eb)),
        "expert_fc1": (2.0 * R * l * m_in, w1 + T * l * eb + R * m * eb),
        "expert_fc2": (2.0 * R * m * l, w2 + R * m * eb + R * l * eb),
        "combine": (0.0, R * l * eb + T * l * eb + (T * d * eb if skip_proj else 0.0)),
        "up_proj": ((0.0, 0.0) if kup == 0 else
                    (2.0 * T * kup * d, T * kup * eb + kup * d * eb + 2.0 * T * d * eb)),
    }
    return s
