#!/usr/bin/env python
"""Benchmark of the LatentMoE layer forward pass on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

One step is one lmoe_forward over the workload's T tokens (router, top-k,
grouping, down-projection, expert FC1/FC2, combine, up-projection, residual).
Inputs are seeded synthetic tensors resident in HBM; the expert weights
(GBs) exceed the 126 MB L2, so every step streams them from HBM.  With N GPUs
(one process each, launched by torchrun) every rank runs an independent
replica on its own batch: tokens are independent, so there is no data-path
collective; the timed region is bracketed by a barrier and
torch.cuda.synchronize(), and the time is the max over ranks.

Prints one JSON line (rank 0).  With the default workload (decode, the
headline) the line also carries "prefill": the two prefill workloads
(latent-prefill-skewed, latent-prefill-shared), and "decode_variants": the
latent decode workload and both decode workloads with fp8 (E4M3) and with
fp4 (MXFP4) expert weights, each with its own clocks, roofline, expert-load
summary, per-stage p50/p95/p99 and projection share; and "variant_sweep": the
standard MoE, l-MoE_eff and l-MoE_acc (LatentMoE, Section 3, Eq. (1) and
(2)) at a latency-bound, a decode and a prefill batch, with the weight and dispatch bytes
each loads.  All are measured in the same run with the same steps and
warm-up (--no-prefill skips them).  --impl reference times the CPU oracle (the reference arm of this
method: a plain float64 C++ implementation) on a bounded token sample of the
same workload.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import hashlib
import io
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from typing import Optional

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from mixture_experts_layer_64_b200 import costmodel, workloads  # noqa: E402

METRIC = "LatentMoE layer tokens/sec at decode & prefill T; HBM GB/s / tensor-pipe % of peak"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "std-moe-decode"
EXPERT_PATHS = ["cuda-core", "tcgen05 token-tiled", "tcgen05 weight-stationary",
                "tcgen05 token-tiled, 2-SM CTA pairs", "tcgen05 weight-stationary, 2-SM CTA pairs",
                "tcgen05 split by load: 2-SM CTA-pair token tiles above 384 rows per expert, "
                "weight-stationary tiles of the expert's rows below"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
_CSRC = "mixture_experts_layer_64_b200/csrc/"
_GEMM_SRC = (_CSRC + "common.cuh", _CSRC + "tc_gemm.cuh")
# device code of each stage's kernel: recorded DRAM traffic is trusted only
# while these files are unchanged since the capture
STAGE_SOURCES = {"router": _GEMM_SRC, "down_proj": _GEMM_SRC, "shared_fc1": _GEMM_SRC,
                 "expert_fc1": _GEMM_SRC, "expert_fc2": _GEMM_SRC, "up_proj": _GEMM_SRC,
                 "topk": (_CSRC + "common.cuh", _CSRC + "routing.cuh"),
                 "group": (_CSRC + "common.cuh", _CSRC + "routing.cuh"),
                 "combine": (_CSRC + "common.cuh", _CSRC + "misc.cuh")}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def kernel_source_hash(stage: str) -> str:
    h = hashlib.sha256()
    for f in STAGE_SOURCES[stage]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def recorded_traffic(workload: str, stage: str):
    """DRAM bytes per launch of `stage` from the committed ncu summary, or None
    when absent or taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as fh:
        d = json.load(fh)
    rec = d.get(workload, {}).get(stage)
    if not rec or rec.get("kernel_sources") != kernel_source_hash(stage):
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

def gpu_uuid(dev) -> Optional[str]:
    """The CUDA device's UUID as NVML spells it (without its "GPU-" prefix)."""
    try:
        return str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        return None


class ClockSampler:
    """SM clock, power and clock-event (throttle) reasons of one GPU while the
    timed region runs.  NVML is read in a thread every 20 ms (read-only
    queries; the device is found by its UUID, since NVML does not follow
    CUDA_VISIBLE_DEVICES); without NVML the nvidia-smi query loop runs
    instead, and timing starts only once its first sample has landed."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_S = 0.02

    def __init__(self, gpu_index: int, path: Optional[str] = None, uuid: Optional[str] = None):
        """Rows go to `path` as CSV (nvidia-smi's columns) when given."""
        self.gpu = gpu_index
        self.uuid = uuid
        self.path = path
        self.proc = None
        self.thread = None
        self.rows = []

    # ---- NVML thread
    def _nvml_handle(self):
        import pynvml
        pynvml.nvmlInit()
        if self.uuid:
            for u in (self.uuid, "GPU-" + self.uuid):
                try:
                    return pynvml, pynvml.nvmlDeviceGetHandleByUUID(u)
                except pynvml.NVMLError:
                    pass
        return pynvml, pynvml.nvmlDeviceGetHandleByIndex(self.gpu)

    def _nvml_row(self, nv, h):
        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
        mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
        pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
        try:
            rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
        except AttributeError:
            rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
        bits = (nv.nvmlClocksEventReasonHwSlowdown, nv.nvmlClocksEventReasonHwThermalSlowdown,
                nv.nvmlClocksEventReasonSwThermalSlowdown, nv.nvmlClocksEventReasonSwPowerCap)
        flags = ["Active" if rs & b else "Not Active" for b in bits]
        return [str(self.gpu), str(sm), str(mx), f"{pw:.2f}", hex(rs)] + flags

    def _loop(self, nv, h):
        while not self.done.is_set():
            try:
                self.rows.append(self._nvml_row(nv, h))
            except Exception:
                pass
            self.done.wait(self.PERIOD_S)

    def start(self):
        import threading
        try:
            nv, h = self._nvml_handle()
            self.rows.append(self._nvml_row(nv, h))
            self.done = threading.Event()
            self.thread = threading.Thread(target=self._loop, args=(nv, h), daemon=True)
            self.thread.start()
            return
        except Exception:
            self.thread = None
        # fallback: nvidia-smi's query loop, into a file
        try:
            self.smi_path = self.path
            if self.smi_path is None:
                fd, self.smi_path = tempfile.mkstemp(prefix=f"clocks_gpu{self.gpu}_", suffix=".csv")
                os.close(fd)
            self.fh = open(self.smi_path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        t_end = time.time() + 5.0
        while time.time() < t_end and not self._smi_rows():
            time.sleep(0.02)

    def _smi_rows(self):
        try:
            with open(self.smi_path) as fh:
                return [[c.strip() for c in r] for r in csv.reader(fh) if len(r) >= 9]
        except OSError:
            return []

    def stop(self):
        if self.thread is not None:
            time.sleep(self.PERIOD_S)
            self.done.set()
            self.thread.join(timeout=2)
            rows = list(self.rows)
            if self.path:
                with open(self.path, "w") as fh:
                    fh.writelines(", ".join(r) + "\n" for r in rows)
        elif self.proc is not None:
            time.sleep(0.15)  # one more sample after the timed region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()
            rows = self._smi_rows()
            if self.path is None:
                os.unlink(self.smi_path)
        else:
            return None
        if not rows:
            return None

        def num(s):
            try:
                return float(s)
            except ValueError:
                return float("nan")

        sm = [num(r[1]) for r in rows]
        mx = [num(r[2]) for r in rows]
        pw = [num(r[3]) for r in rows]
        # samples under load: the top half by power draw
        order = sorted(range(len(rows)), key=lambda i: -pw[i] if pw[i] == pw[i] else 0)
        load = order[: max(1, len(order) // 2)]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[j] for i in load for j in range(4)
                          if rows[i][5 + j].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm[i] for i in load),
                "sm_max_mhz": max(x for x in mx if x == x) if any(x == x for x in mx) else None,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(load),
                "source": "nvml" if self.thread is not None else "nvidia-smi"}


# ---------------------------------------------------------------------------
# oracle (CPU baseline / reference arm)
# ---------------------------------------------------------------------------

class OracleRunner:
    """Times the CPU oracle on token samples of a workload.  Host copies of the
    weights are taken once; expert matrices are copied on first use."""

    def __init__(self, w: workloads.Workload, W_dev, x_dev):
        import oracle

        self.oracle = oracle
        self.w = w
        self.threads = oracle.default_threads()
        cpu = lambda t: None if t is None else t.detach().cpu()
        self.W_dev = W_dev
        self.x = cpu(x_dev)
        self.base = dict(d=w.d, l=w.l, N=w.N, k=w.k, m=w.m, act=w.act, shared_m=w.shared_m,
                         dtype=w.dtype, skip_proj=w.skip_proj, Wg=cpu(W_dev["Wg"]),
                         bias=cpu(W_dev["bias"]), Wdown=cpu(W_dev["Wdown"]),
                         Wup=cpu(W_dev["Wup"]), Ws1=cpu(W_dev["Ws1"]), Ws2=cpu(W_dev["Ws2"]))
        # low-precision experts: the codes plus their scales (fp8: per channel
        # W1s / W2s) or block exponents (fp4: W1e / W2e)
        self.skeys = (("W1s", "W2s") if w.expert_fp8 else ("W1e", "W2e") if w.expert_fp4
                      else ())
        self.probe = oracle.OracleLayer(W1={}, W2={}, **self.base)
        self.W1, self.W2 = {}, {}
        self.S = {k: {} for k in self.skeys}

    def time_tokens(self, tokens: np.ndarray) -> float:
        """Seconds the oracle takes for the whole layer on `tokens` (routing
        probe and weight copies untimed)."""
        lg = self.probe.router_logits(self.x, tokens).astype(np.float32)
        idx, _, _, _ = self.oracle.route(lg, self.w.k)
        for e in np.unique(idx).tolist():
            if e not in self.W1:
                q = "q" if self.skeys else ""
                self.W1[e] = self.W_dev["W1" + q][e].cpu()
                self.W2[e] = self.W_dev["W2" + q][e].cpu()
                for k in self.skeys:
                    self.S[k][e] = self.W_dev[k][e].cpu()
        O = self.oracle.OracleLayer(W1=self.W1, W2=self.W2, **self.S, **self.base)
        t0 = time.perf_counter()
        O.layer(self.x, tokens=tokens)
        return time.perf_counter() - t0

    def sample(self, n: int, seed: int) -> np.ndarray:
        rng = np.random.default_rng(seed)
        n = max(1, min(n, self.w.T))
        return np.sort(rng.choice(self.w.T, size=n, replace=False)).astype(np.int32)

    def calibrated_rate(self, target_s: float, seed: int = 0):
        """(tokens/s, tokens, seconds) on a sample sized to take ~target_s."""
        n = min(self.w.T, 4)
        dt = self.time_tokens(self.sample(n, seed))
        n2 = int(min(self.w.T, max(n, n / dt * target_s)))
        if n2 > n:
            dt = self.time_tokens(self.sample(n2, seed + 1))
            n = n2
        return n / dt, n, dt


# ---------------------------------------------------------------------------
# the arms
# ---------------------------------------------------------------------------

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def workload_config(w: workloads.Workload, n_gpus: int):
    c = costmodel.layer_counts(T=w.T, d=w.d, l=w.l, N=w.N, k=w.k, m=w.m, act=w.act,
                               shared_m=w.shared_m, skip_proj=w.skip_proj,
                               expert_format=w.expert_format)
    return {"workload": w.name, "T": w.T, "d": w.d, "l": w.l, "N": w.N, "k": w.k, "m": w.m,
            "act": w.act, "shared_m": w.shared_m, "skip_proj": w.skip_proj, "bias": w.bias,
            "expert_weights": EXPERT_WEIGHTS.get(w.expert_format, w.dtype),
            "global_batch": w.T * n_gpus, "parallelism": f"replicas{n_gpus}",
            "l2": f"inputs larger than L2: {c.expert_weight_bytes / 1e9:.2f} GB of expert "
                  "weights streamed from HBM every step"}


# ---------------------------------------------------------------------------
# replicas (one process per GPU): the pieces that do not need a GPU
# ---------------------------------------------------------------------------

def replica_workload(w: workloads.Workload, rank: int) -> workloads.Workload:
    """Rank r draws its own batch (seed + 1000 r); weights are the same."""
    return w if rank == 0 else workloads.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def max_over_ranks(pg, value: float, device) -> float:
    """The largest of the ranks' values (the job's time is its slowest rank)."""
    if pg is None:
        return float(value)
    t = torch.tensor([value], device=device, dtype=torch.float64)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_throughput(tokens_per_rank: int, ranks: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * ranks / (ms_per_step / 1000.0)


def run_reference(args):
    ws, rank, _ = dist_env()
    if rank != 0:
        return 0
    w = workloads.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    W = workloads.make_weights(w, device=dev)
    x = workloads.make_x(w, device=dev)
    runner = OracleRunner(w, W, x)
    steps = args.steps + args.warmup
    budget_s = 150.0
    rate, _, _ = runner.calibrated_rate(target_s=min(10.0, budget_s / steps))
    per_step = int(min(w.T, max(1, rate * budget_s / steps)))
    tok, sec = 0, 0.0
    for s in range(steps):
        dt = runner.time_tokens(runner.sample(per_step, seed=100 + s))
        if s >= args.warmup:
            tok += per_step
            sec += dt
    value = tok / sec
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * sec / max(1, args.steps), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, 1),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": runner.threads,
                             "kind": "oracle",
                             "sample": f"{per_step} of {w.T} tokens per step ({w.name}), whole "
                                       "layer from x (fp64 logits, fp32 selection)"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


PREFILL_WORKLOADS = ("latent-prefill-skewed", "latent-prefill-shared")
# the other decode workloads, measured beside the headline in the same run
DECODE_WORKLOADS = ("latent-decode", "std-moe-decode-fp8", "latent-decode-fp8",
                    "std-moe-decode-fp4", "latent-decode-fp4")
EXPERT_WEIGHTS = {"e4m3": "e4m3 codes, fp32 scale per output channel (widened to f16 in the "
                          "expert kernels)",
                  "mxfp4": "MXFP4: e2m1 codes, one e8m0 exponent per 32 inputs (widened to f16 "
                           "in the expert kernels)"}
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s HBM figure the decode target is quoted against
PROJECTION_SHARE_PAGES = 0.09  # the paper's ~9% latent-projection overhead (Section 4.3)


def percentiles(vals):
    a = np.asarray(vals, dtype=np.float64)
    return {"p50": round(float(np.percentile(a, 50)), 5), "p95": round(float(np.percentile(a, 95)), 5),
            "p99": round(float(np.percentile(a, 99)), 5), "mean": round(float(a.mean()), 5)}


def load_summary(loads: np.ndarray):
    """Per-expert routed rows of one forward (from the offsets): touched
    experts, the largest load, and the MMA work of tiles of 16 / 64 / 128 /
    256 rows relative to the routed rows (padding of each expert's last tile)."""
    c = loads[loads > 0]
    if c.size == 0:
        return {"touched": 0}
    pad = {str(tile): round(float((np.ceil(c / tile) * tile).sum() / c.sum()), 4)
           for tile in (16, 64, 128, 256)}
    return {"touched": int(c.size), "max_rows": int(c.max()), "min_rows": int(c.min()),
            "mean_rows_touched": round(float(c.mean()), 2), "routed_rows": int(c.sum()),
            "rows_in_experts_over_4096": int(c[c >= 4096].sum()),
            "experts_under_16_rows": int((c < 16).sum()), "padding_factor": pad}


def measure(args, name: str, pg, rank: int, ws: int, local: int, dev, flags: int = 0,
            n_prof: int = 50):
    """Builds the workload's layer and measures it: an untimed profiled pass
    (events at every stage boundary, n_prof forwards), the timed region of
    args.steps forwards (events around the dominant stage only), and the
    host-buffer entry point.  Every rank takes the same collective steps."""
    from mixture_experts_layer_64_b200 import lmoe

    w = workloads.WORKLOADS[name]
    W = workloads.make_weights(w, device=dev)
    xw = replica_workload(w, rank)  # each replica draws its own batch
    x = workloads.make_x(xw, device=dev)
    L = lmoe.LatentMoELayer(w.d, w.l, w.N, w.k, w.m, act=w.act, shared_m=w.shared_m,
                            dtype=w.dtype, skip_proj=w.skip_proj,
                            flags=flags | (lmoe.EXPERTS_FP8 if w.expert_fp8 else 0) |
                            (lmoe.EXPERTS_FP4 if w.expert_fp4 else 0))
    L.set_weights(W["Wg"], W["bias"], W["Wdown"], W["Wup"], W["W1"], W["W2"], W["Ws1"], W["Ws2"])
    if w.expert_fp8:
        L.set_expert_weights_fp8(W["W1q"], W["W1s"], W["W2q"], W["W2s"])
    if w.expert_fp4:
        L.set_expert_weights_fp4(W["W1q"], W["W1e"], W["W2q"], W["W2e"])
    L.reserve(w.T)
    out = torch.empty_like(x)
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        L.forward(x, out)
    torch.cuda.synchronize()
    st, word = L.last_error()
    if st != lmoe.OK:
        raise RuntimeError(f"device error after warm-up: {lmoe.status_string(st)} word={word}")
    launches_per_step = L.last_launch_count
    loads = np.diff(L.debug_dump("offsets", w.T).cpu().numpy())

    # ---- stage breakdown: an untimed pass with events at every stage boundary
    L.profile_begin(n_prof)
    for _ in range(n_prof):
        L.forward(x, out)
    prof_all = L.profile_end()
    stage_pct = {k: percentiles([p[k] for p in prof_all]) for k in prof_all[0]}
    stage_ms = {k: v["mean"] for k, v in stage_pct.items()}
    dom = max(stage_ms, key=stage_ms.get)

    sampler = ClockSampler(local, args.clocks_csv if name == args.workload else None,
                           gpu_uuid(dev)) if rank == 0 else None
    if sampler:
        sampler.start()
    # ---- timed region: K steps; events on the launching stream around the
    # dominant stage only, so that the other kernel boundaries keep their
    # programmatic dependent launches
    L.profile_begin(args.steps, stages=[dom])
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for _ in range(args.steps):
        L.forward(x, out)
    t1.record(stream)
    torch.cuda.synchronize()
    if pg:
        pg.barrier()
    clocks = sampler.stop() if sampler else None
    elapsed_ms = t0.elapsed_time(t1)
    prof = L.profile_end()
    elapsed_ms = max_over_ranks(pg, elapsed_ms, dev)
    ms_per_step = elapsed_ms / args.steps

    # ---- end to end through the host-buffer entry point (pinned buffers)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    for _ in range(max(1, args.warmup // 2)):
        L.forward_host(xh, oh)
    e_steps = max(3, min(args.steps, 200))
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e_steps):
        L.forward_host(xh, oh)
    e1.record(stream)
    torch.cuda.synchronize()
    e_ms = max_over_ranks(pg, e0.elapsed_time(e1) / e_steps, dev)
    io_bytes = w.T * w.d * (4 if w.dtype == "f32" else 2)

    st, word = L.last_error()
    if st != lmoe.OK:
        raise RuntimeError(f"device error: {lmoe.status_string(st)} word={word}")

    # ---- roofline of the dominant kernel (its average over the timed steps)
    dom_ms = statistics.fmean(p[dom] for p in prof)
    counts = costmodel.stage_counts(T=w.T, d=w.d, l=w.l, N=w.N, k=w.k, m=w.m, act=w.act,
                                    shared_m=w.shared_m, skip_proj=w.skip_proj,
                                    elem_bytes=4 if w.dtype == "f32" else 2, loads=loads,
                                    expert_format=w.expert_format)
    peaks, peak_src = load_peaks()
    roofline = None
    if dom_ms > 0:
        fl, by = counts[dom]
        t = dom_ms / 1000.0
        ridge = peaks["bf16_tflops_sustained"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        if by > 0 and (fl / by) < ridge:
            ach = by / t / 1e9
            roofline = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": ach / peaks["hbm_gbs"],
                        "peak_source": f"{peak_src} (hbm_gbs: a STREAM-style copy)",
                        "frac_of_nominal": ach / NOMINAL_HBM_GBS,
                        "nominal_note": "achieved / 8000 GB/s, the ~8 TB/s B200 HBM figure: a "
                                        "read-only weight stream can exceed the measured copy"}
        else:
            ach = fl / t / 1e12
            pb, psus = peaks["bf16_tflops"], peaks["bf16_tflops_sustained"]
            roofline = {"bound": "tensor", "achieved": ach, "peak": pb, "unit": "TFLOP/s",
                        "frac": ach / pb,
                        "peak_source": f"{peak_src} (bf16_tflops: cuBLAS bf16 burst)",
                        "peak_sustained": psus, "frac_sustained": ach / psus}
        roofline.update({"traffic": recorded_traffic(w.name, dom), "kernel": dom,
                         "algorithmic_per_launch": by if roofline["bound"] == "hbm" else fl,
                         "launch_ms": dom_ms})
    lc = costmodel.layer_counts(T=w.T, d=w.d, l=w.l, N=w.N, k=w.k, m=w.m, act=w.act,
                                shared_m=w.shared_m, skip_proj=w.skip_proj, loads=loads,
                                expert_format=w.expert_format)
    layer = {"alg_bytes": lc.bytes, "alg_flops": lc.flops,
             "hbm_frac": lc.bytes / (ms_per_step / 1e3) / 1e9 / peaks["hbm_gbs"],
             "tensor_frac_burst": lc.flops / (ms_per_step / 1e3) / 1e12 / peaks["bf16_tflops"],
             "touched_experts": lc.touched, "t_exp_mean": round(lc.t_exp_mean, 2),
             "paper_intensity": costmodel.arithmetic_intensity(lc.t_exp_mean, w.l, w.m)
             if lc.touched else None}
    if w.skip_proj:
        proj = {"value": None, "note": "no projections (standard-MoE shape, l = d)"}
    else:
        p50 = stage_pct["down_proj"]["p50"] + stage_pct["up_proj"]["p50"]
        proj = {"value": round(p50 / ms_per_step, 4), "pages": PROJECTION_SHARE_PAGES,
                "down_proj_ms_p50": stage_pct["down_proj"]["p50"],
                "up_proj_ms_p50": stage_pct["up_proj"]["p50"],
                "note": "(down + up projection) p50 / timed step; the down-projection runs "
                        "on a second stream beside the router and routing"}
    res = {"workload": name, "w": w, "W": W, "x": x, "ms_per_step": ms_per_step,
           "value": job_throughput(w.T, ws, ms_per_step),
           "e2e": {"value": job_throughput(w.T, ws, e_ms), "unit": UNIT,
                   "h2d_bytes_per_step": io_bytes, "d2h_bytes_per_step": io_bytes},
           "gpu_launches": launches_per_step * args.steps, "clocks": clocks,
           "roofline": roofline, "layer": layer, "stage_ms": stage_pct,
           "stage_ms_source": f"untimed pass of {n_prof} forwards after {args.warmup} warm-up "
                              "forwards, events at every stage boundary",
           "projection_share": proj, "expert_loads": load_summary(loads),
           "expert_path": {"fc1": EXPERT_PATHS[max(0, L.last_expert_path) & 7],
                           "fc2": EXPERT_PATHS[max(0, L.last_expert_path) >> 3]}}
    L.close()
    return res


def sub_record(r):
    """The JSON of one measured workload beside the headline (prefill)."""
    w = r["w"]
    return {"workload": r["workload"], "value": r["value"], "unit": UNIT,
            "ms_per_step": r["ms_per_step"], "config": {"T": w.T, "d": w.d, "l": w.l, "N": w.N,
                                                        "k": w.k, "m": w.m, "act": w.act,
                                                        "shared_m": w.shared_m, "bias": w.bias,
                                                        "skip_proj": w.skip_proj,
                                                        "expert_weights": w.expert_format
                                                        or w.dtype},
            "e2e": r["e2e"], "gpu_launches": r["gpu_launches"], "clocks": r["clocks"],
            "roofline": r["roofline"], "layer": r["layer"], "expert_loads": r["expert_loads"],
            "projection_share": r["projection_share"], "stage_ms": r["stage_ms"],
            "expert_path": r["expert_path"]}


def sweep_point(variant: str, r) -> dict:
    """One point of the LatentMoE variant sweep: the measured step and the
    costs the paper's Table 1 compares: the expert weight bytes one token
    activates (its k experts: the memory cost of the latency regime), the
    bytes of one token's dispatch to its experts (one direction), the expert
    FLOPs per token; beside them the expert weight bytes the step loads (the
    touched experts: at batch sizes that touch every expert this is the whole
    expert set, the same for all three variants)."""
    w = r["w"] if "w" in r else workloads.WORKLOADS[r["workload"]]
    touched = r["expert_loads"].get("touched", 0)
    m_in = 2 * w.m if w.act == "swiglu" else w.m
    return {"variant": variant, "workload": w.name, "T": w.T, "d": w.d, "l": w.l, "N": w.N,
            "k": w.k, "m": w.m, "value": r["value"], "unit": UNIT,
            "ms_per_step": r["ms_per_step"], "touched_experts": touched,
            "expert_weight_bytes": touched * (w.l * m_in + w.m * w.l) * 2,
            "active_weight_bytes_per_token": w.k * (w.l * m_in + w.m * w.l) * 2,
            "dispatch_bytes_per_token": w.k * w.l * 2,
            "expert_flops_per_token": 2.0 * w.k * (w.l * m_in + w.m * w.l),
            "expert_ms": {k: r["stage_ms"][k]["p50"] for k in ("expert_fc1", "expert_fc2")}}


def variant_sweep(points) -> dict:
    """Ratios of each variant to the standard point of its batch size."""
    std = points[0]
    for p in points:
        p["vs_standard"] = {key: round(p[key] / std[key], 4) if std[key] else None
                            for key in ("ms_per_step", "expert_weight_bytes",
                                        "active_weight_bytes_per_token",
                                        "dispatch_bytes_per_token", "expert_flops_per_token")}
    return {"points": points,
            "paper": "Table 1: per token, l-MoE_eff cuts the active weight bytes and the "
                     "dispatch bytes by alpha = d / l = 4 at 1 / alpha the expert FLOPs; "
                     "l-MoE_acc keeps both costs and the FLOPs of the standard layer"}


def run_ours(args):
    from mixture_experts_layer_64_b200 import build

    ws, rank, local = dist_env()
    pg = None
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
        pg = dist
    else:
        torch.cuda.set_device(0)
    build.build_library()
    dev = torch.device("cuda", torch.cuda.current_device())
    main = measure(args, args.workload, pg, rank, ws, local, dev, flags=args.lib_flags)
    w, W, x = main.pop("w"), main.pop("W"), main.pop("x")
    main_point = sweep_point("standard", dict(main, w=w))

    cpu_baseline = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        try:
            runner = OracleRunner(w, W, x)
            rate, n, dt = runner.calibrated_rate(target_s=15.0)
            cpu_baseline = {"value": rate, "unit": UNIT, "cores": runner.threads,
                            "kind": "oracle",
                            "sample": f"{n} of {w.T} tokens of {w.name} ({dt:.1f} s), whole "
                                      "layer from x"}
        except Exception as e:  # the baseline is reported, never required
            cpu_baseline = {"value": None, "unit": UNIT, "cores": None, "kind": "oracle",
                            "sample": f"failed: {e}"}
    del W, x
    torch.cuda.empty_cache()

    # ---- the prefill workloads (and the other decode workloads), measured in
    # the same run with the same steps
    extra = {"prefill": [], "decode_variants": [], "variant_sweep": {}}
    if not args.no_prefill and args.workload == DEFAULT_WORKLOAD:
        for key, names in (("prefill", PREFILL_WORKLOADS), ("decode_variants", DECODE_WORKLOADS)):
            for name in names:
                r = measure(args, name, pg, rank, ws, local, dev, flags=args.lib_flags)
                del r["W"], r["x"]
                extra[key].append(sub_record(r))
                del r
                torch.cuda.empty_cache()
        # the paper's variants on the same kernels (the standard decode point
        # is the headline workload measured above)
        for batch, *names in workloads.VARIANT_SWEEP:
            points = []
            for variant, name in zip(("standard", "l-MoE_eff", "l-MoE_acc"), names):
                if name == args.workload:
                    points.append(main_point)
                    continue
                r = measure(args, name, pg, rank, ws, local, dev, flags=args.lib_flags)
                del r["W"], r["x"]
                points.append(sweep_point(variant, r))
                del r
                torch.cuda.empty_cache()
            extra["variant_sweep"][batch] = variant_sweep(points)

    if rank == 0:
        roofline = main["roofline"]
        if roofline is not None:
            roofline = dict(roofline, stage_ms={k: v["mean"] for k, v in main["stage_ms"].items()},
                            layer=main["layer"])
        line = {"metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": ws,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": w.dtype, "data": "synthetic", "config": workload_config(w, ws),
                "e2e": main["e2e"], "gpu_launches": main["gpu_launches"],
                "lib_flags": args.lib_flags, "roofline": roofline, "cpu_baseline": cpu_baseline,
                "clocks": main["clocks"], "expert_path": main["expert_path"],
                "stage_ms": main["stage_ms"], "stage_ms_source": main["stage_ms_source"],
                "projection_share": main["projection_share"],
                "expert_loads": main["expert_loads"]}
        for key, recs in extra.items():
            if recs:
                line[key] = recs
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=workloads.WORKLOAD_ORDER, default=DEFAULT_WORKLOAD)

    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="skip the prefill and other decode workloads measured beside the "
                         "default decode line")
    ap.add_argument("--experts", type=int, default=None,
                    help="override N (reduced cases for profiler captures)")
    ap.add_argument("--topk", type=int, default=None, help="override k")
    ap.add_argument("--tokens", type=int, default=None, help="override T")
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region here")
    ap.add_argument("--lib-flags", type=int, default=0,
                    help="lmoe_create flags (e.g. 32 = never use CTA pairs) for A/B runs")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.experts or args.topk or args.tokens:
        import dataclasses
        base = workloads.WORKLOADS[args.workload]
        ch = {k: v for k, v in (("N", args.experts), ("k", args.topk), ("T", args.tokens)) if v}
        name = base.name + "(" + ",".join(f"{k}={v}" for k, v in ch.items()) + ")"
        workloads.WORKLOADS[name] = dataclasses.replace(base, name=name, **ch)
        args.workload = name
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
