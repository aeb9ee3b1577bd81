"""Python binding of liblmoe.so, the C-ABI LatentMoE layer library.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are passed as raw device pointers (torch is used for device
memory and streams); the names mirror the C entry points in include/lmoe.h.
There is no fallback: if the library is missing, or no CUDA device is
present, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "liblmoe.so")

OK, ERR_INVALID_ARG, ERR_NOT_READY, ERR_CUDA, ERR_OOM, ERR_TIMEOUT, ERR_UNSUPPORTED, ERR_DEVICE = range(8)
ACT = {"silu": 0, "swiglu": 1, "relu2": 2}
DTYPE = {"f32": 0, "bf16": 1}
SKIP_PROJ, DEBUG_CHECKS, FORCE_SIMT, FORCE_SWAP, FORCE_NOSWAP, FORCE_NOPAIR, FORCE_WS_PAIR = (
    0x1, 0x2, 0x4, 0x8, 0x10, 0x20, 0x40)
ROUTE_FULL_SOFTMAX, ROUTE_BIAS_SELECT = 0x80, 0x100
EXPERTS_FP8 = 0x200
SINGLE_STREAM = 0x400
NO_PDL = 0x800
LOAD_SPLIT = 0x1000
NO_STREAM_K = 0x2000
SORTED_ROWS = 0x4000
EXPERTS_FP4 = 0x8000
FC2_SPLIT = 0x10000
MAX_EXPERTS, MAX_TOPK = 1024, 32
DEVERR_WAIT_TIMEOUT, DEVERR_RANGE, DEVERR_NONFINITE = 0x1, 0x2, 0x4
STAGES = {"logits": 0, "idx": 1, "w": 2, "offsets": 3, "perm": 4, "z": 5, "h": 6, "ys": 7, "comb": 8}
EXPORTS = ["lmoe_create", "lmoe_set_weights", "lmoe_reserve", "lmoe_forward", "lmoe_forward_host",
           "lmoe_route_only", "lmoe_router_logits", "lmoe_stage_bytes", "lmoe_debug_dump",
           "lmoe_last_error", "lmoe_profile_begin", "lmoe_profile_end", "lmoe_stage_name",
           "lmoe_last_launch_count", "lmoe_last_expert_path", "lmoe_status_string",
           "lmoe_error_detail", "lmoe_destroy", "lmoe_route_only_noalloc",
           "lmoe_set_expert_weights_fp8", "lmoe_set_expert_weights_fp4",
           "lmoe_selftest_wait_timeout",
           "lmoe_profile_begin_stages"]
NOALLOC_MAX_WORDS = 262144


class LmoeError(RuntimeError):
    def __init__(self, status: int, what: str, detail: str = ""):
        self.status = status
        msg = f"{what}: {status_string(status)} ({status})"
        if detail:
            msg += f" -- {detail}"
        super().__init__(msg)


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run "
                               "`python -m mixture_experts_layer_64_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, U, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_uint, ctypes.c_size_t
        sig = {
            "lmoe_create": ([I, I, I, I, I, I, I, I, U, ctypes.POINTER(P)], I),
            "lmoe_set_weights": ([P] * 9, I),
            "lmoe_set_expert_weights_fp8": ([P] * 5, I),
            "lmoe_set_expert_weights_fp4": ([P] * 5, I),
            "lmoe_selftest_wait_timeout": ([P, U, P], I),
            "lmoe_reserve": ([P, I], I),
            "lmoe_forward": ([P, P, P, I, P], I),
            "lmoe_forward_host": ([P, P, P, I, P], I),
            "lmoe_route_only": ([P, P, I, P, P, P, P, P], I),
            "lmoe_router_logits": ([P, P, P, I, P], I),
            "lmoe_stage_bytes": ([P, I, I, ctypes.POINTER(S)], I),
            "lmoe_debug_dump": ([P, I, P, S, P], I),
            "lmoe_last_error": ([P, ctypes.POINTER(I)], I),
            "lmoe_profile_begin": ([P, I], I),
            "lmoe_profile_begin_stages": ([P, I, ctypes.c_uint], I),
            "lmoe_profile_end": ([P, P, I, ctypes.POINTER(I), ctypes.POINTER(I)], I),
            "lmoe_stage_name": ([I], ctypes.c_char_p),
            "lmoe_last_launch_count": ([P], I),
            "lmoe_last_expert_path": ([P], I),
            "lmoe_status_string": ([I], ctypes.c_char_p),
            "lmoe_error_detail": ([P], ctypes.c_char_p),
            "lmoe_destroy": ([P], None),
            "lmoe_route_only_noalloc": ([P, I, I, I, P, P, P, P, P, P], I),
            "lmoe_ep_reserve": ([P, I], I),
            "lmoe_ep_dispatch": ([P, P, I, P, P, P, P], I),
            "lmoe_ep_experts": ([P, P, P, P, I, I, P, P], I),
            "lmoe_ep_combine": ([P, P, P, P, I, P], I),
            "lmoe_ep_local_plan": ([P, I, I, P, P], I),
        }
        for name, (args, res) in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().lmoe_status_string(s).decode()


def stage_name(i: int) -> str:
    return lib().lmoe_stage_name(i).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def ep_local_plan(recv_counts) -> Dict[str, "np.ndarray"]:
    """lmoe_ep_local_plan (host only): the grouped order of the rows a rank
    receives, from recv_counts [world, n] (host).  Returns offsets [n + 1]
    and perm (grouped row -> received row)."""
    import numpy as np
    rc = np.ascontiguousarray(np.asarray(recv_counts, dtype=np.int32))
    world, n = rc.shape
    offsets = np.zeros(n + 1, dtype=np.int32)
    perm = np.zeros(max(1, int(rc.sum())), dtype=np.int32)
    st = lib().lmoe_ep_local_plan(rc.ctypes.data_as(ctypes.c_void_p), world, n,
                                  offsets.ctypes.data_as(ctypes.c_void_p),
                                  perm.ctypes.data_as(ctypes.c_void_p))
    if st != OK:
        raise LmoeError(st, "lmoe_ep_local_plan")
    return {"offsets": offsets, "perm": perm[:int(rc.sum())]}


def route_only_noalloc(logits: torch.Tensor, k: int, stream=None,
                       checks: bool = False) -> Dict[str, torch.Tensor]:
    """lmoe_route_only_noalloc: the routing steps without a layer handle and
    without any device allocation inside the library (its scratch is a fixed
    device array; calls overlapping on the GPU race).  The outputs are
    allocated here by torch, as a caller that owns its memory would.  With
    checks=True a device error word is passed too (returned as
    "error_word", readable once the stream has completed)."""
    if logits.dtype != torch.float32 or logits.dim() != 2 or not logits.is_cuda:
        raise ValueError("logits must be a [T, N] fp32 CUDA tensor")
    logits = logits.contiguous()
    T, N = logits.shape
    dev = logits.device
    with torch.cuda.device(dev):
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        w = torch.empty((T, k), dtype=torch.float32, device=dev)
        offsets = torch.empty((N + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((T * k,), dtype=torch.int32, device=dev)
        word = torch.empty((1,), dtype=torch.int32, device=dev) if checks else None
        st = lib().lmoe_route_only_noalloc(_ptr(logits), T, N, k, _ptr(idx), _ptr(w),
                                           _ptr(offsets), _ptr(perm), _ptr(word), _stream(stream))
    if st != OK:
        raise LmoeError(st, "lmoe_route_only_noalloc")
    res = {"idx": idx, "w": w, "offsets": offsets, "perm": perm}
    if checks:
        res["error_word"] = word
    return res


class LatentMoELayer:
    """One layer handle (lmoe_create ... lmoe_destroy)."""

    def __init__(self, d: int, l: int, N: int, k: int, m: int, act: str = "swiglu",
                 shared_m: int = 0, dtype: str = "bf16", flags: int = 0, skip_proj: bool = False):
        if not torch.cuda.is_available():
            raise RuntimeError("LatentMoELayer needs a CUDA device (no CPU fallback)")
        if skip_proj:
            flags |= SKIP_PROJ
        self.d, self.l, self.N, self.k, self.m = d, l, N, k, m
        self.act, self.shared_m, self.dtype, self.flags = act, shared_m, dtype, flags
        self.torch_dtype = torch.float32 if dtype == "f32" else torch.bfloat16
        self.m_in = 2 * m if act == "swiglu" else m
        self.ms_in = 2 * shared_m if act == "swiglu" else shared_m
        self.device = torch.device("cuda", torch.cuda.current_device())
        h = ctypes.c_void_p()
        self._check(lib().lmoe_create(d, l, N, k, m, ACT[act], shared_m, DTYPE[dtype], flags,
                                      ctypes.byref(h)), "lmoe_create", use_detail=False)
        self._h = h
        self.max_T = 0

    # -- lifetime ------------------------------------------------------------
    def close(self):
        if getattr(self, "_h", None):
            lib().lmoe_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def _check(self, status: int, what: str, use_detail: bool = True):
        if status != OK:
            detail = ""
            if use_detail and getattr(self, "_h", None):
                detail = lib().lmoe_error_detail(self._h).decode()
            raise LmoeError(status, what, detail)

    def _dev(self, t: Optional[torch.Tensor], shape, dtype=None, name="") -> Optional[torch.Tensor]:
        if t is None:
            return None
        dtype = dtype or self.torch_dtype
        if t.device != self.device or t.dtype != dtype or tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name}: expected {tuple(shape)} {dtype} on {self.device}, "
                             f"got {tuple(t.shape)} {t.dtype} on {t.device}")
        return t.contiguous()

    # -- calls ---------------------------------------------------------------
    def set_weights(self, Wg, bias=None, Wdown=None, Wup=None, W1=None, W2=None, Ws1=None,
                    Ws2=None):
        d, l, N, m = self.d, self.l, self.N, self.m
        ts = dict(Wg=self._dev(Wg, (d, N), name="Wg"),
                  bias=self._dev(bias, (N,), torch.float32, "bias"),
                  Wdown=self._dev(Wdown, (d, l), name="Wdown"),
                  Wup=self._dev(Wup, (l, d), name="Wup"),
                  W1=self._dev(W1, (N, l, self.m_in), name="W1"),
                  W2=self._dev(W2, (N, m, l), name="W2"),
                  Ws1=self._dev(Ws1, (d, self.ms_in), name="Ws1"),
                  Ws2=self._dev(Ws2, (self.shared_m, d), name="Ws2"))
        self._check(lib().lmoe_set_weights(self._h, *[_ptr(ts[k]) for k in
                                                      ("Wg", "bias", "Wdown", "Wup", "W1", "W2",
                                                       "Ws1", "Ws2")]), "lmoe_set_weights")

    def set_expert_weights_fp8(self, W1q, W1s, W2q, W2s):
        """fp8 E4M3 expert weights (layer created with EXPERTS_FP8): uint8 codes
        W1q [N, l, m_in], W2q [N, m, l] in the API layout and fp32 scales per
        output channel W1s [N, m_in], W2s [N, l]."""
        N, l, m = self.N, self.l, self.m
        ts = [self._dev(W1q, (N, l, self.m_in), torch.uint8, "W1q"),
              self._dev(W1s, (N, self.m_in), torch.float32, "W1s"),
              self._dev(W2q, (N, m, l), torch.uint8, "W2q"),
              self._dev(W2s, (N, l), torch.float32, "W2s")]
        self._check(lib().lmoe_set_expert_weights_fp8(self._h, *[_ptr(t) for t in ts]),
                    "lmoe_set_expert_weights_fp8")

    def set_expert_weights_fp4(self, W1q, W1e, W2q, W2e):
        """MXFP4 expert weights (layer created with EXPERTS_FP4), output-major
        uint8: code pairs W1q [N, m_in, l / 2], W2q [N, l, m / 2] (low nibble =
        even input channel) and E8M0 block exponents W1e [N, m_in, l / 32],
        W2e [N, l, m / 32]."""
        N, l, m, mi = self.N, self.l, self.m, self.m_in
        ts = [self._dev(W1q, (N, mi, l // 2), torch.uint8, "W1q"),
              self._dev(W1e, (N, mi, l // 32), torch.uint8, "W1e"),
              self._dev(W2q, (N, l, m // 2), torch.uint8, "W2q"),
              self._dev(W2e, (N, l, m // 32), torch.uint8, "W2e")]
        self._check(lib().lmoe_set_expert_weights_fp4(self._h, *[_ptr(t) for t in ts]),
                    "lmoe_set_expert_weights_fp4")

    def selftest_wait_timeout(self, limit_us: int, stream=None):
        """Test hook: a device wait that nothing completes gives up after
        limit_us and flags LMOE_DEVERR_WAIT_TIMEOUT (read with last_error)."""
        self._check(lib().lmoe_selftest_wait_timeout(self._h, limit_us, _stream(stream)),
                    "lmoe_selftest_wait_timeout")

    def reserve(self, max_T: int):
        self._check(lib().lmoe_reserve(self._h, max_T), "lmoe_reserve")
        self.max_T = max(self.max_T, max_T)

    def forward(self, x: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        T = x.shape[0]
        x = self._dev(x, (T, self.d), name="x")
        if out is None:
            out = torch.empty_like(x)
        self._check(lib().lmoe_forward(self._h, _ptr(x), _ptr(out), T, _stream(stream)),
                    "lmoe_forward")
        return out

    __call__ = forward

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor, stream=None):
        """Host buffers in and out (copies enqueued on `stream`; synchronise it
        before reading out_host)."""
        if x_host.device.type != "cpu" or out_host.device.type != "cpu":
            raise ValueError("forward_host takes host tensors")
        T = x_host.shape[0]
        if not (x_host.is_contiguous() and out_host.is_contiguous()):
            raise ValueError("host tensors must be contiguous")
        if tuple(x_host.shape) != (T, self.d) or tuple(out_host.shape) != (T, self.d):
            raise ValueError("host tensors must be [T, d]")
        self._check(lib().lmoe_forward_host(self._h, _ptr(x_host), _ptr(out_host), T,
                                            _stream(stream)), "lmoe_forward_host")

    def router_logits(self, x: torch.Tensor, stream=None) -> torch.Tensor:
        T = x.shape[0]
        x = self._dev(x, (T, self.d), name="x")
        logits = torch.empty((T, self.N), dtype=torch.float32, device=self.device)
        self._check(lib().lmoe_router_logits(self._h, _ptr(x), _ptr(logits), T, _stream(stream)),
                    "lmoe_router_logits")
        return logits

    def route_only(self, logits: torch.Tensor, stream=None) -> Dict[str, torch.Tensor]:
        T = logits.shape[0]
        logits = self._dev(logits, (T, self.N), torch.float32, "logits")
        dev = self.device
        idx = torch.empty((T, self.k), dtype=torch.int32, device=dev)
        w = torch.empty((T, self.k), dtype=torch.float32, device=dev)
        offsets = torch.empty((self.N + 1,), dtype=torch.int32, device=dev)
        perm = torch.empty((T * self.k,), dtype=torch.int32, device=dev)
        self._check(lib().lmoe_route_only(self._h, _ptr(logits), T, _ptr(idx), _ptr(w),
                                          _ptr(offsets), _ptr(perm), _stream(stream)),
                    "lmoe_route_only")
        return {"idx": idx, "w": w, "offsets": offsets, "perm": perm}

    def stage_bytes(self, stage: str, T: int) -> int:
        n = ctypes.c_size_t()
        self._check(lib().lmoe_stage_bytes(self._h, STAGES[stage], T, ctypes.byref(n)),
                    "lmoe_stage_bytes")
        return n.value

    def debug_dump(self, stage: str, T: int, stream=None) -> torch.Tensor:
        """The named intermediate of the last forward (which ran on T tokens)."""
        nbytes = self.stage_bytes(stage, T)
        buf = torch.empty((nbytes,), dtype=torch.uint8, device=self.device)
        self._check(lib().lmoe_debug_dump(self._h, STAGES[stage], _ptr(buf), nbytes,
                                          _stream(stream)), "lmoe_debug_dump")
        R = T * self.k
        shapes = {"logits": ((T, self.N), torch.float32), "idx": ((T, self.k), torch.int32),
                  "w": ((T, self.k), torch.float32), "offsets": ((self.N + 1,), torch.int32),
                  "perm": ((R,), torch.int32), "z": ((T, self.l), self.torch_dtype),
                  "h": ((R, self.m), self.torch_dtype), "ys": ((R, self.l), self.torch_dtype),
                  "comb": ((T, self.l), self.torch_dtype)}
        shape, dt = shapes[stage]
        return buf.view(dt).view(shape)

    def last_error(self):
        """(status, device error word); synchronises the device."""
        word = ctypes.c_int()
        st = lib().lmoe_last_error(self._h, ctypes.byref(word))
        return st, word.value

    def profile_begin(self, max_forwards: int, stages=None):
        """Records stage times of the next max_forwards forwards: every stage,
        or only the named ones (the other boundaries stay free of events)."""
        if stages is None:
            self._check(lib().lmoe_profile_begin(self._h, max_forwards), "lmoe_profile_begin")
        else:
            names = [stage_name(i) for i in range(16) if stage_name(i)]
            mask = 0
            for n in stages:
                mask |= 1 << names.index(n)
            self._check(lib().lmoe_profile_begin_stages(self._h, max_forwards, mask),
                        "lmoe_profile_begin_stages")
        self._prof_cap = max_forwards

    def profile_end(self):
        """Per-forward stage times (ms): a list of dicts stage name -> ms
        (recorded stages only)."""
        cap = self._prof_cap * 16
        buf = (ctypes.c_float * cap)()
        nf, ns = ctypes.c_int(), ctypes.c_int()
        self._check(lib().lmoe_profile_end(self._h, buf, cap, ctypes.byref(nf), ctypes.byref(ns)),
                    "lmoe_profile_end")
        names = [stage_name(i) for i in range(ns.value)]
        return [{names[s]: buf[f * ns.value + s] for s in range(ns.value)
                 if buf[f * ns.value + s] >= 0} for f in range(nf.value)]

    # -- expert parallelism (dispatch / experts / combine in latent space) ----
    def ep_reserve(self, max_recv_rows: int):
        self._check(lib().lmoe_ep_reserve(self._h, max_recv_rows), "lmoe_ep_reserve")

    def ep_dispatch(self, x: torch.Tensor, stream=None):
        """Step 1: (send_rows [T*k, l], send_gates [T*k], expert_counts [N]) on
        the device, rows sorted by expert then token."""
        T = x.shape[0]
        x = self._dev(x, (T, self.d), name="x")
        cols = self.d if self.flags & SKIP_PROJ else self.l
        rows = torch.empty((T * self.k, cols), dtype=self.torch_dtype, device=self.device)
        gates = torch.empty((T * self.k,), dtype=torch.float32, device=self.device)
        counts = torch.empty((self.N,), dtype=torch.int32, device=self.device)
        self._check(lib().lmoe_ep_dispatch(self._h, _ptr(x), T, _ptr(rows), _ptr(gates),
                                           _ptr(counts), _stream(stream)), "lmoe_ep_dispatch")
        return rows, gates, counts

    def ep_experts(self, recv_rows: torch.Tensor, recv_gates: torch.Tensor, recv_counts,
                   rank: int, world: int, stream=None) -> torch.Tensor:
        """Step 3: the local experts on the received rows; recv_counts is a
        host array-like [world, N / world].  Returns out_rows (received order)."""
        rc = torch.as_tensor(recv_counts, dtype=torch.int32).reshape(world, self.N // world)
        rc = rc.contiguous()
        Rr = int(rc.sum())
        cols = self.d if self.flags & SKIP_PROJ else self.l
        out = torch.empty((Rr, cols), dtype=self.torch_dtype, device=self.device)
        if Rr:
            recv_rows = self._dev(recv_rows, (Rr, cols), name="recv_rows")
            recv_gates = self._dev(recv_gates, (Rr,), torch.float32, "recv_gates")
        self._check(lib().lmoe_ep_experts(self._h, _ptr(recv_rows) if Rr else None,
                                          _ptr(recv_gates) if Rr else None,
                                          ctypes.c_void_p(rc.data_ptr()), rank, world,
                                          _ptr(out) if Rr else None, _stream(stream)),
                    "lmoe_ep_experts")
        return out

    def ep_combine(self, x: torch.Tensor, back_rows: torch.Tensor, out=None, stream=None):
        """Step 5: out = x + the layer, from the returned rows (send order)."""
        T = x.shape[0]
        x = self._dev(x, (T, self.d), name="x")
        cols = self.d if self.flags & SKIP_PROJ else self.l
        back_rows = self._dev(back_rows, (T * self.k, cols), name="back_rows")
        if out is None:
            out = torch.empty_like(x)
        self._check(lib().lmoe_ep_combine(self._h, _ptr(x), _ptr(back_rows), _ptr(out), T,
                                          _stream(stream)), "lmoe_ep_combine")
        return out

    @property
    def last_launch_count(self) -> int:
        return lib().lmoe_last_launch_count(self._h)

    @property
    def last_expert_path(self) -> int:
        return lib().lmoe_last_expert_path(self._h)
