"""ctypes front end of the CPU oracle (lmoe_oracle.cpp).

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.  It imports nothing
from the CUDA library's package; arrays come in as numpy arrays or CPU torch
tensors holding the same bytes the library receives.

Functions follow the LatentMoE paper (arXiv 2601.18089), Section 3, Eq. (1)
and Eq. (2); see the header of lmoe_oracle.cpp for the exact definitions.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Sequence

import numpy as np

from .build import LIB_PATH, build_oracle

ACT_CODES = {"silu": 0, "swiglu": 1, "relu2": 2}
DTYPE_CODES = {"f32": 0, "bf16": 1}


class OracleError(RuntimeError):
    pass


class _Layer(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("l", ctypes.c_int), ("N", ctypes.c_int),
                ("k", ctypes.c_int), ("m", ctypes.c_int), ("act", ctypes.c_int),
                ("shared_m", ctypes.c_int), ("dtype", ctypes.c_int),
                ("skip_proj", ctypes.c_int),
                ("Wg", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("Wdown", ctypes.c_void_p), ("Wup", ctypes.c_void_p),
                ("W1", ctypes.c_void_p), ("W2", ctypes.c_void_p),
                ("Ws1", ctypes.c_void_p), ("Ws2", ctypes.c_void_p),
                ("route_mode", ctypes.c_int),
                ("expert_fp8", ctypes.c_int), ("W1s", ctypes.c_void_p), ("W2s", ctypes.c_void_p),
                ("expert_fp4", ctypes.c_int), ("W1e", ctypes.c_void_p), ("W2e", ctypes.c_void_p)]

# routing variants (bits of route_mode)
ROUTE_FULL_SOFTMAX, ROUTE_BIAS_SELECT = 1, 2


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            build_oracle()
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L.oracle_router_logits.argtypes = [P, P, P, I, P, I]
        L.oracle_route.argtypes = [P, I, I, I, P, P, P, P, I]
        L.oracle_route_ex.argtypes = [P, P, I, I, I, I, P, P, P, P, I]
        L.oracle_route_ex.restype = I
        L.oracle_forward.argtypes = [P, P, P, I, P, P, P, P, P, I]
        L.oracle_layer.argtypes = [P, P, P, I, P, P, P, P, I]
        for f in (L.oracle_router_logits, L.oracle_route, L.oracle_forward,
                  L.oracle_layer, L.oracle_hardware_threads):
            f.restype = I
        L.oracle_hardware_threads.argtypes = []
        L.oracle_e4m3_value.argtypes = [I]
        L.oracle_e4m3_value.restype = ctypes.c_double
        L.oracle_e2m1_value.argtypes = [I]
        L.oracle_e2m1_value.restype = ctypes.c_double
        _lib = L
    return _lib


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def _host_array(t, dtype: str) -> np.ndarray:
    """C-contiguous numpy view of a CPU tensor / array with the raw bytes of
    the given storage dtype (bf16 travels as uint16)."""
    if t is None:
        return None
    try:
        import torch
        if isinstance(t, torch.Tensor):
            t = t.detach().contiguous().cpu()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16)
            return np.ascontiguousarray(t.numpy())
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    if dtype == "bf16" and a.dtype != np.uint16:
        raise OracleError("bf16 arrays must be passed as uint16 bit patterns")
    return a


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


class OracleLayer:
    """Host copy of one layer's weights, in the API layout [in, out].

    ``W1``/``W2`` are either full stacks ``[N, ...]`` or a mapping
    expert -> matrix holding only the experts that will be reached.  With
    ``W1s``/``W2s`` (per-expert fp32 scales per output column, ``[N, m_in]``
    and ``[N, l]``, stacks or mappings) ``W1``/``W2`` are fp8 E4M3 codes
    (uint8) in the same layouts.  With ``W1e``/``W2e`` (per-expert E8M0
    block exponents, ``[N, m_in, l / 32]`` and ``[N, l, m / 32]``)
    ``W1``/``W2`` are MXFP4 E2M1 code pairs stored output-major,
    ``[N, m_in, l / 2]`` and ``[N, l, m / 2]`` (uint8).
    """

    def __init__(self, *, d, l, N, k, m, act, shared_m=0, dtype="bf16",
                 skip_proj=False, Wg, bias=None, Wdown=None, Wup=None,
                 W1, W2, Ws1=None, Ws2=None, route_mode=0, W1s=None, W2s=None,
                 W1e=None, W2e=None):
        self.d, self.l, self.N, self.k, self.m = d, l, N, k, m
        self.act, self.shared_m, self.dtype, self.skip_proj = act, shared_m, dtype, skip_proj
        keep = []

        def arr(t):
            a = _host_array(t, dtype)
            if a is not None:
                keep.append(a)
            return a

        self._Wg, self._Wdown, self._Wup = arr(Wg), arr(Wdown), arr(Wup)
        self._Ws1, self._Ws2 = arr(Ws1), arr(Ws2)
        self._bias = None
        if bias is not None:
            self._bias = np.ascontiguousarray(_host_array(bias, "f32"), dtype=np.float32)
            keep.append(self._bias)
        fp8 = W1s is not None or W2s is not None
        if fp8 and (W1s is None or W2s is None):
            raise OracleError("fp8 expert weights need both W1s and W2s")
        fp4 = W1e is not None or W2e is not None
        if fp4 and (W1e is None or W2e is None or fp8):
            raise OracleError("fp4 expert weights need both W1e and W2e (and no fp8 scales)")

        def arr8(t):  # E4M3 codes, or fp32 scales
            if t is None:
                return None
            a = _host_array(t, "f32")
            a = np.ascontiguousarray(a, dtype=np.uint8 if a.dtype == np.uint8 else np.float32)
            keep.append(a)
            return a

        warr = arr8 if (fp8 or fp4) else arr
        p1 = (ctypes.c_void_p * N)()
        p2 = (ctypes.c_void_p * N)()
        s1 = (ctypes.c_void_p * N)()
        s2 = (ctypes.c_void_p * N)()
        e1 = (ctypes.c_void_p * N)()
        e2 = (ctypes.c_void_p * N)()
        for e in range(N):
            a1 = self._expert(W1, e, warr)
            a2 = self._expert(W2, e, warr)
            if (fp8 or fp4) and ((a1 is not None and a1.dtype != np.uint8) or
                                 (a2 is not None and a2.dtype != np.uint8)):
                raise OracleError("fp8 / fp4 expert weights must be uint8 codes")
            p1[e] = _ptr(a1)
            p2[e] = _ptr(a2)
            if fp8:
                s1[e] = _ptr(self._expert(W1s, e, arr8))
                s2[e] = _ptr(self._expert(W2s, e, arr8))
            if fp4:
                e1[e] = _ptr(self._expert(W1e, e, arr8))
                e2[e] = _ptr(self._expert(W2e, e, arr8))
        self._p1, self._p2, self._s1, self._s2, self._keep = p1, p2, s1, s2, keep
        self._e1, self._e2 = e1, e2
        self.struct = _Layer(d, l, N, k, m, ACT_CODES[act], shared_m, DTYPE_CODES[dtype],
                             int(bool(skip_proj)), _ptr(self._Wg), _ptr(self._bias),
                             _ptr(self._Wdown), _ptr(self._Wup),
                             ctypes.cast(p1, ctypes.c_void_p), ctypes.cast(p2, ctypes.c_void_p),
                             _ptr(self._Ws1), _ptr(self._Ws2), int(route_mode),
                             int(fp8), ctypes.cast(s1, ctypes.c_void_p),
                             ctypes.cast(s2, ctypes.c_void_p),
                             int(fp4), ctypes.cast(e1, ctypes.c_void_p),
                             ctypes.cast(e2, ctypes.c_void_p))

    @staticmethod
    def _expert(W, e, arr):
        if isinstance(W, dict):
            return arr(W[e]) if e in W else None
        return arr(W[e])

    # --- calls -----------------------------------------------------------
    def router_logits(self, x, tokens: Optional[Sequence[int]] = None,
                      nthreads: Optional[int] = None) -> np.ndarray:
        xa = _host_array(x, self.dtype)
        tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        S = xa.shape[0] if tk is None else tk.shape[0]
        out = np.empty((S, self.N), dtype=np.float64)
        rc = lib().oracle_router_logits(ctypes.byref(self.struct), _ptr(xa), _ptr(tk), S,
                                        _ptr(out), nthreads or default_threads())
        if rc:
            raise OracleError(f"oracle_router_logits failed ({rc})")
        return out

    def forward(self, x, idx, w, tokens: Optional[Sequence[int]] = None,
                nthreads: Optional[int] = None, stages: bool = False):
        xa = _host_array(x, self.dtype)
        tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        S = xa.shape[0] if tk is None else tk.shape[0]
        ia = np.ascontiguousarray(idx, dtype=np.int32).reshape(S, self.k)
        wa = np.ascontiguousarray(w, dtype=np.float64).reshape(S, self.k)
        out = np.empty((S, self.d), dtype=np.float64)
        z = np.empty((S, self.l), dtype=np.float64) if stages else None
        comb = np.empty((S, self.l), dtype=np.float64) if stages else None
        rc = lib().oracle_forward(ctypes.byref(self.struct), _ptr(xa), _ptr(tk), S,
                                  _ptr(ia), _ptr(wa), _ptr(out), _ptr(z), _ptr(comb),
                                  nthreads or default_threads())
        if rc:
            raise OracleError(f"oracle_forward failed ({rc})")
        return (out, z, comb) if stages else out

    def layer(self, x, tokens: Optional[Sequence[int]] = None,
              nthreads: Optional[int] = None) -> Dict[str, np.ndarray]:
        xa = _host_array(x, self.dtype)
        tk = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
        S = xa.shape[0] if tk is None else tk.shape[0]
        out = np.empty((S, self.d), dtype=np.float64)
        lg = np.empty((S, self.N), dtype=np.float32)
        idx = np.empty((S, self.k), dtype=np.int32)
        w = np.empty((S, self.k), dtype=np.float64)
        rc = lib().oracle_layer(ctypes.byref(self.struct), _ptr(xa), _ptr(tk), S, _ptr(out),
                                _ptr(lg), _ptr(idx), _ptr(w), nthreads or default_threads())
        if rc:
            raise OracleError(f"oracle_layer failed ({rc})")
        return {"out": out, "logits32": lg, "idx": idx, "w": w}


def route(logits32, k: int, nthreads: Optional[int] = None, sel_bias=None,
          full_softmax: bool = False):
    """Top-k + gate weights + expert grouping on fp32 logits.

    Default: selection on the logits, softmax renormalised over the k chosen.
    ``sel_bias`` [N] fp32: select on the fp32 sum logits + sel_bias, gates
    from the logits.  ``full_softmax``: gates are the softmax over all N
    logits at the chosen experts.
    Returns (idx [T,k] int32, w [T,k] float64, offsets [N+1], perm [T*k])."""
    lg = np.ascontiguousarray(_host_array(logits32, "f32"), dtype=np.float32)
    T, N = lg.shape
    idx = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    offsets = np.empty(N + 1, dtype=np.int32)
    perm = np.empty(T * k, dtype=np.int32)
    sb = None
    if sel_bias is not None:
        sb = np.ascontiguousarray(_host_array(sel_bias, "f32"), dtype=np.float32)
    if sb is None and not full_softmax:
        rc = lib().oracle_route(_ptr(lg), T, N, k, _ptr(idx), _ptr(w), _ptr(offsets),
                                _ptr(perm), nthreads or default_threads())
    else:
        rc = lib().oracle_route_ex(_ptr(lg), _ptr(sb), T, N, k, int(bool(full_softmax)),
                                   _ptr(idx), _ptr(w), _ptr(offsets), _ptr(perm),
                                   nthreads or default_threads())
    if rc:
        raise OracleError(f"oracle_route failed ({rc})")
    return idx, w, offsets, perm


def e4m3_value(code: int) -> float:
    """The exact value of one fp8 E4M3 code, as the oracle reads it."""
    return float(lib().oracle_e4m3_value(int(code)))


def e2m1_value(code: int) -> float:
    """The exact value of one fp4 E2M1 code, as the oracle reads it."""
    return float(lib().oracle_e2m1_value(int(code)))


def hardware_threads() -> int:
    return int(lib().oracle_hardware_threads())
