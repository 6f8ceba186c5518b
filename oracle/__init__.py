"""CPU oracle for SAGA + Atop-N decode attention (ctypes wrapper).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline / reference leg are the only callers.  The product
path never imports this module and shares no code with it.

Every function follows "More Value per Key: Asymmetric Sparse Attention for
Faster LLM Decoding" (ai.info summary, "Key Contributions" #2-#3, "Main
Findings" first bullet, "Methodology in Plain English" ¶2); the arithmetic is
in ``oracle.cpp`` next to this file, with the readings of the pages it takes.

Arrays: bf16 tensors travel as ``numpy.uint16`` bit patterns, logits and
outputs as ``float32``.  Shapes: q [b,hq,d], K [b,l_cap,hk,d],
V [b,l_cap,hv,dv], logits [b,hq,l], tau [b,hq], out [b,hq,dv] (dv = d except
for the Sigma-style layout with narrower keys, Main Findings "Head count
beats head dimension").
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.cpp")
LIBRARY = os.path.join(_HERE, "liboracle.so")


def compile_library(src: str, out: str) -> str:
    """g++ -O2 -fopenmp shared build of an oracle source file."""
    cmd = ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", src, "-o", out + ".tmp"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` if it is missing or older than its source."""
    stale = (not os.path.exists(LIBRARY)) or os.path.getmtime(LIBRARY) < os.path.getmtime(SOURCE)
    if force or stale:
        compile_library(SOURCE, LIBRARY)
    return LIBRARY


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, "bf16 tensors are passed as uint16 bit patterns"
    return a


class Oracle:
    """The oracle functions bound to one compiled library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        L, P = ctypes.c_long, ctypes.c_void_p
        lib.oracle_logits.argtypes = [L] * 6 + [P, P, P]
        lib.oracle_nth_largest.argtypes = [P, L, L, L, P]
        lib.oracle_nth_largest_sort.argtypes = [P, L, L, L, P]
        lib.oracle_select.argtypes = [P, L, L, P, P, P]
        lib.oracle_attend_masked.argtypes = [L] * 6 + [P, P, P, P]
        lib.oracle_decode_dense.argtypes = [L] * 8 + [P, P, P, P]
        lib.oracle_atopn_step.argtypes = [L] * 11 + [P] * 8
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        for f in (lib.oracle_logits, lib.oracle_nth_largest, lib.oracle_nth_largest_sort,
                  lib.oracle_select, lib.oracle_attend_masked, lib.oracle_decode_dense,
                  lib.oracle_atopn_step):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))

    def logits(self, q, K, hk: int | None = None, l: int | None = None) -> np.ndarray:
        """s[b,i,j] = fp32(sum_c q*K / sqrt(d)) over the first ``l`` positions."""
        q, K = _u16(q), _u16(K)
        b, hq, d = q.shape
        l_cap, hk_ = K.shape[1], K.shape[2]
        assert hk is None or hk == hk_
        l = l_cap if l is None else l
        assert K.shape == (b, l_cap, hk_, d)
        s = np.empty((b, hq, l), np.float32)
        rc = self.lib.oracle_logits(b, hq, hk_, d, l, l_cap, _p(q), _p(K), _p(s))
        assert rc == 0
        return s

    def nth_largest(self, s, N: int) -> np.ndarray:
        """Exact N-th largest of every row (last axis); -inf if N >= l."""
        s = np.ascontiguousarray(s, np.float32)
        l = s.shape[-1]
        rows = s.size // max(l, 1)
        tau = np.empty(s.shape[:-1], np.float32)
        assert self.lib.oracle_nth_largest(_p(s), rows, l, N, _p(tau)) == 0
        return tau

    def nth_largest_sort(self, s, N: int) -> np.ndarray:
        """The same threshold by a full descending sort (brute force)."""
        s = np.ascontiguousarray(s, np.float32)
        l = s.shape[-1]
        rows = s.size // max(l, 1)
        tau = np.empty(s.shape[:-1], np.float32)
        assert self.lib.oracle_nth_largest_sort(_p(s), rows, l, N, _p(tau)) == 0
        return tau

    def select(self, s, tau):
        """mask = s >= min(tau, row max); returns (bool mask, int32 counts)."""
        s = np.ascontiguousarray(s, np.float32)
        tau = np.ascontiguousarray(tau, np.float32)
        l = s.shape[-1]
        rows = s.size // l
        assert tau.size == rows
        mask = np.empty(s.shape, np.uint8)
        cnt = np.empty(s.shape[:-1], np.int32)
        assert self.lib.oracle_select(_p(s), rows, l, _p(tau), _p(mask), _p(cnt)) == 0
        return mask.astype(bool), cnt

    def attend_masked(self, s, mask, V) -> np.ndarray:
        """Softmax over the kept logits and gathered value sum (value head vh(i))."""
        s = np.ascontiguousarray(s, np.float32)
        mask = np.ascontiguousarray(mask, np.uint8)
        V = _u16(V)
        b, hq, l = s.shape
        _, l_cap, hv, d = V.shape
        out = np.empty((b, hq, d), np.float32)
        rc = self.lib.oracle_attend_masked(b, hq, hv, d, l, l_cap, _p(s), _p(mask), _p(V), _p(out))
        assert rc == 0, "attend_masked: a row kept nothing"
        return out

    def decode_dense(self, q, K, V, l: int | None = None) -> np.ndarray:
        """Full attention over the first ``l`` cached positions."""
        q, K, V = _u16(q), _u16(K), _u16(V)
        b, hq, dk = q.shape
        _, l_cap, hk, _ = K.shape
        hv, dv = V.shape[2], V.shape[3]
        l = l_cap if l is None else l
        out = np.empty((b, hq, dv), np.float32)
        rc = self.lib.oracle_decode_dense(b, hq, hk, hv, dk, dv, l, l_cap, _p(q), _p(K), _p(V),
                                          _p(out))
        assert rc == 0
        return out

    def atopn_step(self, q, K, V, tau_state: np.ndarray, N: int, t: int, n: int,
                   l: int | None = None):
        """One Atop-N decode step; ``tau_state`` [b,hq] float32 is updated in
        place on refresh steps (t mod n == 0).  Returns (out, logits, mask, cnt)."""
        q, K, V = _u16(q), _u16(K), _u16(V)
        b, hq, dk = q.shape
        _, l_cap, hk, _ = K.shape
        hv, dv = V.shape[2], V.shape[3]
        l = l_cap if l is None else l
        assert tau_state.dtype == np.float32 and tau_state.shape == (b, hq)
        assert tau_state.flags["C_CONTIGUOUS"]
        out = np.empty((b, hq, dv), np.float32)
        s = np.empty((b, hq, l), np.float32)
        mask = np.empty((b, hq, l), np.uint8)
        cnt = np.empty((b, hq), np.int32)
        rc = self.lib.oracle_atopn_step(b, hq, hk, hv, dk, dv, l, l_cap, N, t, n,
                                        _p(q), _p(K), _p(V), _p(tau_state), _p(out),
                                        _p(s), _p(mask), _p(cnt))
        assert rc == 0
        return out, s, mask.astype(bool), cnt

    def atopn_run(self, qs, K, V, N: int, n: int, l: int | None = None, t0: int = 0,
                  tau_state: np.ndarray | None = None):
        """Steps t0 .. t0+len(qs)-1 of the decode loop; yields per-step results
        (t, out, logits, mask, cnt, tau copy).  A fresh state is only valid if
        the first step refreshes (t0 mod n == 0)."""
        b, hq = qs.shape[1], qs.shape[2]
        tau = np.full((b, hq), np.nan, np.float32) if tau_state is None else tau_state
        for k in range(qs.shape[0]):
            t = t0 + k
            out, s, mask, cnt = self.atopn_step(qs[k], K, V, tau, N, t, n, l)
            yield t, out, s, mask, cnt, tau.copy()


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from ``oracle.cpp`` (compiled on first use)."""
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def __getattr__(name):  # module-level shortcuts: oracle.logits(...), ...
    if name in ("logits", "nth_largest", "nth_largest_sort", "select", "attend_masked",
                "decode_dense", "atopn_step", "atopn_run", "num_threads", "set_num_threads"):
        return getattr(default(), name)
    raise AttributeError(name)
