"""ctypes binding of ``libsaga.so`` (include/saga.h): argument marshalling only.

Every function here forwards to the C entry point of the same name, passing
device pointers (``tensor.data_ptr()``) and the current CUDA stream; all work
runs in the library's kernels.  A missing library raises immediately: there
is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# The bounds-checked build (SAGA_DEBUG) sits beside the release one; the
# SAGA_LIBRARY environment variable picks the library a process loads.
RELEASE_LIBRARY = os.path.join(_HERE, "libsaga.so")
DEBUG_LIBRARY = os.path.join(_HERE, "libsaga_debug.so")
LIBRARY = os.environ.get("SAGA_LIBRARY") or RELEASE_LIBRARY

SAGA_OK = 0
SAGA_ERR_INVALID_ARG = -1
SAGA_ERR_UNSUPPORTED = -2
SAGA_ERR_WORKSPACE = -3
SAGA_ERR_CUDA = -4
SAGA_ERR_DEVICE = -5
SAGA_ERR_TIMEOUT = -6
SAGA_ERR_BOUNDS = -7

EXPORTS = (
    "saga_workspace_bytes", "saga_decode_dense", "saga_topn_refresh", "saga_atopn_decode",
    "saga_workspace_reset", "saga_workspace_error", "saga_status_string", "saga_launch_count",
    "saga_set_kernel_events", "saga_version", "saga_topn_refresh_noalloc",
    "saga_selftest_wait_timeout", "saga_cache_append", "saga_qk_logits", "saga_topn_histogram",
    "saga_topn_select_digit", "saga_atopn_decode_partial", "saga_merge_partials",
    "saga_atopn_refresh_step", "saga_workspace_empty_rows",
)


class SagaDims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("h_q", ctypes.c_int32), ("h_k", ctypes.c_int32),
                ("h_v", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("l_kv", ctypes.c_int32),
                ("l_cap", ctypes.c_int32), ("v_head_dim", ctypes.c_int32)]


class SagaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {status_string(status)} ({status})")
        self.status = status


_lib = None
_path = LIBRARY


def load(path: str | None = None):
    """Loads the library (once); raises if it has not been built."""
    global _lib, _path
    if path is not None and path != _path:
        _lib, _path = None, path
    if _lib is None:
        if not os.path.exists(_path):
            raise RuntimeError(
                f"{_path} is missing: build it with `python -m sparse_decode_attention_saga_b200.build` "
                "(the CUDA library is required; there is no CPU fallback)")
        lib = ctypes.CDLL(_path)
        P, I32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        D = ctypes.POINTER(SagaDims)
        lib.saga_workspace_bytes.argtypes = [D, I32]
        lib.saga_workspace_bytes.restype = SZ
        lib.saga_decode_dense.argtypes = [D, P, P, P, P, P, SZ, P]
        lib.saga_topn_refresh.argtypes = [D, I32, P, P, P, P, P, P, SZ, P]
        lib.saga_atopn_decode.argtypes = [D, P, P, P, P, P, P, P, P, P, SZ, P]
        lib.saga_atopn_refresh_step.argtypes = [D, I32, P, P, P, P, P, P, P, P, SZ, P]
        lib.saga_topn_refresh_noalloc.argtypes = [D, I32, P, P, P]
        lib.saga_topn_refresh_noalloc.restype = ctypes.c_int
        lib.saga_cache_append.argtypes = [D, P, P, P, P, P]
        lib.saga_cache_append.restype = ctypes.c_int
        lib.saga_selftest_wait_timeout.argtypes = [P, SZ, ctypes.c_uint32, P]
        lib.saga_selftest_wait_timeout.restype = ctypes.c_int
        lib.saga_workspace_reset.argtypes = [P, SZ, P]
        lib.saga_workspace_error.argtypes = [P, SZ, P]
        lib.saga_workspace_empty_rows.argtypes = [P, SZ, ctypes.POINTER(ctypes.c_uint64), P]
        lib.saga_workspace_empty_rows.restype = ctypes.c_int
        lib.saga_status_string.argtypes = [ctypes.c_int]
        lib.saga_status_string.restype = ctypes.c_char_p
        lib.saga_launch_count.restype = ctypes.c_uint64
        lib.saga_set_kernel_events.argtypes = [P, P]
        lib.saga_set_kernel_events.restype = None
        lib.saga_qk_logits.argtypes = [D, P, P, P, P, SZ, P]
        lib.saga_topn_histogram.argtypes = [D, I32, P, P, P, P]
        lib.saga_topn_select_digit.argtypes = [D, I32, I32, P, P, P, P]
        lib.saga_atopn_decode_partial.argtypes = [D, P, P, P, P, P, P, P, SZ, P]
        lib.saga_merge_partials.argtypes = [D, P, I32, P, P, P]
        for f in ("saga_decode_dense", "saga_topn_refresh", "saga_atopn_decode", "saga_atopn_refresh_step",
                  "saga_workspace_reset", "saga_workspace_error", "saga_version", "saga_qk_logits",
                  "saga_topn_histogram", "saga_topn_select_digit", "saga_atopn_decode_partial",
                  "saga_merge_partials"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(fn: str, status: int) -> None:
    if status != SAGA_OK:
        raise SagaError(fn, status)


def dims(batch, h_q, h_k, h_v, head_dim, l_kv, l_cap=None, v_head_dim=None) -> SagaDims:
    """head_dim is the key (and query) head dim; v_head_dim the value head dim
    (None: the same)."""
    return SagaDims(batch, h_q, h_k, h_v, head_dim, l_kv, l_kv if l_cap is None else l_cap,
                    0 if v_head_dim is None else v_head_dim)


def status_string(status: int) -> str:
    return load().saga_status_string(int(status)).decode()


def workspace_bytes(d: SagaDims, N: int) -> int:
    return int(load().saga_workspace_bytes(ctypes.byref(d), int(N)))


def decode_dense(d, q, k, v, out, ws, stream=None) -> None:
    st = load().saga_decode_dense(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("saga_decode_dense", st)


def topn_refresh(d, N, q, k, logits_in, logits_out, thresh_out, ws, stream=None) -> None:
    st = load().saga_topn_refresh(ctypes.byref(d), int(N), _ptr(q), _ptr(k), _ptr(logits_in),
                                  _ptr(logits_out), _ptr(thresh_out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream))
    _check("saga_topn_refresh", st)


def atopn_decode(d, q, k, v, thresh, logits_in, out, sel_idx, sel_cnt, ws, stream=None) -> None:
    st = load().saga_atopn_decode(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(thresh),
                                  _ptr(logits_in), _ptr(out), _ptr(sel_idx), _ptr(sel_cnt),
                                  _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("saga_atopn_decode", st)


def topn_refresh_noalloc(d, N, logits_in, thresh_out, stream=None) -> None:
    """Threshold refresh without a workspace (scratch is a fixed array inside
    the library); for callers that cannot allocate device memory."""
    st = load().saga_topn_refresh_noalloc(ctypes.byref(d), int(N), _ptr(logits_in),
                                          _ptr(thresh_out), _stream(stream))
    _check("saga_topn_refresh_noalloc", st)


def cache_append(d, k_new, v_new, k, v, stream=None) -> None:
    """Write this step's new key/value rows at position d.l_kv of the caches."""
    _check("saga_cache_append",
           load().saga_cache_append(ctypes.byref(d), _ptr(k_new), _ptr(v_new), _ptr(k), _ptr(v),
                                    _stream(stream)))


# ---- sequence shards (one rank's calls; the cross-rank sums are the caller's)

def qk_logits(d, q, k, logits_out, ws, stream=None) -> None:
    _check("saga_qk_logits",
           load().saga_qk_logits(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(logits_out), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)))


def topn_histogram(d, pass_: int, logits, state, hist, stream=None) -> None:
    _check("saga_topn_histogram",
           load().saga_topn_histogram(ctypes.byref(d), int(pass_), _ptr(logits), _ptr(state),
                                      _ptr(hist), _stream(stream)))


def topn_select_digit(d, N: int, pass_: int, hist, state, thresh_out, stream=None) -> None:
    _check("saga_topn_select_digit",
           load().saga_topn_select_digit(ctypes.byref(d), int(N), int(pass_), _ptr(hist),
                                         _ptr(state), _ptr(thresh_out), _stream(stream)))


def atopn_refresh_step(d, N, q, k, v, thresh_out, out, sel_idx, sel_cnt, ws, stream=None) -> None:
    st = load().saga_atopn_refresh_step(ctypes.byref(d), int(N), _ptr(q), _ptr(k), _ptr(v),
                                        _ptr(thresh_out), _ptr(out), _ptr(sel_idx), _ptr(sel_cnt),
                                        _ptr(ws), ws.numel() * ws.element_size(), _stream(stream))
    _check("saga_atopn_refresh_step", st)


def atopn_decode_partial(d, q, k, v, thresh, logits_in, part, ws, stream=None) -> None:
    _check("saga_atopn_decode_partial",
           load().saga_atopn_decode_partial(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(thresh), _ptr(logits_in), _ptr(part), _ptr(ws),
                                            ws.numel() * ws.element_size(), _stream(stream)))


def merge_partials(d, parts, R: int, out, sel_cnt=None, stream=None) -> None:
    _check("saga_merge_partials",
           load().saga_merge_partials(ctypes.byref(d), _ptr(parts), int(R), _ptr(out),
                                      _ptr(sel_cnt), _stream(stream)))


def selftest_wait_timeout(ws, limit_us: int, stream=None) -> None:
    """Make a bounded device wait run out on purpose (sets the timeout flag)."""
    _check("saga_selftest_wait_timeout",
           load().saga_selftest_wait_timeout(_ptr(ws), ws.numel() * ws.element_size(),
                                             int(limit_us), _stream(stream)))


def workspace_reset(ws, stream=None) -> None:
    _check("saga_workspace_reset",
           load().saga_workspace_reset(_ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))


def workspace_error(ws, stream=None) -> int:
    return int(load().saga_workspace_error(_ptr(ws), ws.numel() * ws.element_size(),
                                           _stream(stream)))


def workspace_empty_rows(ws, stream=None) -> int:
    """Rows that took the empty-set rule since the last read (read and cleared)."""
    n = ctypes.c_uint64(0)
    _check("saga_workspace_empty_rows",
           load().saga_workspace_empty_rows(_ptr(ws), ws.numel() * ws.element_size(), ctypes.byref(n),
                                            _stream(stream)))
    return int(n.value)


def launch_count() -> int:
    return int(load().saga_launch_count())


def set_kernel_events(start=None, stop=None) -> None:
    """``start``/``stop`` are torch.cuda.Event objects (or None to clear)."""
    s = None if start is None else start.cuda_event
    e = None if stop is None else stop.cuda_event
    load().saga_set_kernel_events(s, e)


def version() -> int:
    return int(load().saga_version())
