"""The C-ABI library: it loads, exports every symbol include/saga.h declares,
and rejects bad arguments on the host before any CUDA call (CPU only)."""
import ctypes
import os
import re

import pytest
import torch

from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200 import build as saga_build
from sparse_decode_attention_saga_b200.workload import CONFIGS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "saga.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIBRARY):
        saga_build.build()
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(saga_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("saga_decode_dense", "saga_topn_refresh", "saga_atopn_decode",
                     "saga_workspace_bytes", "saga_status_string"):
        assert required in names
    assert set(names) == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_debug_library_exports_every_declared_symbol():
    """The bounds-checked build (SAGA_DEBUG) has the same boundary."""
    if not os.path.exists(_lib.DEBUG_LIBRARY):
        saga_build.build(debug=True)
    dbg = ctypes.CDLL(_lib.DEBUG_LIBRARY)
    for name in declared_functions():
        assert hasattr(dbg, name), name


def test_status_strings(lib):
    for code in (0, -1, -2, -3, -4, -5, -6, -7):
        assert _lib.status_string(code) not in ("", "unknown status")
    assert _lib.status_string(-99) == "unknown status"


def _ws(n=1 << 16):
    return torch.zeros(n, dtype=torch.uint8)


@pytest.mark.parametrize("bad,code", [
    (dict(batch=0), _lib.SAGA_ERR_INVALID_ARG),
    (dict(l_kv=0), _lib.SAGA_ERR_INVALID_ARG),
    (dict(l_kv=100, l_cap=99), _lib.SAGA_ERR_INVALID_ARG),
    (dict(head_dim=96), _lib.SAGA_ERR_UNSUPPORTED),
    (dict(h_k=3, h_q=6), _lib.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=6, h_k=4), _lib.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=8, h_v=3), _lib.SAGA_ERR_UNSUPPORTED),
    (dict(h_q=64, h_k=2, h_v=2), _lib.SAGA_ERR_UNSUPPORTED),  # 32 query heads per key head
])
def test_shape_validation(lib, bad, code):
    base = dict(batch=1, h_q=4, h_k=1, h_v=2, head_dim=64, l_kv=64, l_cap=None)
    base.update(bad)
    d = _lib.dims(base["batch"], base["h_q"], base["h_k"], base["h_v"], base["head_dim"],
                  base["l_kv"], base["l_cap"])
    assert _lib.workspace_bytes(d, 8) == 0
    ws = _ws()
    st = lib.saga_atopn_decode(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None,
                               ws.data_ptr(), ws.numel(), None)
    assert st == code


def test_pointer_and_workspace_validation(lib):
    d = _lib.dims(1, 4, 1, 2, 64, 64)
    need = _lib.workspace_bytes(d, 8)
    assert need > 0
    big = _ws(need + 512)
    base = (big.data_ptr() + 255) // 256 * 256
    # null value cache
    assert lib.saga_atopn_decode(ctypes.byref(d), 16, 16, None, 16, None, 16, None, None,
                                 base, need, None) == _lib.SAGA_ERR_INVALID_ARG
    # misaligned key cache
    assert lib.saga_atopn_decode(ctypes.byref(d), 16, 18, 16, 16, None, 16, None, None,
                                 base, need, None) == _lib.SAGA_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert lib.saga_atopn_decode(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None,
                                 base, need - 1, None) == _lib.SAGA_ERR_WORKSPACE
    assert lib.saga_atopn_decode(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None,
                                 base + 8, need, None) == _lib.SAGA_ERR_INVALID_ARG
    # N <= 0
    assert lib.saga_topn_refresh(ctypes.byref(d), 0, 16, 16, None, None, 16, base, need,
                                 None) == _lib.SAGA_ERR_INVALID_ARG
    # dense: more than two value heads per key head only when each value
    # head can stand as a key head of its own (h_v in {1, 2, 4, 8})
    d2 = _lib.dims(1, 12, 2, 6, 64, 64)
    n2 = _lib.workspace_bytes(d2, 8)
    ws2 = _ws(n2 + 512)
    b2 = (ws2.data_ptr() + 255) // 256 * 256
    assert lib.saga_decode_dense(ctypes.byref(d2), 16, 16, 16, 16, b2, n2, None) == \
        _lib.SAGA_ERR_UNSUPPORTED


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
@pytest.mark.parametrize("hq,hk,hv,d,dv", [
    (16, 1, 8, 64, 64),    # SAGA (1, 8): one key head per value head in the dense kernel
    (16, 2, 8, 32, 64),    # Sigma-style 32-dim keys, h_v = 4 h_k
    (16, 4, 8, 32, 64),    # h_v = 2 h_k whose stage (value rows 4x the keys) would not fit twice
    (32, 8, 8, 64, 64),    # dense GQA
])
def test_dense_layouts_pass_validation(lib, hq, hk, hv, d, dv):
    """Every SAGA layout the kernels take is a valid dense call: with no
    device the call gets as far as the device check (arguments, shape and
    workspace size accepted); a workspace too small for the dense kernel's
    own geometry is refused before anything runs."""
    dd = _lib.dims(2, hq, hk, hv, d, 3000, 3000, dv)
    need = _lib.workspace_bytes(dd, 8)
    assert need > 0
    big = _ws(need + 512)
    base = (big.data_ptr() + 255) // 256 * 256
    st = lib.saga_decode_dense(ctypes.byref(dd), 16, 16, 16, 16, base, need, None)
    assert st in (_lib.SAGA_ERR_DEVICE, _lib.SAGA_ERR_CUDA)
    assert lib.saga_decode_dense(ctypes.byref(dd), 16, 16, 16, 16, base, 256, None) == \
        _lib.SAGA_ERR_WORKSPACE


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_valid_call_without_a_device_reports_no_device(lib):
    d = _lib.dims(1, 4, 1, 2, 64, 64)
    need = _lib.workspace_bytes(d, 8)
    big = _ws(need + 512)
    base = (big.data_ptr() + 255) // 256 * 256
    st = lib.saga_atopn_decode(ctypes.byref(d), 16, 16, 16, 16, None, 16, None, None,
                               base, need, None)
    assert st in (_lib.SAGA_ERR_DEVICE, _lib.SAGA_ERR_CUDA)


def test_workspace_sizes_for_every_workload(lib):
    for name, w in CONFIGS.items():
        d = _lib.dims(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, w.l_kv, w.cap, w.dv)
        n = _lib.workspace_bytes(d, w.N)
        assert 0 < n < 4 << 30, name


def test_missing_library_fails_loudly(tmp_path):
    missing = str(tmp_path / "libsaga.so")
    try:
        with pytest.raises(RuntimeError, match="no CPU fallback"):
            _lib.load(missing)
    finally:
        _lib.load(_lib.LIBRARY)


def test_cache_append_validation(lib):
    full = _lib.dims(1, 4, 1, 2, 64, 64, 64)        # l_kv == l_cap: no free row
    assert lib.saga_cache_append(ctypes.byref(full), 16, 16, 16, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    d = _lib.dims(1, 4, 1, 2, 64, 64, 65)
    assert lib.saga_cache_append(ctypes.byref(d), None, 16, 16, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG                   # null new key row
    assert lib.saga_cache_append(ctypes.byref(d), 16, 16, 24, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG                   # misaligned key cache
    bad = _lib.dims(1, 4, 1, 2, 96, 64, 65)
    assert lib.saga_cache_append(ctypes.byref(bad), 16, 16, 16, 16, None) == \
        _lib.SAGA_ERR_UNSUPPORTED


@pytest.mark.parametrize("hk,d,dv,ok", [
    (2, 32, 64, True),     # Sigma-style keys: 32 dims, values 64
    (1, 32, 64, False),    # one key head: a 32 KB tile would need 512 rows
    (2, 32, 128, False),
    (2, 64, 32, False),
    (2, 64, 128, False),
    (2, 128, 0, True),     # 0: values share the key dim
])
def test_value_head_dim_validation(lib, hk, d, dv, ok):
    dims = _lib.dims(1, 16, hk, 8, d, 256, None, dv)
    assert (_lib.workspace_bytes(dims, 8) > 0) == ok


def test_sequence_shard_call_validation(lib):
    d = _lib.dims(1, 4, 1, 2, 64, 64)
    need = _lib.workspace_bytes(d, 8)
    big = _ws(need + 512)
    base = (big.data_ptr() + 255) // 256 * 256
    # radix pass out of range, missing state after pass 0, null histogram
    assert lib.saga_topn_histogram(ctypes.byref(d), 3, 16, 16, 16, None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_topn_histogram(ctypes.byref(d), 1, 16, None, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_topn_histogram(ctypes.byref(d), 0, 16, None, None, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    # N <= 0, pass out of range, null threshold output
    assert lib.saga_topn_select_digit(ctypes.byref(d), 0, 0, 16, 16, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_topn_select_digit(ctypes.byref(d), 8, -1, 16, 16, 16, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_topn_select_digit(ctypes.byref(d), 8, 2, 16, 16, None, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    # the partial decode needs q and k even with stored logits, and a record buffer
    assert lib.saga_atopn_decode_partial(ctypes.byref(d), None, None, 16, 16, 16, 16, base, need,
                                         None) == _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_atopn_decode_partial(ctypes.byref(d), 16, 16, 16, 16, None, None, base, need,
                                         None) == _lib.SAGA_ERR_INVALID_ARG
    # merge: at least one record set, aligned output
    assert lib.saga_merge_partials(ctypes.byref(d), 16, 0, 16, None, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    assert lib.saga_merge_partials(ctypes.byref(d), 16, 2, 18, None, None) == \
        _lib.SAGA_ERR_INVALID_ARG
    # logits: workspace too small
    assert lib.saga_qk_logits(ctypes.byref(d), 16, 16, 16, base, need - 1, None) == \
        _lib.SAGA_ERR_WORKSPACE


def test_host_loop_checks_its_buffers():
    """The host loop refuses host buffers that do not cover its steps or are
    not pinned, before it touches a device."""
    from sparse_decode_attention_saga_b200.decoder import HostLoop
    with pytest.raises(ValueError, match="cover"):
        HostLoop(None, None, None, torch.zeros(4, 2), torch.zeros(2, 2), 0, 3)
    with pytest.raises(ValueError, match="cover"):
        HostLoop(None, None, None, torch.zeros(4, 2), torch.zeros(3, 2), 2, 3)
    with pytest.raises(ValueError, match="cover"):
        HostLoop(None, None, None, torch.zeros(4, 2), torch.zeros(3, 2), 0, 0)
    with pytest.raises(ValueError, match="pinned"):
        HostLoop(None, None, None, torch.zeros(4, 2), torch.zeros(3, 2), 0, 3)
