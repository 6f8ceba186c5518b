"""The allocation-free threshold refresh, saga_topn_refresh_noalloc.

Some callers cannot hand the library a workspace because they may not
allocate device memory on the decode path (a plugin inside an engine that
owns all device memory; a loop that must not call cudaMalloc after start-up).
For them the radix select keeps its scratch in a fixed array inside the
library.  These tests call that entry point through the C ABI and check that
it returns the same thresholds as the workspace entry point
(saga_topn_refresh with stored logits) on two calls in a row, bit for bit:
the scratch left by the first call must not leak into the second.
"""
import ctypes

import pytest
import torch

from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload, make_cache, make_queries

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _noalloc(lib, dims, N, logits, out):
    return lib.saga_topn_refresh_noalloc(ctypes.byref(dims), int(N), logits.data_ptr(),
                                         out.data_ptr(), torch.cuda.current_stream().cuda_stream)


def test_noalloc_refresh_matches_workspace_refresh_on_two_calls():
    lib = _lib.load()
    w = Workload("noalloc", 2, 32, 4, 8, 64, 6000, 150, 4, steps=2)
    K, V = make_cache(w, 3, "cuda")
    qs = make_queries(w, 3, "cuda")
    dec = AtopNDecoder.for_workload(w)
    for call, N in enumerate((150, 37)):
        dec.refresh(qs[call], K)               # logits of this call's query
        ref = torch.empty((w.batch, w.h_q), dtype=torch.float32, device="cuda")
        _lib.topn_refresh(dec.dims, N, None, None, dec.logits, None, ref, dec.ws)
        got = torch.full((w.batch, w.h_q), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, dec.dims, N, dec.logits, got) == _lib.SAGA_OK
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32)), f"call {call}"


def test_noalloc_refresh_keeps_everything_when_N_covers_the_cache():
    lib = _lib.load()
    d = _lib.dims(1, 8, 2, 2, 64, 100)
    logits = torch.randn(1, 8, 100, device="cuda")
    got = torch.zeros(1, 8, device="cuda")
    assert _noalloc(lib, d, 100, logits, got) == _lib.SAGA_OK
    torch.cuda.synchronize()
    assert torch.all(got == float("-inf"))


def test_noalloc_refresh_rejects_shapes_beyond_its_scratch():
    lib = _lib.load()
    d = _lib.dims(683, 1, 1, 1, 64, 16)       # 683 rows > 682 the fixed scratch holds
    logits = torch.zeros(683, 1, 16, device="cuda")
    got = torch.full((683, 1), 7.0, device="cuda")
    assert _noalloc(lib, d, 4, logits, got) == _lib.SAGA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(got == 7.0)               # nothing was enqueued
