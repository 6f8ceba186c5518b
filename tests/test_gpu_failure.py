"""Failure detection on the GPU without a fault: a bounded device wait that
runs out (a barrier nothing completes) is reported through the workspace's
sticky flag, and the context keeps working afterwards."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload, bf16_bits, make_cache, make_queries

from .gpu_helpers import assert_outputs_close

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_bounded_wait_timeout_is_reported_and_context_survives():
    w = Workload("fail", 1, 8, 2, 4, 64, 700, 20, 4, steps=2)
    K, V = make_cache(w, 1, "cuda")
    qs = make_queries(w, 1, "cuda")
    dec = AtopNDecoder.for_workload(w)
    assert dec.error() == _lib.SAGA_OK
    _lib.selftest_wait_timeout(dec.ws, 20000)       # 20 ms limit
    assert dec.error() == _lib.SAGA_ERR_TIMEOUT     # read and cleared
    assert dec.error() == _lib.SAGA_OK
    out = dec.step(0, qs[0], K, V).cpu().numpy()    # the context still works
    assert dec.error() == _lib.SAGA_OK
    tau = np.full((1, w.h_q), np.nan, np.float32)
    ref, *_ = oracle.atopn_step(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V), tau, w.N, 0, w.n)
    assert_outputs_close(out, ref, "after timeout")


def test_selftest_rejects_bad_limits():
    ws = torch.zeros(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(_lib.SagaError):
        _lib.selftest_wait_timeout(ws, 0)
    with pytest.raises(_lib.SagaError):
        _lib.selftest_wait_timeout(ws, 2_000_000)
