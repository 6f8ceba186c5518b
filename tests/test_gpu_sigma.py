"""Keys narrower than values: the pages' Sigma-style head layout ((h_k, d_k)
= (2, 32) next to h_v = 8, d_v = 64; Main Findings, "Head count beats head
dimension").  The decode loop (refresh and reuse steps), the dense baseline
and cache growth against the oracle."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload

from .gpu_helpers import assert_outputs_close, bits, device_inputs
from .test_gpu_growth import _growth_loop
from .test_gpu_parity import run_loop_and_compare

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

SIGMA = [
    # name, b, hq, hk, hv, l, cap
    ("sigma_smollm", 2, 16, 2, 8, 3000, None),     # SmolLM2-360M-like: h_q 16
    ("sigma_ragged", 1, 16, 2, 8, 777, 800),
    ("sigma_g16", 1, 32, 2, 8, 1100, None),         # 16 query heads per key head
    ("sigma_hk4", 2, 16, 4, 8, 999, None),          # two value heads per key head
]


def _w(name, b, hq, hk, hv, l, cap, N=None, n=4, steps=9):
    N = max(1, l // 40) if N is None else N
    return Workload(name, b, hq, hk, hv, 32, l, N, n, steps=steps, l_cap=cap, v_head_dim=64)


@pytest.mark.parametrize("s", SIGMA, ids=lambda s: s[0])
def test_sigma_decode_loop_matches_oracle(s):
    run_loop_and_compare(_w(*s), seed=31)


@pytest.mark.parametrize("s", SIGMA, ids=lambda s: s[0])
def test_sigma_full_attention_matches_oracle_dense(s):
    """N >= l keeps everything: full attention, against the oracle's, and the
    dense kernel (four value heads per key head: one key head per value head,
    each reading its key head's rows) against the same."""
    name, b, hq, hk, hv, l, _ = s
    w = _w(name, b, hq, hk, hv, min(l, 400), None, N=400, steps=1)
    qs, K, V = device_inputs(w, seed=33, steps=1)
    dec = AtopNDecoder.for_workload(w)
    out_a = dec.step(0, qs[0], K, V).clone()
    out_d = dec.dense(qs[0], K, V).clone()
    torch.cuda.synchronize()
    ref = oracle.decode_dense(bits(qs[0]), bits(K), bits(V))
    assert_outputs_close(out_a.cpu().numpy(), ref, "N >= l")
    assert_outputs_close(out_d.cpu().numpy(), ref, "dense")
    assert dec.error() == _lib.SAGA_OK


def test_narrow_keys_dense_where_it_fits():
    """Dense with 32-dim keys and one value head per key head (h_k = h_v)."""
    w = Workload("narrow_gqa", 2, 16, 4, 4, 32, 1500, 40, 4, steps=1, v_head_dim=64)
    qs, K, V = device_inputs(w, seed=35, steps=1)
    dec = AtopNDecoder.for_workload(w)
    out = dec.dense(qs[0], K, V)
    torch.cuda.synchronize()
    ref = oracle.decode_dense(bits(qs[0]), bits(K), bits(V))
    assert_outputs_close(out.cpu().numpy(), ref, "dense, narrow keys")
    assert dec.error() == _lib.SAGA_OK


def test_sigma_cache_growth():
    w = Workload("sigma_grow", 2, 16, 2, 8, 32, 510, 12, 3, steps=7, l_cap=520, v_head_dim=64)
    assert _growth_loop(w, seed=34).l_kv == 517
