"""Decode with a growing cache: each step appends its own key and value rows
(saga_cache_append) and attends over l_kv + 1 positions, the thresholds of
the last refresh meeting positions that did not exist when they were
computed.  Every step is checked against the oracle run on the host copy of
the grown cache."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload, make_new_rows

from .gpu_helpers import (assert_mask_within_band, assert_outputs_close, bits, device_inputs,
                          gpu_step_with_mask, mask_from_lists, assert_mask_exact)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _growth_loop(w: Workload, seed: int):
    steps = w.steps
    qs, K, V = device_inputs(w, seed=seed)
    k_new, v_new = (x.cuda() for x in make_new_rows(w, seed))
    dec = AtopNDecoder.for_workload(w)
    Kh, Vh = bits(K).copy(), bits(V).copy()
    tau_ref = np.full((w.batch, w.h_q), np.nan, np.float32)
    for t in range(steps):
        pos = dec.l_kv
        dec.append(k_new[t], v_new[t], K, V)
        Kh[:, pos] = bits(k_new[t])
        Vh[:, pos] = bits(v_new[t])
        l = pos + 1
        assert dec.l_kv == l
        out_f = torch.empty_like(dec.out)
        cnt_f = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
        dec.step(t, qs[t], K, V, out=out_f, sel_cnt=cnt_f)
        out_l, idx, cnt = gpu_step_with_mask(dec, t, qs[t], K, V)
        torch.cuda.synchronize()
        assert dec.error() == _lib.SAGA_OK
        # the cache rows written on the device are exactly the new rows
        assert np.array_equal(bits(K[:, pos]), bits(k_new[t]))
        assert np.array_equal(bits(V[:, pos]), bits(v_new[t]))
        o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bits(qs[t]), Kh, Vh, tau_ref, w.N, t, w.n,
                                                       l=l)
        mask_gpu = mask_from_lists(idx, cnt, l)
        assert np.array_equal(cnt_f.cpu().numpy(), cnt.cpu().numpy()), f"t={t}"
        assert_mask_exact(dec, qs[t], K, idx, cnt, what=f"t={t}")
        assert_mask_within_band(mask_gpu, m_ref, s_ref, tau_ref, f"t={t}")
        ref = oracle.attend_masked(s_ref, mask_gpu, Vh)
        assert_outputs_close(out_l.cpu().numpy(), ref, f"t={t} with positions")
        assert_outputs_close(out_f.cpu().numpy(), ref, f"t={t} fused")
    return dec


@pytest.mark.parametrize("shape", [
    # name, b, hq, hk, hv, d, l0, N, n, steps
    ("llama_like", 2, 32, 4, 8, 64, 700, 20, 4, 9),
    ("qwen_like", 1, 12, 1, 2, 128, 1023, 30, 3, 8),
    ("tile_boundary", 2, 8, 2, 4, 64, 254, 8, 4, 6),  # grows across a tile edge (128-position tiles)
    # 32-position tiles and one refresh: the reuse steps that follow see the
    # tile count (and the workspace's record region) grow without a refresh
    # clearing anything in between
    ("small_tiles_one_refresh", 2, 8, 8, 8, 64, 94, 10, 16, 9),
], ids=lambda s: s[0])
def test_decode_with_cache_growth_matches_oracle(shape):
    name, b, hq, hk, hv, d, l0, N, n, steps = shape
    w = Workload(name, b, hq, hk, hv, d, l0, N, n, steps=steps, l_cap=l0 + steps + 3)
    dec = _growth_loop(w, seed=21)
    assert dec.l_kv == l0 + steps


def test_append_rejects_a_full_cache():
    w = Workload("full", 1, 4, 1, 2, 64, 100, 8, 4, steps=1, l_cap=100)
    qs, K, V = device_inputs(w, seed=0, steps=1)
    k_new, v_new = (x.cuda() for x in make_new_rows(w, 0, steps=1))
    dec = AtopNDecoder.for_workload(w)
    with pytest.raises(_lib.SagaError):
        dec.append(k_new[0], v_new[0], K, V)
    assert dec.l_kv == 100
