"""One batch row at a long context (32K and 128K positions, ragged last
tile): every streaming CTA of the fused reuse step holds a slot of the same
row, so each row's kept entries are spread over about 300 per-warp lists and
the gather kernel runs part-major with most parts of a row empty.  Every
step is checked against the oracle, with the mask taken from the list path
of the same step; the edge thresholds (above every logit, and -inf) run at
the same size."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload

from .gpu_helpers import (assert_mask_within_band, assert_outputs_close, bits, device_inputs,
                          gpu_step_with_mask, mask_from_lists, assert_mask_exact)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

SHAPES = [
    # name, hq, hk, hv, d, dv, l (ragged last tile), N
    ("llama_like", 32, 4, 8, 64, 64, 32768 - 37, 300),
    ("narrow_keys", 16, 2, 8, 32, 64, 131072 - 5, 700),
]


def _fused_step(dec, t, q, K, V):
    out = torch.empty_like(dec.out)
    cnt = torch.zeros((1, dec.dims.h_q), dtype=torch.int32, device="cuda")
    dec.step(t, q, K, V, out=out, sel_cnt=cnt)
    return out, cnt


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s[0])
def test_one_row_fused_steps_match_oracle(shape):
    name, hq, hk, hv, d, dv, l, N = shape
    w = Workload(name, 1, hq, hk, hv, d, l, N, 4, steps=6, v_head_dim=dv)
    qs, K, V = device_inputs(w, seed=41)
    Kh, Vh = bits(K), bits(V)
    dec = AtopNDecoder.for_workload(w)
    tau_ref = np.full((1, hq), np.nan, np.float32)
    for t in range(w.steps):
        out_f, cnt_f = _fused_step(dec, t, qs[t], K, V)
        out_l, idx, cnt = gpu_step_with_mask(dec, t, qs[t], K, V)
        torch.cuda.synchronize()
        assert dec.error() == _lib.SAGA_OK
        o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bits(qs[t]), Kh, Vh, tau_ref, N, t, w.n)
        mask_gpu = mask_from_lists(idx, cnt, l)
        assert np.array_equal(cnt_f.cpu().numpy(), cnt.cpu().numpy()), f"t={t}"
        assert_mask_exact(dec, qs[t], K, idx, cnt, what=f"t={t}")
        assert_mask_within_band(mask_gpu, m_ref, s_ref, tau_ref, f"t={t}")
        ref = oracle.attend_masked(s_ref, mask_gpu, Vh)
        assert_outputs_close(out_f.cpu().numpy(), ref, f"t={t} fused")
        assert_outputs_close(out_l.cpu().numpy(), ref, f"t={t} lists")


@pytest.mark.parametrize("case", ["stale_above_all", "keep_everything"])
def test_one_row_fused_edge_thresholds(case):
    name, hq, hk, hv, d, dv, l, N = SHAPES[0]
    w = Workload(name, 1, hq, hk, hv, d, l, N, 4, steps=1, v_head_dim=dv)
    qs, K, V = device_inputs(w, seed=43, steps=1)
    dec = AtopNDecoder.for_workload(w)
    dec.refresh(qs[0], K)
    torch.cuda.synchronize()
    s = dec.logits.cpu().numpy()   # the GPU's logits: the selection is compared bit for bit
    if case == "stale_above_all":   # no logit reaches it: each row keeps its maxima
        tau = s.max(axis=-1) + 1.0
    else:                           # -inf: every position is kept
        tau = np.full((1, hq), -np.inf, np.float32)
    dec.thresh.copy_(torch.from_numpy(tau.astype(np.float32)))
    out_f, cnt_f = _fused_step(dec, 1, qs[0], K, V)
    torch.cuda.synchronize()
    assert dec.error() == _lib.SAGA_OK
    mask, cnt_ref = oracle.select(s, tau.astype(np.float32))
    assert np.array_equal(cnt_f.cpu().numpy(), cnt_ref)
    ref = oracle.attend_masked(s, mask, bits(V))
    assert_outputs_close(out_f.cpu().numpy(), ref, case)
