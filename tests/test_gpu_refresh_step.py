"""The refresh step in one call (saga_atopn_refresh_step): its compaction
reads the candidates the second radix pass copied out (every logit at or
above the lower edge of the threshold's first-digit bucket) instead of the
stored logits.  Thresholds, kept positions, counts and outputs must be the
same bits as the two-call form (saga_topn_refresh, then saga_atopn_decode
over the same logits), the thresholds the oracle's exact N-th largest of the
GPU's own logits and the kept set the oracle's selection over them."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload

from .gpu_helpers import assert_outputs_close, bits, device_inputs, gpu_logits, mask_from_lists

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

SHAPES = [
    # name, b, hq, hk, hv, d, l, N
    ("llama_like", 2, 32, 4, 8, 64, 3000, 70),
    ("qwen_like", 2, 12, 1, 2, 128, 4097, 100),      # rows not 16-byte aligned: scalar passes
    ("gqa_hk8", 1, 8, 8, 8, 64, 777, 9),
    ("narrow_keys", 2, 16, 2, 8, 32, 2500, 60),
    ("one_row_long", 1, 32, 4, 8, 64, 70000, 900),   # few long rows: the fused decode after the refresh
    ("rows_long", 4, 32, 4, 8, 64, 70000, 900),      # several radix chunks per row; staged gather
    ("ragged_long", 2, 40, 4, 8, 64, 20001, 300),    # several chunks, rows not 16-byte aligned
    ("short", 3, 8, 2, 4, 64, 65, 1),
    ("N_is_l_minus_1", 1, 8, 2, 4, 64, 300, 299),
    ("N_at_least_l", 1, 8, 2, 4, 64, 300, 300),      # every entry kept: stored-logits compaction
]


def _empty(dec):
    w = dec.dims
    out = torch.empty_like(dec.out)
    thresh = torch.empty((w.batch, w.h_q), dtype=torch.float32, device="cuda")
    idx = torch.full((w.batch, w.h_q, w.l_kv), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
    return thresh, out, idx, cnt


def _one_call(dec, q, K, V):
    thresh, out, idx, cnt = _empty(dec)
    _lib.atopn_refresh_step(dec.dims, dec.N, q, K, V, thresh, out, idx, cnt, dec.ws)
    torch.cuda.synchronize()
    assert dec.error() == _lib.SAGA_OK
    return thresh, out, idx, cnt


def _two_calls(dec, q, K, V):
    thresh, out, idx, cnt = _empty(dec)
    _lib.topn_refresh(dec.dims, dec.N, q, K, None, dec.logits, thresh, dec.ws)
    _lib.atopn_decode(dec.dims, q, K, V, thresh, dec.logits, out, idx, cnt, dec.ws)
    torch.cuda.synchronize()
    assert dec.error() == _lib.SAGA_OK
    return thresh, out, idx, cnt


def _fused_after_refresh(dims):
    """Few long rows: the one-call step decodes through the fused path (its
    gather merges the kept entries in another order than the compaction's
    lists, so outputs agree within rounding, not bit for bit)."""
    return dims.batch * dims.h_q <= 64 and dims.l_kv >= 65536


def _same(a, b, what, exact_out=True):
    ta, oa, ia, ca = a
    tb, ob, ib, cb = b
    assert torch.equal(ta.view(torch.int32), tb.view(torch.int32)), f"{what}: thresholds"
    assert torch.equal(ca, cb), f"{what}: counts"
    n = int(ca.max())
    assert torch.equal(ia[..., :n], ib[..., :n]), f"{what}: kept positions"
    if exact_out:
        assert torch.equal(oa, ob), f"{what}: outputs"
    else:
        assert_outputs_close(oa.cpu().numpy(), ob.cpu().numpy(), what)


def _check_against_oracle(dec, q, K, V, got, N, name):
    s = gpu_logits(dec, q, K).cpu().numpy()
    tau_ref = oracle.nth_largest(s, N)
    assert np.array_equal(got[0].cpu().numpy().view(np.int32), tau_ref.view(np.int32)), name
    mask_ref, cnt_ref = oracle.select(s, tau_ref)
    assert np.array_equal(got[3].cpu().numpy(), cnt_ref), name
    assert np.array_equal(mask_from_lists(got[2], got[3], s.shape[-1]), mask_ref), name
    s_o = oracle.logits(bits(q), bits(K), l=s.shape[-1])
    assert_outputs_close(got[1].cpu().numpy(), oracle.attend_masked(s_o, mask_ref, bits(V)), name)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: s[0])
def test_refresh_step_matches_two_calls_and_oracle(shape):
    name, b, hq, hk, hv, d, l, N = shape
    dv = 64 if d == 32 else d
    w = Workload(name, b, hq, hk, hv, d, l, N, 4, steps=2, v_head_dim=dv)
    qs, K, V = device_inputs(w, seed=71)
    dec = AtopNDecoder.for_workload(w)
    for t in range(2):
        one = _one_call(dec, qs[t], K, V)
        two = _two_calls(dec, qs[t], K, V)
        _same(one, two, f"{name} t={t}", exact_out=not _fused_after_refresh(dec.dims))
        _check_against_oracle(dec, qs[t], K, V, one, N, f"{name} t={t}")


def test_refresh_step_with_every_logit_tied():
    """Identical key rows: every logit of a row is equal, the threshold's
    bucket holds the whole row and every position is a candidate."""
    w = Workload("tied", 2, 8, 2, 4, 64, 5000, 40, 4, steps=1)
    qs, K, V = device_inputs(w, seed=73)
    K[:] = K[:, :1]
    dec = AtopNDecoder.for_workload(w)
    one = _one_call(dec, qs[0], K, V)
    _same(one, _two_calls(dec, qs[0], K, V), "tied")
    assert (one[3].cpu().numpy() == w.l_kv).all()
    _check_against_oracle(dec, qs[0], K, V, one, w.N, "tied")


def test_refresh_step_with_zero_queries():
    """A zero query: every logit is +-0, keyed alike; all of them are kept."""
    w = Workload("zeros", 1, 8, 2, 4, 64, 1000, 10, 4, steps=1)
    qs, K, V = device_inputs(w, seed=74)
    qs.zero_()
    dec = AtopNDecoder.for_workload(w)
    one = _one_call(dec, qs[0], K, V)
    _same(one, _two_calls(dec, qs[0], K, V), "zeros")
    assert (one[3].cpu().numpy() == w.l_kv).all()
    _check_against_oracle(dec, qs[0], K, V, one, w.N, "zeros")


def test_decoder_refresh_steps_match_the_oracle_loop():
    """Refresh every 2 steps over 5 steps through AtopNDecoder.step, which
    takes the one-call refresh on refresh steps."""
    w = Workload("loop", 2, 16, 2, 4, 64, 5000, 80, 2, steps=5)
    qs, K, V = device_inputs(w, seed=72)
    dec = AtopNDecoder.for_workload(w)
    Kh, Vh = bits(K), bits(V)
    tau_ref = np.full((w.batch, w.h_q), np.nan, np.float32)
    for t in range(w.steps):
        out = dec.step(t, qs[t], K, V).clone()
        torch.cuda.synchronize()
        assert dec.error() == _lib.SAGA_OK
        o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bits(qs[t]), Kh, Vh, tau_ref, w.N, t, w.n)
        s = gpu_logits(dec, qs[t], K).cpu().numpy()
        if t % w.n == 0:
            assert np.array_equal(dec.thresh.cpu().numpy().view(np.int32),
                                  oracle.nth_largest(s, w.N).view(np.int32)), f"t={t}"
        mask, _ = oracle.select(s, dec.thresh.cpu().numpy())
        assert_outputs_close(out.cpu().numpy(), oracle.attend_masked(s_ref, mask, Vh), f"t={t}")
