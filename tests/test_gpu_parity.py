"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Small shapes span several 32 KB tiles and a ragged tail; the full-size
workloads are checked on sampled batch elements.  Thresholds and masks are
bit-exact on identical logits; end-to-end masks may differ only inside the
1e-4|tau| band; outputs agree to 1e-3 + 1e-3|o| (see gpu_helpers).
"""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import CONFIGS, Workload

from .gpu_helpers import (LOGIT_ATOL, LOGIT_RTOL, assert_mask_exact, assert_mask_within_band,
                          assert_outputs_close, bits, device_inputs, gpu_logits, gpu_step_with_mask,
                          mask_from_lists)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

SHAPES = [
    # name, b, hq, hk, hv, d, l, cap
    ("tiny", 1, 4, 1, 2, 64, 2048, None),
    ("qwen_like_ragged", 2, 12, 1, 2, 128, 1000, 1100),
    ("llama_like_ragged", 2, 32, 4, 8, 64, 777, None),
    ("gqa_hk8", 1, 8, 8, 8, 64, 300, 333),
    ("g8_d128_hk2", 2, 16, 2, 4, 128, 513, None),
    ("g16_two_ntiles", 1, 16, 1, 16, 64, 1100, None),
    ("g3_d128", 3, 6, 2, 2, 128, 4097, None),
    ("saga_1_8", 2, 16, 1, 8, 64, 3000, None),
    # h_q > 32: the reuse step takes the list path (compare kernel, gather, combine)
    ("hq64_lists", 2, 64, 4, 8, 64, 1500, None),
    # more rows than two per SM: the compare kernel's 4-wide form (the shapes
    # above take its 16-wide form for few rows)
    ("rows_320", 10, 32, 4, 8, 64, 1000, None),
]


def wl(name, b, hq, hk, hv, d, l, cap, N=None, n=4, steps=6):
    N = max(1, l // 40) if N is None else N
    return Workload(name, b, hq, hk, hv, d, l, N, n, steps=steps, l_cap=cap)


@pytest.fixture(params=SHAPES, ids=[s[0] for s in SHAPES])
def shape(request):
    return wl(*request.param)


# ---------------------------------------------------------------- logits (a1)

def test_logits_match_oracle(shape):
    w = shape
    qs, K, V = device_inputs(w, seed=1, steps=2)
    dec = AtopNDecoder.for_workload(w)
    dec.refresh(qs[0], K)
    torch.cuda.synchronize()
    s_gpu = dec.logits.cpu().numpy()
    s_ref = oracle.logits(bits(qs[0]), bits(K), l=w.l_kv)
    err = np.abs(s_gpu.astype(np.float64) - s_ref)
    assert np.all(err <= LOGIT_ATOL + LOGIT_RTOL * np.abs(s_ref)), f"max logit error {err.max():.3g}"
    assert dec.error() == _lib.SAGA_OK


# ---------------------------------------------------------------- threshold (a2)

def _thresholds(w, logits: torch.Tensor, N):
    dec = AtopNDecoder(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, w.l_kv, N, w.n, w.cap)
    tau = torch.empty((w.batch, w.h_q), dtype=torch.float32, device="cuda")
    _lib.topn_refresh(dec.dims, N, None, None, logits, None, tau, dec.ws)
    torch.cuda.synchronize()
    return tau.cpu().numpy()


@pytest.mark.parametrize("which", ["gpu_logits", "tied_logits"])
def test_threshold_bit_exact_on_identical_logits(shape, which):
    w = shape
    if which == "gpu_logits":
        qs, K, V = device_inputs(w, seed=2, steps=1)
        dec = AtopNDecoder.for_workload(w)
        dec.refresh(qs[0], K)
        logits = dec.logits.clone()
    else:
        g = torch.Generator(device="cuda").manual_seed(3)
        logits = (torch.randint(-8, 9, (w.batch, w.h_q, w.l_kv), generator=g, device="cuda")
                  .float() * 0.25)
        logits[..., ::7] = -0.0
    host = logits.cpu().numpy()
    for N in sorted({1, 7, w.l_kv // 3, w.l_kv - 1, w.l_kv, w.l_kv + 5} - {0}):
        tau_gpu = _thresholds(w, logits, N)
        tau_ref = oracle.nth_largest(host, N)
        assert np.array_equal(tau_gpu.view(np.int32), tau_ref.view(np.int32)), f"N={N}"


# ---------------------------------------------------------------- mask (a3) + output (a4, a5)

def test_mask_bit_exact_and_output_given_mask(shape):
    w = shape
    qs, K, V = device_inputs(w, seed=4, steps=2)
    dec = AtopNDecoder.for_workload(w)
    out, idx, cnt = gpu_step_with_mask(dec, 0, qs[0], K, V)   # refresh step
    s = gpu_logits(dec, qs[0], K).cpu().numpy()
    tau = dec.thresh.cpu().numpy()
    mask_gpu = mask_from_lists(idx, cnt, w.l_kv)
    mask_ref, cnt_ref = oracle.select(s, tau)
    assert np.array_equal(mask_gpu, mask_ref)
    assert np.array_equal(cnt.cpu().numpy(), cnt_ref)
    assert np.all(cnt_ref >= min(w.N, w.l_kv))
    ref = oracle.attend_masked(s, mask_gpu, bits(V))
    assert_outputs_close(out.cpu().numpy(), ref, "refresh-step output")


@pytest.mark.parametrize("pick", ["rank_N", "random"])
def test_fused_mask_exact_at_threshold_boundaries(shape, pick):
    """Thresholds equal to one of the row's logits, or one ulp above or below
    it: the fused kernel compares the raw tensor-core accumulator with a
    threshold mapped back through the 1/sqrt(d) scale, and must keep exactly
    what comparing the scaled logits keeps (head dim 128: the scale is not a
    power of two)."""
    w = shape
    qs, K, V = device_inputs(w, seed=13, steps=1)
    dec = AtopNDecoder.for_workload(w)
    s = gpu_logits(dec, qs[0], K)
    torch.cuda.synchronize()
    sh = s.cpu().numpy()
    if pick == "rank_N":
        j = np.minimum(w.N, w.l_kv) - 1
        base = -np.sort(-sh, axis=-1)[..., j]
    else:
        rng = np.random.default_rng(w.l_kv)
        j = rng.integers(0, w.l_kv, size=(w.batch, w.h_q))
        base = np.take_along_axis(sh, j[..., None], -1)[..., 0]
    s_ref = oracle.logits(bits(qs[0]), bits(K), l=w.l_kv)
    for kind, tau in (("at", base), ("above", np.nextafter(base, np.float32(np.inf))),
                      ("below", np.nextafter(base, np.float32(-np.inf)))):
        tau = tau.astype(np.float32)
        dec.thresh.copy_(torch.from_numpy(tau))
        out = torch.empty_like(dec.out)
        idx = torch.full((w.batch, w.h_q, w.l_kv), -1, dtype=torch.int32, device="cuda")
        cnt = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
        _lib.atopn_decode(dec.dims, qs[0], K, V, dec.thresh, None, out, idx, cnt, dec.ws)
        torch.cuda.synchronize()
        mask_ref, cnt_ref = oracle.select(sh, tau)
        assert np.array_equal(cnt.cpu().numpy(), cnt_ref), kind
        mask_gpu = mask_from_lists(idx, cnt, w.l_kv)
        assert np.array_equal(mask_gpu, mask_ref), f"{kind}: {(mask_gpu != mask_ref).sum()} differ"
        assert_outputs_close(out.cpu().numpy(), oracle.attend_masked(s_ref, mask_gpu, bits(V)), kind)
    assert dec.error() == _lib.SAGA_OK


def test_stale_threshold_above_every_logit_keeps_the_maxima(shape):
    w = shape
    qs, K, V = device_inputs(w, seed=5, steps=2)
    dec = AtopNDecoder.for_workload(w)
    dec.refresh(qs[0], K)
    torch.cuda.synchronize()
    s = dec.logits.cpu().numpy()
    dec.thresh.copy_(torch.from_numpy(s.max(-1) + 1.0))
    assert dec.empty_rows() == 0
    # fused path (fallback in the combine kernel)
    out_fused = torch.empty_like(dec.out)
    cnt_fused = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
    idx_fused = torch.full((w.batch, w.h_q, w.l_kv), -1, dtype=torch.int32, device="cuda")
    _lib.atopn_decode(dec.dims, qs[0], K, V, dec.thresh, None, out_fused, idx_fused, cnt_fused,
                      dec.ws)
    rows = w.batch * w.h_q
    assert dec.empty_rows() == rows   # every row took the rule, counted once
    # stored-logits path
    out_l, idx, cnt = torch.empty_like(dec.out), None, None
    idx = torch.full((w.batch, w.h_q, w.l_kv), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
    _lib.atopn_decode(dec.dims, None, None, V, dec.thresh, dec.logits, out_l, idx, cnt, dec.ws)
    torch.cuda.synchronize()
    assert dec.empty_rows() == rows
    mask_ref, cnt_ref = oracle.select(s, dec.thresh.cpu().numpy())
    assert np.array_equal(mask_from_lists(idx, cnt, w.l_kv), mask_ref)
    assert np.array_equal(cnt_fused.cpu().numpy(), cnt_ref)
    assert np.array_equal(mask_from_lists(idx_fused, cnt_fused, w.l_kv), mask_ref)
    ref = oracle.attend_masked(s, mask_ref, bits(V))
    assert_outputs_close(out_l.cpu().numpy(), ref, "stored-logits fallback")
    assert_outputs_close(out_fused.cpu().numpy(), ref, "fused fallback")
    assert dec.error() == _lib.SAGA_OK


# ---------------------------------------------------------------- whole loop

def run_loop_and_compare(w, seed=0, gen_device="cuda", rows=None):
    """Steps 0..steps-1 on the GPU and in the oracle; returns the number of
    in-band mask flips.  Each step runs twice: without and with the kept
    positions emitted.  On reuse steps both runs take the fused path (the
    on-chip compare of the streaming kernel), on refresh steps the one-call
    refresh step (its candidate compaction); either way the emitted mask is
    checked bit for bit
    against the oracle's selection over the GPU's own logits, and against
    the oracle's end-to-end step within the band."""
    qs, K, V = device_inputs(w, seed, gen_device=gen_device)
    dec = AtopNDecoder.for_workload(w)
    b_sel = list(range(w.batch)) if rows is None else rows
    Kh = bits(K[b_sel])
    Vh = bits(V[b_sel])
    tau_ref = np.full((len(b_sel), w.h_q), np.nan, np.float32)
    flips = 0
    for t in range(w.steps):
        out_fused = torch.empty_like(dec.out)
        cnt_fused = torch.zeros((w.batch, w.h_q), dtype=torch.int32, device="cuda")
        dec.step(t, qs[t], K, V, out=out_fused, sel_cnt=cnt_fused)
        out_l, idx, cnt = gpu_step_with_mask(dec, t, qs[t], K, V)
        torch.cuda.synchronize()
        assert dec.error() == _lib.SAGA_OK
        o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bits(qs[t][b_sel]), Kh, Vh, tau_ref,
                                                       w.N, t, w.n, l=w.l_kv)
        mask_gpu = mask_from_lists(idx[b_sel], cnt[b_sel], w.l_kv)
        # the same kernels decide the output whether or not the positions are emitted
        assert np.array_equal(cnt_fused[b_sel].cpu().numpy(), cnt[b_sel].cpu().numpy()), f"t={t}"
        if not dec.is_refresh(t):
            assert torch.equal(out_fused, out_l), f"t={t}: emitting positions changed the output"
        assert_mask_exact(dec, qs[t], K, idx, cnt, b_sel, f"t={t}")
        flips += assert_mask_within_band(mask_gpu, m_ref, s_ref, tau_ref, f"t={t}")
        ref = oracle.attend_masked(s_ref, mask_gpu, Vh)
        assert_outputs_close(out_l[b_sel].cpu().numpy(), ref, f"t={t} with positions")
        assert_outputs_close(out_fused[b_sel].cpu().numpy(), ref, f"t={t} fused")
    return flips


def test_decode_loop_matches_oracle(shape):
    run_loop_and_compare(shape.scaled(steps=9, n=4), seed=6)


def test_tiny_workload_32_steps():
    run_loop_and_compare(CONFIGS["tiny"], seed=0)


def test_refresh_every_step_is_exact_topN():
    w = wl("n1", 2, 8, 2, 4, 64, 900, None, N=30, n=1, steps=3)
    run_loop_and_compare(w, seed=7)


# ---------------------------------------------------------------- dense (a7)

@pytest.mark.parametrize("s", [x for x in SHAPES if x[4] <= 2 * x[3] or x[4] in (4, 8)],
                         ids=lambda x: x[0])
def test_dense_matches_oracle(s):
    w = wl(*s)
    qs, K, V = device_inputs(w, seed=8, steps=1)
    dec = AtopNDecoder.for_workload(w)
    out = dec.dense(qs[0], K, V)
    torch.cuda.synchronize()
    ref = oracle.decode_dense(bits(qs[0]), bits(K), bits(V), l=w.l_kv)
    assert_outputs_close(out.cpu().numpy(), ref, "dense")
    assert dec.error() == _lib.SAGA_OK


def test_N_at_least_l_equals_dense():
    w = wl("full", 1, 8, 2, 4, 64, 500, None, N=500, n=4, steps=2)
    qs, K, V = device_inputs(w, seed=9, steps=2)
    dec = AtopNDecoder.for_workload(w)
    out_a = dec.step(0, qs[0], K, V).clone()
    assert np.all(dec.thresh.cpu().numpy() == -np.inf)
    out_d = dec.dense(qs[0], K, V).clone()
    torch.cuda.synchronize()
    ref = oracle.decode_dense(bits(qs[0]), bits(K), bits(V))
    assert_outputs_close(out_a.cpu().numpy(), ref, "N>=l")
    assert_outputs_close(out_d.cpu().numpy(), ref, "dense")


# ---------------------------------------------------------------- edge cases

@pytest.mark.parametrize("l", [1, 2, 15, 16, 17, 33, 255, 257])
@pytest.mark.parametrize("N", [1, 5, 10**6])
def test_short_and_ragged_caches(l, N):
    w = wl("edge", 2, 8, 2, 4, 64, l, l + 3, N=N, n=3, steps=4)
    run_loop_and_compare(w, seed=l + N % 97)


def test_zero_query_and_unit_values():
    w = wl("zero", 1, 8, 2, 4, 64, 300, None, N=5, n=2, steps=2)
    qs, K, V = device_inputs(w, seed=10, steps=2)
    q = torch.zeros_like(qs[0])
    ones = torch.ones_like(V)
    dec = AtopNDecoder.for_workload(w)
    out, idx, cnt = gpu_step_with_mask(dec, 0, q, K, ones)
    torch.cuda.synchronize()
    assert np.all(cnt.cpu().numpy() == w.l_kv)          # all logits 0 = tau: ties all kept
    np.testing.assert_allclose(out.cpu().numpy(), 1.0, rtol=1e-6)
    out_f = dec.step(1, qs[1], K, ones).clone()          # reuse step, fused path
    torch.cuda.synchronize()
    np.testing.assert_allclose(out_f.cpu().numpy(), 1.0, rtol=1e-6)


def test_same_query_reuse_keeps_the_refresh_mask():
    """A reuse step with the refresh step's own query keeps exactly the
    refresh step's set: the fused on-chip compare (reuse) against the
    refresh step's compaction of its candidates.  The outputs sum the same
    entries in a different order, so they agree to rounding."""
    w = wl("same", 2, 32, 4, 8, 64, 5000, None, N=100, n=4, steps=1)
    qs, K, V = device_inputs(w, seed=11, steps=1)
    dec = AtopNDecoder.for_workload(w)
    o_ref, i_ref, c_ref = gpu_step_with_mask(dec, 0, qs[0], K, V)
    o_reu, i_reu, c_reu = gpu_step_with_mask(dec, 1, qs[0], K, V)
    o_again, i_again, c_again = gpu_step_with_mask(dec, 2, qs[0], K, V)
    torch.cuda.synchronize()
    assert torch.equal(c_ref, c_reu)
    assert torch.equal(i_ref, i_reu)
    torch.testing.assert_close(o_reu, o_ref, rtol=1e-5, atol=1e-6)
    # the fused path is deterministic
    assert torch.equal(i_reu, i_again) and torch.equal(c_reu, c_again)
    assert torch.equal(o_reu, o_again)


def test_resume_from_saved_state_is_bit_identical():
    w = wl("resume", 1, 12, 1, 2, 128, 3000, None, N=60, n=4, steps=10)
    qs, K, V = device_inputs(w, seed=12)
    a = AtopNDecoder.for_workload(w)
    outs = [a.step(t, qs[t], K, V).clone() for t in range(w.steps)]
    b = AtopNDecoder.for_workload(w)
    b.step(4, qs[4], K, V)        # refresh at t=4 recreates the state of t=4..7
    resumed = [b.step(t, qs[t], K, V).clone() for t in range(5, w.steps)]
    torch.cuda.synchronize()
    for x, y in zip(outs[5:], resumed):
        assert torch.equal(x, y)


# ---------------------------------------------------------------- full-size workloads

FULL = ["qwen_b1_32k", "llama_b16_128k", "qwen_b16_128k_saga_N1024", "qwen_b16_128k_gqa_N2048",
        "llama_sweep_b1_l128k", "llama_sweep_b16_l8k", "sigma_b16_128k"]


@pytest.mark.parametrize("name", FULL)
def test_full_size_workloads_on_sampled_rows(name):
    w = CONFIGS[name].scaled(steps=3, n=2)  # refresh, reuse, refresh
    rows = [0] if w.batch == 1 else [0, w.batch - 1]
    run_loop_and_compare(w, seed=0, rows=rows)


@pytest.mark.parametrize("name", ["llama_b16_128k", "qwen_b1_32k", "qwen_b16_128k_gqa_N1024"])
def test_full_size_dense_on_sampled_rows(name):
    w = CONFIGS[name]
    qs, K, V = device_inputs(w, seed=0, steps=1)
    dec = AtopNDecoder.for_workload(w)
    out = dec.dense(qs[0], K, V)
    torch.cuda.synchronize()
    rows = [0] if w.batch == 1 else [3]
    ref = oracle.decode_dense(bits(qs[0][rows]), bits(K[rows]), bits(V[rows]))
    assert_outputs_close(out[rows].cpu().numpy(), ref, name)
