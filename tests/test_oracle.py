"""Pins for the CPU oracle against facts fixed outside it.

Every oracle function is checked here against something other than itself:
a float64 library matmul (logits), a full sort (threshold), library softmax
attention (N >= l, h_k == h_v, n == 1 with a library top-k), closed forms
(sum p == 1, N == 1 argmax, q == 0 mean, a worked example) and invariants
(permutation equivariance, resume).  ``test_oracle_mutants.py`` plants
mistakes in copies of the oracle and checks that these pins catch them.

Method: "More Value per Key: Asymmetric Sparse Attention for Faster LLM
Decoding" (ai.info summary, Key Contributions #2-#3, Main Findings).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200.workload import (
    CONFIGS, Workload, bf16_bits, kv_cache_bytes, make_cache, make_queries)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def small(b=2, hq=8, hk=2, hv=4, d=64, l=200, N=16, n=4, cap=None, name="pin"):
    return Workload(name, b, hq, hk, hv, d, l, N, n, steps=6, l_cap=cap)


def inputs(w: Workload, seed=0):
    K, V = make_cache(w, seed)
    qs = make_queries(w, seed)
    return qs, K, V


def ref_attention(q, K, V, l, mask=None):
    """float64 softmax attention with key/value heads repeated to the query
    heads (torch library ops); ``mask`` [b,hq,l] bool keeps entries."""
    b, hq, d = q.shape
    hk, hv = K.shape[2], V.shape[2]
    Kq = K[:, :l].double().repeat_interleave(hq // hk, dim=2)
    Vq = V[:, :l].double().repeat_interleave(hq // hv, dim=2)
    qq = q.double()[:, :, None, :]
    attn_mask = None if mask is None else torch.as_tensor(mask)[:, :, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(
        qq, Kq.transpose(1, 2), Vq.transpose(1, 2), attn_mask=attn_mask)
    return o[:, :, 0, :].numpy()


def ref_logits64(q, K, l):
    b, hq, d = q.shape
    Kq = K[:, :l].double().repeat_interleave(hq // K.shape[2], dim=2)
    return (torch.einsum("bhd,blhd->bhl", q.double(), Kq) / math.sqrt(d)).numpy()


# ---------------------------------------------------------------- a1 logits

@pytest.mark.parametrize("d,hq,hk,cap", [(64, 8, 2, None), (128, 12, 1, 230), (64, 4, 4, None)])
def test_logits_match_float64_matmul(d, hq, hk, cap):
    w = small(hq=hq, hk=hk, hv=hk, d=d, l=200, cap=cap)
    qs, K, V = inputs(w, seed=3)
    s = oracle.logits(bf16_bits(qs[0]), bf16_bits(K), l=w.l_kv)
    ref = ref_logits64(qs[0], K, w.l_kv).astype(np.float32)
    np.testing.assert_array_max_ulp(s, ref, maxulp=1)


# ---------------------------------------------------------------- a2 threshold

@pytest.mark.parametrize("l,N", [(1, 1), (2, 1), (31, 5), (32, 31), (33, 33), (257, 300), (257, 64)])
def test_threshold_matches_full_sort(l, N):
    rng = np.random.default_rng(l * 1000 + N)
    # small integer range -> many ties; include +-0
    s = rng.integers(-6, 7, size=(5, l)).astype(np.float32) * 0.5
    s[1] = -0.0
    s[2, ::2] = 0.0
    s[2, 1::2] = -0.0
    tau = oracle.nth_largest(s, N)
    brute = oracle.nth_largest_sort(s, N)
    for r in range(s.shape[0]):
        if N >= l:
            assert tau[r] == -np.inf
            continue
        expect = np.sort(s[r])[::-1][N - 1]          # numpy sort, descending
        assert tau[r] == expect and brute[r] == expect
        assert not np.signbit(tau[r]) or tau[r] != 0  # -0 stored as +0


def test_threshold_counts_duplicates():
    s = np.array([[3, 3, 3, 1, 0]], np.float32)
    assert oracle.nth_largest(s, 1)[0] == 3
    assert oracle.nth_largest(s, 3)[0] == 3
    assert oracle.nth_largest(s, 4)[0] == 1


# ---------------------------------------------------------------- a3 select

def test_select_definition_and_empty_set_reading():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((6, 50)).astype(np.float32)
    tau = np.array([0.0, 1.0, -np.inf, 10.0, np.float32(s[4].max()), -1.0], np.float32)
    mask, cnt = oracle.select(s, tau)
    for r in range(6):
        t_eff = min(tau[r], s[r].max())
        np.testing.assert_array_equal(mask[r], s[r] >= t_eff)
        assert cnt[r] == mask[r].sum()
    # tau above every logit keeps exactly the maximal entries
    np.testing.assert_array_equal(mask[3], s[3] == s[3].max())


# ---------------------------------------------------------------- a4/a5/a7

@pytest.mark.parametrize("hq,hk,hv,d", [(8, 2, 4, 64), (12, 1, 2, 128), (4, 1, 2, 64)])
def test_N_at_least_l_is_full_attention(hq, hk, hv, d):
    w = small(hq=hq, hk=hk, hv=hv, d=d, l=150, N=150)
    qs, K, V = inputs(w, seed=5)
    tau = np.zeros((w.batch, hq), np.float32)
    for N in (w.l_kv, w.l_kv + 7):
        out, s, mask, cnt = oracle.atopn_step(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V),
                                              tau, N, 0, 1)
        assert np.all(tau == -np.inf) and mask.all() and np.all(cnt == w.l_kv)
        np.testing.assert_allclose(out, ref_attention(qs[0], K, V, w.l_kv), rtol=1e-5, atol=1e-6)
    dense = oracle.decode_dense(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V))
    np.testing.assert_allclose(dense, ref_attention(qs[0], K, V, w.l_kv), rtol=1e-5, atol=1e-6)


def test_narrow_keys_sigma_layout_is_attention_with_separate_head_dims():
    """Keys (and queries) of 32 dims, values of 64 (the pages' Sigma-style
    (h_k, d_k) = (2, 32) next to h_v = 8, d_v = 64): the logits scale by
    1/sqrt(32) and the output has the value dim.  Full attention (N >= l)
    against library float64 attention, and a reuse step against library
    attention restricted to the oracle's mask."""
    w = Workload("sigma", 2, 16, 2, 8, 32, 180, 180, 4, steps=2, v_head_dim=64)
    qs, K, V = inputs(w, seed=13)
    assert qs.shape[-1] == 32 and K.shape[-1] == 32 and V.shape[-1] == 64
    tau = np.zeros((w.batch, w.h_q), np.float32)
    out, s, mask, cnt = oracle.atopn_step(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V), tau,
                                          w.l_kv, 0, 4)
    assert out.shape == (w.batch, w.h_q, 64)
    np.testing.assert_allclose(out, ref_attention(qs[0], K, V, w.l_kv), rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(s, ref_logits64(qs[0], K, w.l_kv), rtol=1e-6, atol=1e-6)
    dense = oracle.decode_dense(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V))
    np.testing.assert_allclose(dense, ref_attention(qs[0], K, V, w.l_kv), rtol=1e-5, atol=1e-6)
    tau = np.zeros((w.batch, w.h_q), np.float32)
    oracle.atopn_step(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V), tau, 12, 0, 4)  # refresh
    out1, s1, mask1, _ = oracle.atopn_step(bf16_bits(qs[1]), bf16_bits(K), bf16_bits(V), tau,
                                           12, 1, 4)                                 # reuse
    np.testing.assert_allclose(out1, ref_attention(qs[1], K, V, w.l_kv, mask=mask1),
                               rtol=1e-5, atol=1e-6)


def test_hk_equal_hv_is_grouped_query_attention():
    w = small(hq=8, hk=2, hv=2, d=64, l=120)
    qs, K, V = inputs(w, seed=6)
    dense = oracle.decode_dense(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V))
    o = torch.nn.functional.scaled_dot_product_attention(
        qs[0].double()[:, :, None, :], K.double().transpose(1, 2), V.double().transpose(1, 2),
        enable_gqa=True)[:, :, 0, :].numpy()
    np.testing.assert_allclose(dense, o, rtol=1e-5, atol=1e-6)


def test_refresh_every_step_is_exact_topN():
    w = small(hq=8, hk=2, hv=4, d=64, l=300, N=20, n=1)
    qs, K, V = inputs(w, seed=7)
    for t, out, s, mask, cnt, tau in oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(V),
                                                        w.N, 1):
        s64 = ref_logits64(qs[t], K, w.l_kv)
        top = torch.topk(torch.from_numpy(s64), w.N, dim=-1).indices.numpy()
        ref_mask = np.zeros_like(mask)
        np.put_along_axis(ref_mask, top, True, axis=-1)
        np.testing.assert_array_equal(mask, ref_mask)
        assert np.all(cnt == w.N)  # h_q x N value vectors per token (l_q = 1)
        np.testing.assert_allclose(out, ref_attention(qs[t], K, V, w.l_kv, ref_mask),
                                   rtol=1e-5, atol=1e-6)


def test_kept_weights_sum_to_one():
    w = small(l=90, N=7, n=3)
    qs, K, V = inputs(w, seed=8)
    ones = torch.ones_like(V)
    for t, out, *_ in oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(ones), w.N, w.n):
        np.testing.assert_array_equal(out, np.ones_like(out))


def test_N1_unique_max_returns_that_value_row():
    w = small(hq=4, hk=1, hv=2, l=77, N=1, n=1)
    qs, K, V = inputs(w, seed=9)
    tau = np.zeros((w.batch, w.h_q), np.float32)
    out, s, mask, cnt = oracle.atopn_step(bf16_bits(qs[0]), bf16_bits(K), bf16_bits(V), tau, 1, 0, 1)
    Vf = V.float().numpy()
    for bb in range(w.batch):
        for i in range(w.h_q):
            j = int(np.argmax(s[bb, i]))
            assert (s[bb, i] == s[bb, i, j]).sum() == 1
            np.testing.assert_array_equal(out[bb, i], Vf[bb, j, i * w.h_v // w.h_q])


def test_zero_query_keeps_everything_and_averages():
    w = small(hq=4, hk=2, hv=2, l=64, N=5)
    _, K, V = inputs(w, seed=10)
    q = torch.zeros(w.batch, w.h_q, w.head_dim, dtype=torch.bfloat16)
    tau = np.zeros((w.batch, w.h_q), np.float32)
    out, s, mask, cnt = oracle.atopn_step(bf16_bits(q), bf16_bits(K), bf16_bits(V), tau, 5, 0, 4)
    assert np.all(s == 0) and np.all(tau == 0) and mask.all()
    mean = V.double().mean(dim=1).repeat_interleave(w.h_q // w.h_v, dim=1).numpy()
    np.testing.assert_allclose(out, mean, rtol=1e-6, atol=1e-7)


def test_permuting_positions_permutes_the_mask():
    w = small(l=180, N=12, n=4)
    qs, K, V = inputs(w, seed=11)
    perm = torch.randperm(w.l_kv, generator=torch.Generator().manual_seed(0))
    Kp, Vp = K[:, perm], V[:, perm]
    a = list(oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(V), w.N, w.n))
    b = list(oracle.atopn_run(bf16_bits(qs), bf16_bits(Kp), bf16_bits(Vp), w.N, w.n))
    for (t, oa, sa, ma, ca, ta), (_, ob, sb, mb, cb, tb) in zip(a, b):
        np.testing.assert_array_equal(ma[..., perm.numpy()], mb)
        np.testing.assert_array_equal(ta, tb)
        np.testing.assert_allclose(oa, ob, rtol=1e-6, atol=1e-7)


def test_resume_from_saved_threshold_is_bit_identical():
    w = small(l=160, N=10, n=4).scaled(steps=12)
    qs, K, V = inputs(w, seed=12)
    full = list(oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(V), w.N, w.n))
    saved_tau = full[6][5].copy()  # state after step t=6 (tau last refreshed at t=4)
    resumed = list(oracle.atopn_run(bf16_bits(qs[7:]), bf16_bits(K), bf16_bits(V), w.N, w.n,
                                    t0=7, tau_state=saved_tau))
    for x, y in zip(full[7:], resumed):
        assert x[0] == y[0]
        np.testing.assert_array_equal(x[1], y[1])
        np.testing.assert_array_equal(x[3], y[3])


def test_reuse_steps_keep_the_refresh_threshold():
    w = small(l=128, N=9, n=4).scaled(steps=8)
    qs, K, V = inputs(w, seed=13)
    run = list(oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(V), w.N, w.n))
    for t, out, s, mask, cnt, tau in run:
        t_ref = run[(t // w.n) * w.n]
        np.testing.assert_array_equal(tau, t_ref[5])
        if t % w.n == 0:
            np.testing.assert_array_equal(tau, oracle.nth_largest_sort(s, w.N))


def test_same_query_reuse_equals_refresh():
    w = small(l=140, N=11, n=4)
    qs, K, V = inputs(w, seed=14)
    q2 = torch.stack([qs[0], qs[0]])
    (_, o0, s0, m0, c0, _), (_, o1, s1, m1, c1, _) = oracle.atopn_run(
        bf16_bits(q2), bf16_bits(K), bf16_bits(V), w.N, w.n)
    np.testing.assert_array_equal(m0, m1)
    np.testing.assert_array_equal(o0, o1)


# ---------------------------------------------------------------- worked example

def test_worked_example_closed_form():
    """b=1, h_q=2, h_k=1, h_v=2, d=64, l=4, N=2, n=4.  Only coordinate 0 of q
    and K is non-zero: K[j,0,0] = (8, 4, 0, -4), so s = q0 * K / 8.
    V[j,0,1] = j+1 (value head 0) and V[j,1,2] = 10(j+1) (value head 1).
      t=0 (refresh): q0 = (2, 4) -> s = (2,1,0,-1), (4,2,0,-2); tau = (1, 2);
        both heads keep j in {0,1}:
        o[0,1] = (e+2)/(e+1),  o[1,2] = 10 (e^2+2)/(e^2+1).
      t=1 (reuse): q0 = (-2, 0) -> head 0: s = (-2,-1,0,1) >= 1 keeps j=3 -> 4;
        head 1: s = 0 everywhere < tau = 2 -> keeps the maxima (all) -> 25.
      t=2 (reuse): q0 = (1, 8) -> head 0 keeps j=0 -> 1;
        head 1: s = (8,4,0,-4) keeps {0,1} -> 10 (1 + 2e^-4)/(1 + e^-4).
    """
    d = 64
    K = torch.zeros(1, 4, 1, d)
    K[0, :, 0, 0] = torch.tensor([8.0, 4.0, 0.0, -4.0])
    V = torch.zeros(1, 4, 2, d)
    V[0, :, 0, 1] = torch.arange(1, 5, dtype=torch.float32)
    V[0, :, 1, 2] = 10 * torch.arange(1, 5, dtype=torch.float32)
    qs = torch.zeros(3, 1, 2, d)
    qs[:, 0, :, 0] = torch.tensor([[2.0, 4.0], [-2.0, 0.0], [1.0, 8.0]])
    to = lambda x: bf16_bits(x.to(torch.bfloat16))
    run = list(oracle.atopn_run(to(qs), to(K), to(V), N=2, n=4))
    e = math.e
    expect = [
        ((e + 2) / (e + 1), 10 * (e * e + 2) / (e * e + 1)),
        (4.0, 25.0),
        (1.0, 10 * (1 + 2 * math.exp(-4)) / (1 + math.exp(-4))),
    ]
    kept = [([1, 1, 0, 0], [1, 1, 0, 0]), ([0, 0, 0, 1], [1, 1, 1, 1]), ([1, 0, 0, 0], [1, 1, 0, 0])]
    for (t, out, s, mask, cnt, tau), (e0, e1), (k0, k1) in zip(run, expect, kept):
        assert tau.tolist() == [[1.0, 2.0]]
        assert mask[0, 0].astype(int).tolist() == k0 and mask[0, 1].astype(int).tolist() == k1
        np.testing.assert_allclose([out[0, 0, 1], out[0, 1, 2]], [e0, e1], rtol=1e-7)
        other = out.copy()
        other[0, 0, 1] = other[0, 1, 2] = 0
        assert np.all(other == 0)


# ---------------------------------------------------------------- pages' facts

def test_pages_facts():
    facts = json.load(open(os.path.join(GOLDEN, "pages_facts.json")))
    kv = facts["kv_cache_saga_1_8_vs_gqa_8_8"]
    ratio = kv_cache_bytes(1, 4096, 1, 8, 64) / kv_cache_bytes(1, 4096, 8, 8, 64)
    assert ratio == 9 / 16 and kv["lower_exclusive"] < ratio < kv["upper_exclusive"]
    hr = facts["head_reductions"]
    assert CONFIGS["llama_b16_128k"].h_k == hr["llama_h_k"][1]
    assert CONFIGS["qwen_b1_32k"].h_k == hr["qwen_h_k"][1]
    assert CONFIGS["qwen_b16_128k_gqa_N1024"].h_k == hr["qwen_h_k"][0]
    lp = facts["latency_protocol"]
    sweep = [w for k, w in CONFIGS.items() if k.startswith("llama_sweep")]
    assert min(w.l_kv for w in sweep) == lp["context_min"]
    assert max(w.l_kv for w in sweep) == lp["context_max"]
    assert {w.N for k, w in CONFIGS.items() if k.startswith("qwen_b16")} == set(lp["N_values"])
    assert all(w.steps == lp["generated_tokens"] for w in CONFIGS.values())


def test_tiny_config_refresh_counts_are_N():
    """On refresh steps every (batch, query head) keeps exactly N entries when
    the N-th and (N+1)-th logits differ: h_q x N value vectors per token."""
    w = CONFIGS["tiny"].scaled(steps=9)
    qs, K, V = inputs(w, seed=0)
    for t, out, s, mask, cnt, tau in oracle.atopn_run(bf16_bits(qs), bf16_bits(K), bf16_bits(V),
                                                        w.N, w.n):
        if t % w.n == 0:
            srt = -np.sort(-s, axis=-1)
            distinct = srt[..., w.N - 1] != srt[..., w.N]
            assert np.all(cnt[distinct] == w.N)
            assert cnt.sum() >= w.h_q * w.N
