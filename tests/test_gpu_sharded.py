"""Sequence-sharded decode (sharded.py) on one GPU: the shards run one after
the other with the cross-rank sums done in the test (the multi-process
exchange itself is covered on the host by test_sharded_host.py).  Each
shard's caches are separate tensors, as on separate GPUs.  Thresholds must
equal a single-GPU refresh over the whole cache bit for bit, kept counts
must equal the single-GPU list path's, and outputs match the oracle given
that path's mask."""
import numpy as np
import pytest
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.sharded import RADIX_PASSES, ShardOps
from sparse_decode_attention_saga_b200.workload import Workload

from .gpu_helpers import (assert_mask_within_band, assert_outputs_close, bits, device_inputs,
                          gpu_step_with_mask, mask_from_lists)

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)

SPLITS = [
    # name, b, hq, hk, hv, d, shard lengths (ragged, a 1-position shard, uneven)
    ("llama_like_2", 2, 32, 4, 8, 64, [700, 555]),
    ("qwen_like_3", 1, 12, 1, 2, 128, [1000, 1, 2048]),
    ("even_4", 2, 8, 2, 4, 64, [300, 300, 300, 300]),
]


class Shards:
    """R ranks' ShardOps over slices of one cache, exchanged in-process."""

    def __init__(self, w, lengths, K, V):
        self.offsets = np.concatenate([[0], np.cumsum(lengths)])
        self.K = [K[:, a:b].contiguous() for a, b in zip(self.offsets[:-1], self.offsets[1:])]
        self.V = [V[:, a:b].contiguous() for a, b in zip(self.offsets[:-1], self.offsets[1:])]
        self.ops = [ShardOps(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, l, w.N) for l in lengths]

    def refresh(self, q):
        for o, k in zip(self.ops, self.K):
            o.compute_logits(q, k)
        for p in range(RADIX_PASSES):
            total = sum(o.histogram(p).clone() for o in self.ops)  # the all-reduce
            for o in self.ops:
                o.select_digit(p, total)

    def decode(self, q, refresh, out, cnt):
        parts = torch.stack([o.partial(q, k, v, refresh).clone()  # the all-gather
                             for o, k, v in zip(self.ops, self.K, self.V)])
        self.ops[0].merge(parts, out, cnt)


@pytest.mark.parametrize("split", SPLITS, ids=lambda s: s[0])
def test_sharded_loop_matches_single_gpu_and_oracle(split):
    name, b, hq, hk, hv, d, lengths = split
    l = int(sum(lengths))
    w = Workload(name, b, hq, hk, hv, d, l, max(1, l // 40), 3, steps=5)
    qs, K, V = device_inputs(w, seed=51)
    Kh, Vh = bits(K), bits(V)
    sh = Shards(w, lengths, K, V)
    full = AtopNDecoder.for_workload(w)
    tau_ref = np.full((b, hq), np.nan, np.float32)
    for t in range(w.steps):
        refresh = t % w.n == 0
        if refresh:
            sh.refresh(qs[t])
        out = torch.empty((b, hq, w.dv), dtype=torch.float32, device="cuda")
        cnt = torch.zeros((b, hq), dtype=torch.int32, device="cuda")
        sh.decode(qs[t], refresh, out.view(b * hq, w.dv), cnt)
        out_l, idx, cnt_l = gpu_step_with_mask(full, t, qs[t], K, V)
        torch.cuda.synchronize()
        for o in sh.ops:
            assert np.array_equal(o.thresh.cpu().numpy().view(np.int32),
                                  full.thresh.cpu().numpy().view(np.int32)), f"t={t}"
            assert _lib.workspace_error(o.ws) == _lib.SAGA_OK
        assert np.array_equal(cnt.cpu().numpy(), cnt_l.cpu().numpy()), f"t={t}"
        o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bits(qs[t]), Kh, Vh, tau_ref, w.N, t, w.n)
        mask = mask_from_lists(idx, cnt_l, l)
        assert_mask_within_band(mask, m_ref, s_ref, tau_ref, f"t={t}")
        ref = oracle.attend_masked(s_ref, mask, Vh)
        assert_outputs_close(out.cpu().numpy(), ref, f"t={t} sharded")


@pytest.mark.parametrize("case", ["stale_above_all", "N_at_least_l"])
def test_sharded_edge_thresholds(case):
    name, b, hq, hk, hv, d, lengths = SPLITS[2]
    l = int(sum(lengths))
    N = l + 3 if case == "N_at_least_l" else 20
    w = Workload(name, b, hq, hk, hv, d, l, N, 4, steps=1)
    qs, K, V = device_inputs(w, seed=53, steps=1)
    sh = Shards(w, lengths, K, V)
    full = AtopNDecoder.for_workload(w)
    full.refresh(qs[0], K)
    sh.refresh(qs[0])
    torch.cuda.synchronize()
    s = full.logits.cpu().numpy()
    if case == "stale_above_all":  # no logit of any shard reaches it: the row maxima are kept
        tau = (s.max(-1) + 1.0).astype(np.float32)
        for o in sh.ops:
            o.thresh.copy_(torch.from_numpy(tau))
        refresh = False
    else:
        tau = np.full((b, hq), -np.inf, np.float32)
        for o in sh.ops:
            assert np.array_equal(o.thresh.cpu().numpy(), tau)
        refresh = True
    out = torch.empty((b * hq, w.dv), dtype=torch.float32, device="cuda")
    cnt = torch.zeros((b, hq), dtype=torch.int32, device="cuda")
    sh.decode(qs[0], refresh, out, cnt)
    torch.cuda.synchronize()
    mask, cnt_ref = oracle.select(s, tau)
    assert np.array_equal(cnt.cpu().numpy(), cnt_ref)
    ref = oracle.attend_masked(s, mask, bits(V))
    assert_outputs_close(out.view(b, hq, w.dv).cpu().numpy(), ref, case)
