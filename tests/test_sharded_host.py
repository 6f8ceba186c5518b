"""The multi-process plumbing of the sequence-sharded decode on CPU (gloo,
world size 2 and 3): SequenceShardedDecoder with TorchComm, each rank holding
one contiguous shard of the cache, and the device calls replaced by a host
stand-in (HostShardOps) that computes each call's documented result from the
oracle's logits.  Every rank must end each step with the thresholds and the
output of the oracle run over the whole cache.  The CUDA kernels behind the
same calls are checked on the GPU by test_gpu_sharded.py."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _key(s: np.ndarray) -> np.ndarray:
    """Order-preserving 32-bit key of float32 values (-0 like +0)."""
    u = np.where(s == 0, np.float32(0), s).astype(np.float32).view(np.uint32)
    return np.where(u >> 31, ~u, u | np.uint32(0x80000000)).astype(np.uint32)


def _unkey(k: np.uint32) -> np.float32:
    k = np.uint32(k)
    u = k & np.uint32(0x7FFFFFFF) if k >> 31 else ~k
    return np.array([u], np.uint32).view(np.float32)[0]


DIGITS = [(21, 11), (10, 11), (0, 10)]  # (shift, width) of the three passes


class HostShardOps:
    """ShardOps' calls computed on the host from the oracle's logits."""

    def __init__(self, w, N):
        import oracle
        from sparse_decode_attention_saga_b200.workload import bf16_bits
        self.oracle, self.bits = oracle, bf16_bits
        self.w, self.N = w, N
        self.rows = w.batch * w.h_q
        self.state = np.zeros((self.rows, 2), np.uint32)
        self.thresh = np.full(self.rows, np.nan, np.float32)

    def compute_logits(self, q, k):
        self.s = self.oracle.logits(self.bits(q), self.bits(k)).reshape(self.rows, -1)

    def histogram(self, p):
        shift, width = DIGITS[p]
        keys = _key(self.s)
        hist = np.zeros((self.rows, 2048), np.int64)
        for r in range(self.rows):
            if p > 0 and self.state[r, 1] == 0:
                continue
            kr = keys[r]
            if p > 0:
                kr = kr[(kr >> np.uint32(shift + width)) == self.state[r, 0]]
            np.add.at(hist[r], (kr >> np.uint32(shift)) & np.uint32((1 << width) - 1), 1)
        return torch.from_numpy(hist.astype(np.int32))

    def select_digit(self, p, hist_sum):
        shift, width = DIGITS[p]
        h = hist_sum.numpy().astype(np.int64)
        for r in range(self.rows):
            rank = self.N if p == 0 else int(self.state[r, 1])
            if p > 0 and rank == 0:
                continue
            if p == 0 and self.N >= h[r].sum():  # N >= l: every position is kept
                self.thresh[r], self.state[r] = -np.inf, (0, 0)
                continue
            desc = h[r][: 1 << width][::-1]  # this pass's bins, top first
            cum = np.cumsum(desc)
            i = int(np.argmax(cum >= rank))
            digit = (1 << width) - 1 - i
            before = int(cum[i] - desc[i])
            key = (int(self.state[r, 0]) << width) | digit if p > 0 else digit
            if p < 2:
                self.state[r] = (key, rank - before)
            else:
                self.thresh[r], self.state[r, 1] = _unkey(np.uint32(key)), 0

    def partial(self, q, k, v, use_logits):
        if not use_logits:
            self.compute_logits(q, k)
        w, Vb = self.w, self.bits(v).view(np.uint16)
        Vf = (Vb.astype(np.uint32) << 16).view(np.float32)  # [b, l, hv, dv]
        part = np.zeros((self.rows, w.dv + 4), np.float32)
        for r in range(self.rows):
            bb, i = divmod(r, w.h_q)
            vh = i * w.h_v // w.h_q
            s = self.s[r].astype(np.float64)
            keep = self.s[r] >= self.thresh[r]
            mx = self.s[r].max()
            if keep.any():
                e = np.exp(s[keep] - mx)
                part[r, 0], part[r, 1] = mx, e.sum()
                part[r, 2] = np.array([keep.sum()], np.int32).view(np.float32)[0]
                part[r, 4:] = e @ Vf[bb, keep, vh].astype(np.float64)
            else:
                at = self.s[r] == mx
                part[r, 0], part[r, 1] = -np.inf, at.sum()
                part[r, 4:] = Vf[bb, at, vh].sum(0)
            part[r, 3] = mx
        return torch.from_numpy(part)

    def merge(self, parts, out, sel_cnt=None):
        P = parts.numpy().astype(np.float64)
        cnt = parts.numpy()[..., 2].copy().view(np.int32)
        for r in range(self.rows):
            c = cnt[:, r]
            if c.sum() > 0:
                m = P[c > 0, r, 0]
                wgt = np.exp(m - m.max())
                o = (wgt[:, None] * P[c > 0, r, 4:]).sum(0) / (wgt * P[c > 0, r, 1]).sum()
            else:
                mx = P[:, r, 3]
                sel = mx == mx.max()
                o = P[sel, r, 4:].sum(0) / P[sel, r, 1].sum()
            out[r] = torch.from_numpy(o.astype(np.float32))


def _worker(rank, world, port, lengths, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        import oracle
        from sparse_decode_attention_saga_b200.sharded import SequenceShardedDecoder, TorchComm
        from sparse_decode_attention_saga_b200.workload import (Workload, bf16_bits, make_cache,
                                                                make_queries)
        l = int(sum(lengths))
        w = Workload("host_shards", 2, 8, 2, 4, 64, l, 37, 3, steps=4)
        K, V = make_cache(w, 5)
        qs = make_queries(w, 5)
        a = int(sum(lengths[:rank]))
        k_r, v_r = K[:, a:a + lengths[rank]].contiguous(), V[:, a:a + lengths[rank]].contiguous()
        ops = HostShardOps(w, w.N)
        dec = SequenceShardedDecoder(ops, TorchComm(), w.n)
        tau_ref = np.full((w.batch, w.h_q), np.nan, np.float32)
        worst = 0.0
        for t in range(w.steps):
            out = torch.empty((w.batch * w.h_q, w.dv), dtype=torch.float32)
            dec.step(t, qs[t], k_r, v_r, out)
            o_ref, s_ref, m_ref, c_ref = oracle.atopn_step(bf16_bits(qs[t]), bf16_bits(K),
                                                           bf16_bits(V), tau_ref, w.N, t, w.n)
            assert np.array_equal(ops.thresh.view(np.int32), tau_ref.reshape(-1).view(np.int32)), t
            worst = max(worst, float(np.abs(out.numpy().reshape(o_ref.shape) - o_ref).max()))
        results.put((rank, worst))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("lengths", [[300, 211], [100, 1, 250]], ids=["two", "three_with_one"])
def test_sharded_decoder_over_gloo_matches_oracle(lengths):
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    world = len(lengths)
    procs = [ctx.Process(target=_worker, args=(r, world, port, lengths, results))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
        assert p.exitcode == 0
    got = sorted(results.get(timeout=5) for _ in range(world))
    assert [g[0] for g in got] == list(range(world))
    assert all(g[1] <= 1e-5 for g in got), got
