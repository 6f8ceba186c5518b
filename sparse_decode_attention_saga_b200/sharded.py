"""Decode over a cached sequence split into contiguous shards, one per rank.

The pages run one GPU; this spreads one layer's cache over ranks when it does
not fit or when the per-token latency must drop further.  Rank r holds the
positions [offset_r, offset_r + l_r) of the key and value caches (its own
tensors, any split) and the same queries.  Per step, with AtopNDecoder's
schedule (refresh when t mod n == 0, "More Value per Key", ai.info summary,
Key Contributions #2):

* refresh: the logits of the shard; for each of the three radix passes the
  shard's digit histogram, summed over the ranks (all-reduce), and the digit
  chosen from the sum, identical on every rank -- so every rank ends with the
  exact N-th largest logit of the whole row, bit for bit what one GPU finds;
* decode: the shard's partial record per row (softmax numerator and
  denominator over its kept entries, or its maximal entries), the records of
  all ranks (all-gather), merged into the output by log-sum-exp, identical on
  every rank.

Per step the exchange is 3 x b*h_q*2048 int32 counts on refresh steps and
R x b*h_q*(d_v + 4) floats; every kernel is libsaga.so's (ShardOps).  The
exchange goes through a communicator object (TorchComm: torch.distributed,
so NCCL between GPUs, gloo on the host).
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _lib

RADIX_PASSES = 3
RADIX_BINS = 2048


class ShardOps:
    """The device calls of one rank over its shard (libsaga.so)."""

    def __init__(self, batch, h_q, h_k, h_v, head_dim, l_local, N, l_cap=None, v_head_dim=None,
                 device="cuda"):
        self.l_cap = int(l_local if l_cap is None else l_cap)
        self.dv = int(head_dim if v_head_dim is None else v_head_dim)
        self.N = int(N)
        self.dims = _lib.dims(batch, h_q, h_k, h_v, head_dim, l_local, self.l_cap, self.dv)
        rows = batch * h_q
        nbytes = _lib.workspace_bytes(_lib.dims(batch, h_q, h_k, h_v, head_dim, self.l_cap,
                                                self.l_cap, self.dv), self.N)
        if nbytes == 0:
            raise _lib.SagaError("saga_workspace_bytes", _lib.SAGA_ERR_UNSUPPORTED)
        dev = torch.device(device)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        self._logits = torch.empty(rows * self.l_cap, dtype=torch.float32, device=dev)
        self.state = torch.zeros((rows, 2), dtype=torch.int32, device=dev)
        self.hist = torch.zeros((rows, RADIX_BINS), dtype=torch.int32, device=dev)
        self.thresh = torch.full((batch, h_q), float("nan"), dtype=torch.float32, device=dev)
        self.part = torch.empty((rows, self.dv + 4), dtype=torch.float32, device=dev)

    @property
    def logits(self) -> torch.Tensor:
        d = self.dims
        return self._logits[: d.batch * d.h_q * d.l_kv].view(d.batch, d.h_q, d.l_kv)

    def compute_logits(self, q, k) -> None:
        _lib.qk_logits(self.dims, q, k, self.logits, self.ws)

    def histogram(self, pass_: int) -> torch.Tensor:
        _lib.topn_histogram(self.dims, pass_, self.logits, self.state, self.hist)
        return self.hist

    def select_digit(self, pass_: int, hist_sum: torch.Tensor) -> None:
        _lib.topn_select_digit(self.dims, self.N, pass_, hist_sum, self.state, self.thresh)

    def partial(self, q, k, v, use_logits: bool) -> torch.Tensor:
        _lib.atopn_decode_partial(self.dims, q, k, v, self.thresh,
                                  self.logits if use_logits else None, self.part, self.ws)
        return self.part

    def merge(self, parts: torch.Tensor, out: torch.Tensor, sel_cnt=None) -> None:
        _lib.merge_partials(self.dims, parts, parts.shape[0], out, sel_cnt)


class TorchComm:
    """The cross-rank exchange over a torch.distributed process group."""

    def __init__(self, group=None):
        self.group = group
        self.world = dist.get_world_size(group)

    def all_reduce_sum(self, t: torch.Tensor) -> None:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=self.group)

    def all_gather(self, t: torch.Tensor) -> torch.Tensor:
        parts = [torch.empty_like(t) for _ in range(self.world)]
        dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)


class SequenceShardedDecoder:
    """One rank's side of the sharded decode loop (every rank calls step with
    the same t and q, and its own shard of the caches)."""

    def __init__(self, ops, comm, n: int):
        self.ops, self.comm, self.n = ops, comm, int(n)

    def is_refresh(self, t: int) -> bool:
        return t % self.n == 0

    def refresh(self, q, k) -> None:
        """Exact thresholds of the whole rows from the shards' histograms."""
        self.ops.compute_logits(q, k)
        for p in range(RADIX_PASSES):
            h = self.ops.histogram(p)
            self.comm.all_reduce_sum(h)
            self.ops.select_digit(p, h)

    def step(self, t: int, q, k, v, out, sel_cnt=None):
        refresh = self.is_refresh(t)
        if refresh:
            self.refresh(q, k)
        part = self.ops.partial(q, k, v, use_logits=refresh)
        parts = self.comm.all_gather(part)
        self.ops.merge(parts, out, sel_cnt)
        return out
