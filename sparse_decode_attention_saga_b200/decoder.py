"""Host-side driver of the decode loop over the C ABI.

``AtopNDecoder`` owns the caller-side state the method needs (the threshold
tensor, the workspace and a logits buffer for refresh steps) and applies the
refresh schedule of "More Value per Key" (ai.info summary, Key Contributions
#2: the exact threshold is recomputed on every n-th token only and reused on
the tokens in between):
step t refreshes when t mod n == 0, then decodes with the stored thresholds.
Every step is one C call; all compute runs in libsaga.so.
``HostLoop`` (``AtopNDecoder.host_loop``) runs a span of steps as one CUDA
graph fed from, and writing to, pinned host memory.
"""
from __future__ import annotations

import torch

from . import _lib


class AtopNDecoder:
    """Decode-loop state for one layer.  The cache holds l_kv valid rows out of
    l_cap; ``append`` adds the step's own key/value rows (the cached length
    grows by one), so buffers are sized for l_cap."""

    def __init__(self, batch, h_q, h_k, h_v, head_dim, l_kv, N, n, l_cap=None, device="cuda",
                 v_head_dim=None):
        self.l_cap = int(l_kv if l_cap is None else l_cap)
        self.dv = int(head_dim if v_head_dim is None else v_head_dim)
        self.dims = _lib.dims(batch, h_q, h_k, h_v, head_dim, l_kv, self.l_cap, self.dv)
        self.N, self.n = int(N), int(n)
        self.device = torch.device(device)
        # a workspace sized for the full capacity serves every shorter length
        nbytes = _lib.workspace_bytes(_lib.dims(batch, h_q, h_k, h_v, head_dim, self.l_cap,
                                                self.l_cap, self.dv), self.N)
        if nbytes == 0:
            raise _lib.SagaError("saga_workspace_bytes", _lib.SAGA_ERR_UNSUPPORTED)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.thresh = torch.full((batch, h_q), float("nan"), dtype=torch.float32, device=self.device)
        self._logits = torch.empty(batch * h_q * self.l_cap, dtype=torch.float32, device=self.device)
        self.out = torch.empty((batch, h_q, self.dv), dtype=torch.float32, device=self.device)

    @property
    def l_kv(self) -> int:
        return int(self.dims.l_kv)

    @property
    def logits(self) -> torch.Tensor:
        """[b, h_q, l_kv] view of the logits buffer (written on refresh steps)."""
        d = self.dims
        return self._logits[: d.batch * d.h_q * d.l_kv].view(d.batch, d.h_q, d.l_kv)

    def append(self, k_new, v_new, k, v, stream=None) -> None:
        """Writes this step's key/value rows ([b,h_k,d], [b,h_v,d_v] bf16) at
        position l_kv of the caches; the following steps see l_kv + 1 rows."""
        _lib.cache_append(self.dims, k_new, v_new, k, v, stream)
        d = self.dims
        self.dims = _lib.dims(d.batch, d.h_q, d.h_k, d.h_v, d.head_dim, d.l_kv + 1, self.l_cap,
                              self.dv)

    @classmethod
    def for_workload(cls, w, device="cuda"):
        return cls(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, w.l_kv, w.N, w.n, w.cap, device,
                   w.dv)

    def is_refresh(self, t: int) -> bool:
        return t % self.n == 0

    def refresh(self, q, k, stream=None) -> None:
        """Exact thresholds from this step's logits (kept in self.logits);
        ``step`` refreshes through the workspace instead, in the same call as
        the decode."""
        _lib.topn_refresh(self.dims, self.N, q, k, None, self.logits, self.thresh, self.ws, stream)

    def step(self, t: int, q, k, v, out=None, sel_idx=None, sel_cnt=None, stream=None):
        """Decode step t: refresh if t mod n == 0, then Atop-N attention."""
        out = self.out if out is None else out
        if self.is_refresh(t):
            _lib.atopn_refresh_step(self.dims, self.N, q, k, v, self.thresh, out, sel_idx, sel_cnt,
                                    self.ws, stream)
        else:
            _lib.atopn_decode(self.dims, q, k, v, self.thresh, None, out, sel_idx, sel_cnt,
                              self.ws, stream)
        return out

    def dense(self, q, k, v, out=None, stream=None):
        out = self.out if out is None else out
        _lib.decode_dense(self.dims, q, k, v, out, self.ws, stream)
        return out

    def error(self, stream=None) -> int:
        return _lib.workspace_error(self.ws, stream)

    def empty_rows(self, stream=None) -> int:
        """Rows that kept nothing and took the empty-set rule (their maxima)
        since the last call."""
        return _lib.workspace_empty_rows(self.ws, stream)

    def host_loop(self, k, v, q_host, out_host, t0: int, steps: int, stream=None,
                  restore: bool = True) -> "HostLoop":
        """Captures decode steps t0 .. t0 + steps - 1 fed from pinned host
        memory (see HostLoop); the decoder must have run a step outside a
        capture first, and its cached length stays fixed inside the loop."""
        return HostLoop(self, k, v, q_host, out_host, t0, steps, stream, restore)


class HostLoop:
    """A decode loop whose queries come from, and whose outputs go to, pinned
    host memory: step t copies q_host[t] in and its output out to
    out_host[t - t0].  One CUDA graph holds all the steps; the copies run on
    two copy streams into and out of double buffers, so that they overlap the
    kernels of the neighbouring steps: query buffer t mod 2 is refilled once
    step t - 2 has run, and output buffer t mod 2 is rewritten once its copy
    of step t - 2 is out.  The graph keeps the addresses of k, v, the host
    buffers and the decoder's state, so the loop holds references to all of
    them; replay() enqueues the whole loop on the loop's stream (a side
    stream: a capture cannot run on the default stream).

    Thresholds entering t0: the steps before the loop's first refresh reuse
    the thresholds of the refresh that opened t0's period (step t0 - t0 mod n,
    from q_host of that step).  With restore=True (default) and t0 not a
    refresh step, that refresh heads the graph, so every replay gives the
    outputs of running steps t0 - t0 mod n .. t0 + steps - 1 one by one.
    With restore=False the graph holds only the loop's own steps and the
    caller puts that state in place before each replay (restore_state(), or
    the steps before t0 run on the same decoder)."""

    def __init__(self, dec, k, v, q_host, out_host, t0, steps, stream=None, restore=True):
        steps, t0 = int(steps), int(t0)
        if steps < 1 or t0 < 0 or q_host.shape[0] < t0 + steps or out_host.shape[0] < steps:
            raise ValueError("host buffers do not cover the steps")
        if not (q_host.is_pinned() and out_host.is_pinned()):
            raise ValueError("host buffers must be pinned")
        self.stream = torch.cuda.Stream() if stream is None else stream
        self.q_host, self.out_host = q_host, out_host
        self.t0, self.t_open = t0, t0 - t0 % dec.n  # step whose refresh holds for t0
        self._keep = (dec, k, v)  # the graph reads their memory on every replay
        self._h2d, self._d2h = torch.cuda.Stream(), torch.cuda.Stream()
        self._q = [torch.empty(q_host.shape[1:], dtype=q_host.dtype, device=dec.device)
                   for _ in range(2)]
        self._q_open = torch.empty(q_host.shape[1:], dtype=q_host.dtype, device=dec.device)
        self._o = [torch.empty_like(dec.out) for _ in range(2)]
        done = [torch.cuda.Event() for _ in range(steps)]
        q_in = [torch.cuda.Event() for _ in range(steps)]
        o_out = [torch.cuda.Event() for _ in range(steps)]
        torch.cuda.synchronize()  # buffers made on other streams are ready
        s, h2d, d2h = self.stream, self._h2d, self._d2h
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=s):
            if restore and self.t_open < t0:
                self._open_period(s)
            h2d.wait_stream(s)  # the copy streams join the capture
            d2h.wait_stream(s)
            for i in range(steps):
                t = t0 + i
                with torch.cuda.stream(h2d):
                    if i >= 2:
                        h2d.wait_event(done[i - 2])
                    self._q[i % 2].copy_(q_host[t], non_blocking=True)
                    q_in[i].record(h2d)
                s.wait_event(q_in[i])
                if i >= 2:
                    s.wait_event(o_out[i - 2])
                dec.step(t, self._q[i % 2], k, v, out=self._o[i % 2])
                done[i].record(s)
                with torch.cuda.stream(d2h):
                    d2h.wait_event(done[i])
                    out_host[i].copy_(self._o[i % 2], non_blocking=True)
                    o_out[i].record(d2h)
            s.wait_stream(h2d)
            s.wait_stream(d2h)

    def _open_period(self, s) -> None:
        """The refresh of step t_open on stream s (its query from q_host)."""
        dec, k, _ = self._keep
        with torch.cuda.stream(s):
            self._q_open.copy_(self.q_host[self.t_open], non_blocking=True)
            dec.refresh(self._q_open, k)

    def restore_state(self) -> None:
        """Enqueues, outside the graph, the refresh that opened t0's period
        (nothing when t0 is a refresh step): the state a loop built with
        restore=False expects at the start of each replay."""
        if self.t_open < self.t0:
            self._open_period(self.stream)

    def replay(self) -> None:
        """Enqueues the loop on its stream (asynchronous: synchronise the
        stream before reading out_host)."""
        with torch.cuda.stream(self.stream):
            self.graph.replay()
