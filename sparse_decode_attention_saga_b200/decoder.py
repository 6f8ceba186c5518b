"""Host-side driver of the decode loop over the C ABI.

``AtopNDecoder`` owns the caller-side state the method needs (the threshold
tensor, the workspace and a logits buffer for refresh steps) and applies the
refresh schedule of "More Value per Key" (ai.info summary, Key Contributions
#2: exact top-N thresholds computed once every n tokens and reused between):
step t refreshes when t mod n == 0, then decodes with the stored thresholds.
Every step is two or three C calls; all compute runs in libsaga.so.
"""
from __future__ import annotations

import torch

from . import _lib


class AtopNDecoder:
    def __init__(self, batch, h_q, h_k, h_v, head_dim, l_kv, N, n, l_cap=None, device="cuda"):
        self.dims = _lib.dims(batch, h_q, h_k, h_v, head_dim, l_kv, l_cap)
        self.N, self.n = int(N), int(n)
        self.device = torch.device(device)
        nbytes = _lib.workspace_bytes(self.dims, self.N)
        if nbytes == 0:
            raise _lib.SagaError("saga_workspace_bytes", _lib.SAGA_ERR_UNSUPPORTED)
        self.ws = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        self.thresh = torch.full((batch, h_q), float("nan"), dtype=torch.float32, device=self.device)
        self.logits = torch.empty((batch, h_q, l_kv), dtype=torch.float32, device=self.device)
        self.out = torch.empty((batch, h_q, head_dim), dtype=torch.float32, device=self.device)

    @classmethod
    def for_workload(cls, w, device="cuda"):
        return cls(w.batch, w.h_q, w.h_k, w.h_v, w.head_dim, w.l_kv, w.N, w.n, w.cap, device)

    def is_refresh(self, t: int) -> bool:
        return t % self.n == 0

    def refresh(self, q, k, stream=None) -> None:
        """Exact thresholds from this step's logits (kept in self.logits)."""
        _lib.topn_refresh(self.dims, self.N, q, k, None, self.logits, self.thresh, self.ws, stream)

    def step(self, t: int, q, k, v, out=None, sel_idx=None, sel_cnt=None, stream=None):
        """Decode step t: refresh if t mod n == 0, then Atop-N attention."""
        out = self.out if out is None else out
        if self.is_refresh(t):
            self.refresh(q, k, stream)
            _lib.atopn_decode(self.dims, q, k, v, self.thresh, self.logits, out, sel_idx, sel_cnt,
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
