"""Seeded synthetic decode workloads (shapes + random inputs only).

This module holds the workload shapes and the seeded input recipe shared by
the tests, the benchmark and the smoke check.  It contains none of the
attention arithmetic: it only draws bf16 tensors.

Shapes follow the decode layers the pages measure ("More Value per Key",
ai.info summary, "Main Findings": Llama 3.2-1B with h_k 8 -> 4 and
Qwen2.5-1.5B with h_k 2 -> 1, contexts 8K-128K, N in {512, 1024, 2048},
32 generated tokens).

Input recipe (the same on every device, deterministic per seed):
  * a unit "topic" vector u_k per key head (shared across the batch);
  * K, V ~ N(0, 1) in fp32, rounded to bf16 (round-to-nearest-even);
  * for each (batch, key head) a seeded random 2 % of the positions get
    2 * u_k added to K before rounding (V is not shifted);
  * the query of head i at each step is bf16(2 * u_{k(i)} + N(0, 1)), drawn
    fresh per step, where k(i) is the key head whose group holds query head
    i (contiguous groups of h_q / h_k query heads).
"""
from __future__ import annotations

import dataclasses

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    h_q: int
    h_k: int
    h_v: int
    head_dim: int
    l_kv: int
    N: int
    n: int
    steps: int = 32
    l_cap: int | None = None
    v_head_dim: int | None = None  # value head dim where it differs from head_dim

    @property
    def cap(self) -> int:
        return self.l_kv if self.l_cap is None else self.l_cap

    @property
    def dv(self) -> int:
        return self.head_dim if self.v_head_dim is None else self.v_head_dim

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _sweep():
    out = {}
    for b in (1, 16):
        for l in (8192, 16384, 32768, 65536, 131072):
            name = f"llama_sweep_b{b}_l{l // 1024}k"
            out[name] = Workload(name, b, 32, 4, 8, 64, l, 1024, 16)
    return out


def _headcount():
    out = {}
    for kind, hk in (("gqa", 2), ("saga", 1)):
        for N in (512, 1024, 2048):
            name = f"qwen_b16_128k_{kind}_N{N}"
            out[name] = Workload(name, 16, 12, hk, 2, 128, 131072, N, 16)
    return out


CONFIGS: dict[str, Workload] = {
    # small case the oracle finishes in well under a second
    "tiny": Workload("tiny", 1, 4, 1, 2, 64, 2048, 64, 8),
    # Qwen2.5-1.5B-shaped SAGA layer, batch 1, 32K context
    "qwen_b1_32k": Workload("qwen_b1_32k", 1, 12, 1, 2, 128, 32768, 1024, 16),
    # Llama-3.2-1B-shaped SAGA layer, batch 16, 128K context
    "llama_b16_128k": Workload("llama_b16_128k", 16, 32, 4, 8, 64, 131072, 2048, 16),
    **_headcount(),
    **_sweep(),
    # keys narrower than values (the pages' Sigma-style head layout: (h_k, d_k)
    # = (2, 32) next to h_v = 8, d_v = 64, h_q 16), batch 16, 128K context
    "sigma_b16_128k": Workload("sigma_b16_128k", 16, 16, 2, 8, 32, 131072, 2048, 16,
                               v_head_dim=64),
}

TOPIC_FRACTION = 0.02
TOPIC_SHIFT = 2.0


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def topic_vectors(w: Workload, seed: int, device="cpu") -> torch.Tensor:
    """[h_k, d] fp32 unit vectors, one per key head."""
    g = _gen(seed * 7919 + 1, device)
    u = torch.randn(w.h_k, w.head_dim, generator=g, device=device, dtype=torch.float32)
    return u / u.norm(dim=-1, keepdim=True)


def make_cache(w: Workload, seed: int = 0, device="cpu"):
    """Returns (K [b,l_cap,h_k,d] bf16, V [b,l_cap,h_v,d_v] bf16).

    Drawn one batch element at a time so the fp32 temporaries stay small.
    Rows at positions >= l_kv (spare capacity) are drawn like the others.
    """
    u = topic_vectors(w, seed, device)
    g = _gen(seed * 7919 + 2, device)
    b, L, hk, hv, d, dv = w.batch, w.cap, w.h_k, w.h_v, w.head_dim, w.dv
    K = torch.empty(b, L, hk, d, dtype=torch.bfloat16, device=device)
    V = torch.empty(b, L, hv, dv, dtype=torch.bfloat16, device=device)
    n_topic = max(1, int(round(TOPIC_FRACTION * w.l_kv)))
    for bb in range(b):
        kf = torch.randn(L, hk, d, generator=g, device=device, dtype=torch.float32)
        for kh in range(hk):
            pos = torch.randperm(w.l_kv, generator=g, device=device)[:n_topic]
            kf[pos, kh, :] += TOPIC_SHIFT * u[kh]
        K[bb] = kf.to(torch.bfloat16)
        del kf
        V[bb] = torch.randn(L, hv, dv, generator=g, device=device,
                            dtype=torch.float32).to(torch.bfloat16)
    return K, V


def make_queries(w: Workload, seed: int = 0, device="cpu", steps: int | None = None):
    """[steps, b, h_q, d] bf16: step t's query is 2*u_{k(i)} + N(0,1)."""
    steps = w.steps if steps is None else steps
    u = topic_vectors(w, seed, device)
    g = _gen(seed * 7919 + 3, device)
    group = torch.arange(w.h_q, device=device) // (w.h_q // w.h_k)
    base = TOPIC_SHIFT * u[group]  # [h_q, d]
    z = torch.randn(steps, w.batch, w.h_q, w.head_dim, generator=g, device=device,
                    dtype=torch.float32)
    return (z + base).to(torch.bfloat16)


def make_new_rows(w: Workload, seed: int = 0, device="cpu", steps: int | None = None):
    """Key and value rows generated one per decode step, for a growing cache:
    ([steps, b, h_k, d], [steps, b, h_v, d_v]) bf16, drawn like the cache rows
    (N(0,1); each (step, batch, key head) key row gets 2*u_k added with
    probability 2 %)."""
    steps = w.steps if steps is None else steps
    u = topic_vectors(w, seed, device)
    g = _gen(seed * 7919 + 4, device)
    kf = torch.randn(steps, w.batch, w.h_k, w.head_dim, generator=g, device=device,
                     dtype=torch.float32)
    shift = torch.rand(steps, w.batch, w.h_k, generator=g, device=device) < TOPIC_FRACTION
    kf += TOPIC_SHIFT * shift[..., None].float() * u[None, None]
    vf = torch.randn(steps, w.batch, w.h_v, w.dv, generator=g, device=device,
                     dtype=torch.float32)
    return kf.to(torch.bfloat16), vf.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """A bf16 tensor as a numpy uint16 array of its bit patterns (host copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


def kv_cache_bytes(batch: int, l: int, h_k: int, h_v: int, head_dim: int,
                   elem_bytes: int = 2) -> int:
    """Bytes of a K + V cache with h_k key heads and h_v value heads."""
    return batch * l * (h_k + h_v) * head_dim * elem_bytes
