"""Shared helpers of the GPU parity tests: run the CUDA path through the C
ABI, run the oracle on the same seeded inputs, compare with the stated
tolerances.

Tolerances (north star of the method's port):
  * thresholds and masks: bit-exact when both sides see identical logits;
  * end to end: masks may differ only where |s - tau| <= 1e-4 |tau| (oracle's
    logits and threshold);
  * outputs: |gpu - oracle| <= 1e-3 + 1e-3 |oracle|, the oracle evaluated
    with the GPU's mask so a legitimate borderline flip is not counted twice;
  * logits: |gpu - oracle| <= 1e-4 + 1e-5 |s| (fp32 tensor-core accumulation
    of exact bf16 products versus one rounding of the float64 sum).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import bf16_bits, make_cache, make_queries

OUT_ATOL = 1e-3
OUT_RTOL = 1e-3
BAND = 1e-4
LOGIT_ATOL = 1e-4
LOGIT_RTOL = 1e-5


def device_inputs(w, seed=0, steps=None, gen_device="cuda"):
    K, V = make_cache(w, seed, gen_device)
    qs = make_queries(w, seed, gen_device, steps)
    return qs.cuda(), K.cuda(), V.cuda()


def mask_from_lists(idx: torch.Tensor, cnt: torch.Tensor, l: int) -> np.ndarray:
    idx = idx.cpu().numpy()
    cnt = cnt.cpu().numpy()
    b, hq = cnt.shape
    mask = np.zeros((b, hq, l), bool)
    for bb in range(b):
        for i in range(hq):
            c = int(cnt[bb, i])
            sel = idx[bb, i, :c]
            assert np.all(np.diff(sel) > 0), "kept positions must be strictly ascending"
            assert c == 0 or (sel[0] >= 0 and sel[-1] < l)
            mask[bb, i, sel] = True
    return mask


def assert_outputs_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    err = np.abs(gpu - ref)
    bound = OUT_ATOL + OUT_RTOL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} outputs outside 1e-3+1e-3|o|; "
                           f"max err {err.max():.3g} at {np.unravel_index(err.argmax(), err.shape)}")


def assert_mask_within_band(mask_gpu, mask_ref, s_ref, tau_ref, what=""):
    diff = mask_gpu != mask_ref
    if not diff.any():
        return 0
    tau = tau_ref[..., None].astype(np.float64)
    near = np.abs(s_ref.astype(np.float64) - tau) <= BAND * np.abs(tau)
    outside = diff & ~near
    assert not outside.any(), f"{what}: {outside.sum()} mask differences outside the 1e-4|tau| band"
    return int(diff.sum())


def gpu_step_with_mask(dec: AtopNDecoder, t, q, K, V):
    """Decode step t through the path that emits the kept positions."""
    b, hq = dec.thresh.shape
    l = dec.dims.l_kv
    idx = torch.full((b, hq, l), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((b, hq), dtype=torch.int32, device="cuda")
    out = torch.empty_like(dec.out)
    dec.step(t, q, K, V, out=out, sel_idx=idx, sel_cnt=cnt)
    return out, idx, cnt


def bits(t: torch.Tensor) -> np.ndarray:
    return bf16_bits(t)


def gpu_logits(dec: AtopNDecoder, q, K) -> torch.Tensor:
    """This step's logits [b, h_q, l_kv] from the library's logits kernel,
    which shares its tensor-core routine with the fused compare."""
    d = dec.dims
    s = torch.empty((d.batch, d.h_q, d.l_kv), dtype=torch.float32, device="cuda")
    _lib.qk_logits(d, q, K, s, dec.ws)
    return s


def assert_mask_exact(dec: AtopNDecoder, q, K, idx, cnt, rows=None, what=""):
    """The kept positions a decode step emitted equal, bit for bit, the
    oracle's selection over the GPU's own logits of that step and the
    thresholds it used (identical logits must give identical masks)."""
    s = gpu_logits(dec, q, K)
    torch.cuda.synchronize()
    sel = list(range(s.shape[0])) if rows is None else list(rows)
    s_h = s[sel].cpu().numpy()
    tau = dec.thresh[sel].cpu().numpy()
    mask_ref, cnt_ref = oracle.select(s_h, tau)
    got_cnt = cnt[sel].cpu().numpy()
    assert np.array_equal(got_cnt, cnt_ref), f"{what}: kept counts differ in {(got_cnt != cnt_ref).sum()} rows"
    mask_gpu = mask_from_lists(idx[sel], cnt[sel], s_h.shape[-1])
    assert np.array_equal(mask_gpu, mask_ref), f"{what}: {(mask_gpu != mask_ref).sum()} mask entries differ"
