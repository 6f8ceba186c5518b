"""AtopNDecoder.host_loop: decode steps fed from pinned host queries, with
their outputs written to pinned host memory (one CUDA graph; the copies on
two copy streams with double buffers) give, bit for bit, the outputs of the
same steps run one by one on device buffers, and the same again on a second
replay, also when the loop starts inside a refresh period."""
import pytest
import torch

from sparse_decode_attention_saga_b200 import _lib
from sparse_decode_attention_saga_b200.decoder import AtopNDecoder
from sparse_decode_attention_saga_b200.workload import Workload

from .gpu_helpers import device_inputs

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():  # collected on CPU boxes, selected out by -m "not gpu"
    pytest.skip("needs a CUDA device", allow_module_level=True)


@pytest.mark.parametrize("restore", [True, False], ids=["restore_in_graph", "restore_state"])
@pytest.mark.parametrize("t0,steps", [(0, 1), (0, 2), (3, 7), (6, 12), (4, 5), (2, 1)],
                         ids=["one", "two", "from_3_seven", "from_6_twelve", "mid_period_4_five",
                              "mid_period_2_one"])
def test_host_loop_matches_device_steps(t0, steps, restore):
    w = Workload("host_loop", 2, 8, 2, 4, 64, 1000, 25, 3, steps=t0 + steps)
    qs, K, V = device_inputs(w, seed=61)
    ref = AtopNDecoder.for_workload(w)
    expect = []
    for t in range(t0 + steps):
        o = ref.step(t, qs[t], K, V)
        if t >= t0:
            expect.append(o.cpu())
    dec = AtopNDecoder.for_workload(w)
    dec.step(0, qs[0], K, V)  # one call outside a capture
    # thresholds that belong to no step of this loop: a replay must not use them
    dec.thresh.fill_(0.5)
    q_host = qs.cpu().pin_memory()
    out_host = torch.empty((steps,) + tuple(dec.out.shape), dtype=torch.float32).pin_memory()
    torch.cuda.synchronize()
    loop = dec.host_loop(K, V, q_host, out_host, t0, steps, restore=restore)
    for rep in range(2):
        out_host.fill_(float("nan"))
        if not restore:
            loop.restore_state()
        loop.replay()
        loop.stream.synchronize()
        for i in range(steps):
            assert torch.equal(out_host[i], expect[i]), f"replay {rep}, step {t0 + i}"
    assert dec.error() == _lib.SAGA_OK
