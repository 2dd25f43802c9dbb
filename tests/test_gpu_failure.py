"""Failure detection on the GPU without a fault: a time-limited wait that runs out.

The layer kernel's CTAs hand off through counters in the caller's workspace.
Here the activation hand-off counter is left at a value no launch can bring
to its target (as if the workspace had not been zeroed), with a short wait
limit.  Every wait on it must run out, the kernel must end on its own and
report through the status word, the context must stay usable, and the next
launch on the same workspace must be correct again (the kernel's last CTA
resets the counter on its way out).  A CTA whose wait ran out writes NaN to its
output rows, so the result of the starved launch is not plausible numbers.
Both launch modes (programmatic dependent and cooperative) are covered.
"""
import numpy as np
import pytest
import torch

import synth as S
from tests import cases as C

pytestmark = pytest.mark.gpu

STATUS_GRID_BARRIER_TIMEOUT = 1


@pytest.fixture(scope="module")
def F():
    from bit_quantized_expert_router_b200 import build as B
    B.build_engine()
    import synth.gpu as SG
    SG.build()
    import bit_quantized_expert_router_b200 as F
    F.lib()
    assert torch.cuda.is_available()
    return F


def test_wait_limit_bounds(F):
    with pytest.raises(F.FmoeError):
        F.set_wait_limit_ns(10)
    with pytest.raises(F.FmoeError):
        F.set_wait_limit_ns(10 ** 12)
    prev = F.set_wait_limit_ns(2_000_000_000)
    assert F.set_wait_limit_ns(prev) == 2_000_000_000


@pytest.mark.parametrize("dependent", [True, False], ids=["dependent_launch", "cooperative_launch"])
def test_unreachable_counter_times_out_and_recovers(F, dependent):
    prev_mode = F.set_dependent_launch(dependent)
    try:
        unreachable_counter_case(F)
    finally:
        F.set_dependent_launch(prev_mode)


def unreachable_counter_case(F):
    import synth.gpu as SG
    shape, seed, layer = C.TINY, 21, 0
    dev = torch.device("cuda:0")
    t = SG.make_layer(seed, layer, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                      F.blob_offsets, F.expert_bytes, dev)
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter, shape.top_k,
                shape.bits, shape.shared_bits)
    wr = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    x = C.parity_x(seed, layer, 0, wr, shape.top_k, shape.hidden)[0]
    res = S.token_residual(seed, layer, 0, 1, shape.hidden)[0]
    xd, rd = torch.from_numpy(x).to(dev), torch.from_numpy(res).to(dev)
    ws = L.workspace(1)
    assert F.get_status() == 0

    prev = F.set_wait_limit_ns(20_000_000)  # 20 ms
    try:
        counters = ws[:12].view(torch.int32)
        epoch = int(counters[0])
        counters[1:2].fill_(-1024)  # hand-off counter 0xFFFFFC00: above any grid size, never "reached"
        out = L.decode(xd, rd, ws=ws)
        bits = F.get_status()  # synchronises: the launch ended on its own
        assert bits & STATUS_GRID_BARRIER_TIMEOUT, f"status bits {bits:#x}"
        assert F.get_status() == 0  # read-and-clear
        # every CTA waited in vain at the hand-off: every output row is NaN
        assert torch.isnan(out).all()
        # the last CTA advanced the launch epoch and put both hand-off
        # counters back to zero
        assert counters.cpu().tolist() == [epoch + 1, 0, 0]
    finally:
        F.set_wait_limit_ns(prev)

    out = L.decode(xd, rd, ws=ws)
    assert F.get_status() == 0
    r = C.oracle_layer(seed, layer, shape, x, res)
    C.assert_close(out.cpu().numpy()[0], r["out"], "after recovery")
    assert np.isfinite(out.cpu().numpy()).all()
