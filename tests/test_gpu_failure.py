"""Failure detection on the GPU without a fault: a time-limited wait that runs out.

The layer kernel's CTAs hand off through words in the caller's workspace
tagged with the launch's epoch + 1.  Here the epoch is left at a value no
launch leaves behind (top bit set, as if the workspace had not been zeroed),
with a short wait limit: such a launch tags nothing, so every tagged wait (the
router logits, the activations) must run out.  The kernel must end on its own
and report through the status word, the context must stay usable, and the next
launch on the same workspace must be correct again (the kernel's last CTA
restarts the epoch at 0 and clears the tagged words on its way out).  A CTA
whose wait ran out writes NaN to its output rows, so the result of the starved
launch is not plausible numbers.  Both launch modes (programmatic dependent and
cooperative) are covered.
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
def test_invalid_epoch_times_out_and_recovers(F, dependent):
    prev_mode = F.set_dependent_launch(dependent)
    try:
        invalid_epoch_case(F)
    finally:
        F.set_dependent_launch(prev_mode)


def invalid_epoch_case(F):
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
        counters[0:1].fill_(-1024)  # epoch 0xFFFFFC00: no launch leaves it, so this one tags nothing
        tagged = ws[256:256 + (1025 * 8 + 255) // 256 * 256 + 10240 * 8]
        tagged.fill_(0x5A)  # stale words (their tags never match either)
        out = L.decode(xd, rd, ws=ws)
        bits = F.get_status()  # synchronises: the launch ended on its own
        assert bits & STATUS_GRID_BARRIER_TIMEOUT, f"status bits {bits:#x}"
        assert F.get_status() == 0  # read-and-clear
        # every CTA waited in vain for the logits: every output row is NaN
        assert torch.isnan(out).all()
        # the last CTA restarted the epoch at 0, reset the counters and
        # cleared every tagged word
        assert counters.cpu().tolist() == [0, 0, 0]
        tlog_words = tagged[:1025 * 8].cpu()  # (the rest of its 256-byte block is padding, never read)
        tact_words = tagged[(1025 * 8 + 255) // 256 * 256:].cpu()
        assert (tlog_words == 0).all() and (tact_words == 0).all()
    finally:
        F.set_wait_limit_ns(prev)

    out = L.decode(xd, rd, ws=ws)
    assert F.get_status() == 0
    r = C.oracle_layer(seed, layer, shape, x, res)
    C.assert_close(out.cpu().numpy()[0], r["out"], "after recovery")
    assert np.isfinite(out.cpu().numpy()).all()
