"""The allocation-free decode entry point against the regular one.

fmoe_layer_decode_noalloc serves callers that cannot allocate device memory
(for instance code running inside another runtime's fixed memory budget, or a
plain C caller without a device allocator): it takes its workspace from a fixed
device array inside the library.  Here it is called through the C ABI twice in
a row and each result is compared with fmoe_layer_decode given a normal
workspace, at the same tolerance as the other layer tests.  The file is named
so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth as S
from tests import cases as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    from bit_quantized_expert_router_b200 import build as B
    import synth.gpu as SG
    B.build_engine()
    SG.build()
    import bit_quantized_expert_router_b200 as F
    F.lib()
    SG.lib()
    return F


@pytest.mark.parametrize("shape", [C.TINY, C.FULL4], ids=lambda s: s.name)
def test_noalloc_matches_workspace_entry_point(F, shape):
    import synth.gpu as SG
    dev = torch.device("cuda:0")
    seed, layer = 31, 0
    t = SG.make_layer(seed, layer, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                      F.blob_offsets, F.expert_bytes, dev)
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter, shape.top_k,
                shape.bits, shape.shared_bits)
    wr = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    stream = torch.cuda.current_stream().cuda_stream
    for step in range(2):  # two calls in a row: the shared scratch must not carry state between them
        x = torch.from_numpy(C.parity_x(seed, layer, step, wr, shape.top_k, shape.hidden)[0]).to(dev)
        res = torch.from_numpy(S.token_residual(seed, layer, step, 1, shape.hidden)[0]).to(dev)
        want = L.decode(x, res).clone()
        want_idx = torch.empty(1, shape.top_k, dtype=torch.int32, device=dev)
        L.decode(x, res, idx_out=want_idx)
        out = torch.empty(1, shape.hidden, dtype=torch.float32, device=dev)
        idx = torch.empty(1, shape.top_k, dtype=torch.int32, device=dev)
        rc = F.lib().fmoe_layer_decode_noalloc(ctypes.byref(L.c), x.data_ptr(), res.data_ptr(), out.data_ptr(), 1,
                                               idx.data_ptr(), None, stream)
        assert rc == F.FMOE_OK, F.strerror(rc)
        assert F.get_status() == 0
        assert torch.equal(idx, want_idx)
        C.assert_close(out.cpu().numpy(), want.cpu().numpy(), f"{shape.name} call {step}")


def test_noalloc_rejects_oversized_layer(F):
    # the largest single-token layer fits the fixed scratch: its workspace is
    # the header alone, whatever the shape
    base = dict(w_router=1 << 20, w_sgate=1 << 20, experts=1 << 20, expert_stride=1 << 24, shared=1 << 20,
                hidden=8192, inter=2048, n_experts=1024, top_k=4, bits=4, shared_bits=4, group=64)
    c = F.FmoeLayerC(**base)
    assert F.lib().fmoe_workspace_bytes(ctypes.byref(c), 1) <= 128 * 1024
    # a layer above the decode's limit ((K+1)*I > 10240) is refused on the host
    big = F.FmoeLayerC(**{**base, "inter": 4096})
    rc = F.lib().fmoe_layer_decode_noalloc(ctypes.byref(big), 1 << 20, None, 1 << 21, 1, None, None,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == F.FMOE_EINVAL
    # grouped calls (T > 1) are not served: refused on the host, nothing enqueued
    small = F.FmoeLayerC(**{**base, "hidden": 512, "inter": 128, "n_experts": 16})
    rc = F.lib().fmoe_layer_decode_noalloc(ctypes.byref(small), 1 << 20, None, 1 << 21, 2, None, None,
                                           torch.cuda.current_stream().cuda_stream)
    assert rc == F.FMOE_EINVAL
    assert F.get_status() == 0
