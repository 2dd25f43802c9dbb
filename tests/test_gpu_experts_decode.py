"""The expert path with the routing given (fmoe_experts_decode) against the oracle.

The routed experts are copied into slots of a separate device buffer, as an
expert cache holds them, in an order unrelated to their expert indices; the
call gets the slots' addresses, the combine weights and the shared gate, and
must give out = residual + sum_k w_k E_k(x) + g E_shared(x) as the oracle
computes it from the same blobs.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth as S
from tests import cases as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def F():
    from bit_quantized_expert_router_b200 import build as B
    B.build_engine()
    import synth.gpu as SG
    SG.build()
    import bit_quantized_expert_router_b200 as F
    F.lib()
    SG.lib()
    return F


def dev():
    return torch.device("cuda:0")


def oracle_given(blobs, shared, weights, sg, x, res, shape):
    H, I = shape.hidden, shape.inter
    out = np.asarray(res, dtype=np.float64).copy()
    for b, w in zip(blobs, weights):
        out += float(w) * O.expert_forward(b, H, I, shape.bits, x)
    if shared is not None:
        out += float(sg) * O.expert_forward(shared, H, I, shape.shared_bits, x)
    return out


@pytest.mark.parametrize("shape", [C.TINY, C.FULL4, C.FULL2,
                                   C.Shape("mixed_h1024_i256_e64_k8_r4_s2", 1024, 256, 64, 8, 4, 2)],
                         ids=lambda s: s.name)
def test_experts_decode_from_slots(F, shape):
    import synth.gpu as SG
    seed, layer = 41, 0
    H, I, K = shape.hidden, shape.inter, shape.top_k
    t = SG.make_layer(seed, layer, H, I, shape.n_experts, shape.bits, shape.shared_bits, F.blob_offsets,
                      F.expert_bytes, dev())
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], H, I, K, shape.bits, shape.shared_bits)
    wr = S.router_bf16(seed, layer, shape.n_experts, H)
    wsg = S.sgate_bf16(seed, layer, H)
    x = C.parity_x(seed, layer, 0, wr, K, H)[0]
    res = S.token_residual(seed, layer, 0, 1, H)[0]
    r = O.route(wr, wsg, x, K)
    # slots: a separate buffer, the selected experts in a shuffled slot order
    n_slots = K + 3
    stride = t["experts"].stride(0)
    slots = torch.zeros(n_slots, stride, dtype=torch.uint8, device=dev())
    order = np.random.default_rng(seed).permutation(n_slots)[:K]
    for k, e in enumerate(r["idx"]):
        slots[int(order[k])].copy_(t["experts"][int(e)])
    ptrs = [slots[int(order[k])].data_ptr() for k in range(K)]
    w32 = r["w"].astype(np.float32)
    sg32 = np.float32(r["sg"])
    blobs = [C.cpu_blob(seed, layer, int(e), H, I, shape.bits) for e in r["idx"]]
    shared = C.cpu_blob(seed, layer, S.SHARED_EXPERT_ID, H, I, shape.shared_bits)
    xd = torch.from_numpy(x).to(dev())
    for with_res in (True, False):
        rd = torch.from_numpy(res).to(dev()) if with_res else None
        out = F.experts_decode(L, ptrs, w32, float(sg32), xd, rd)
        assert F.get_status() == 0
        want = oracle_given(blobs, shared, w32, sg32, x, res if with_res else np.zeros(H), shape)
        C.assert_close(out.cpu().numpy(), want, f"{shape.name} residual={with_res}")
    # the same call from the layer's own table equals the routed decode's experts
    ptrs_tab = [t["experts"][int(e)].data_ptr() for e in r["idx"]]
    a = F.experts_decode(L, ptrs_tab, w32, float(sg32), xd, None)
    b = F.experts_decode(L, ptrs, w32, float(sg32), xd, None)
    assert torch.equal(a, b)


def test_experts_decode_repeated_blob_and_ungated(F):
    """The same blob listed twice with weights 1/2 each equals it once with
    weight 1; a gate of 1 is the ungated shared expert."""
    import synth.gpu as SG
    shape = C.Shape("rep_h512_i128_e16_k2", 512, 128, 16, 2, 4)
    seed, layer = 43, 0
    H, I = shape.hidden, shape.inter
    t = SG.make_layer(seed, layer, H, I, shape.n_experts, shape.bits, shape.shared_bits, F.blob_offsets,
                      F.expert_bytes, dev())
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], H, I, 2, shape.bits, shape.shared_bits)
    x = S.token_x(seed, layer, 0, 1, H)[0]
    xd = torch.from_numpy(x).to(dev())
    p5 = t["experts"][5].data_ptr()
    out = F.experts_decode(L, [p5, p5], [0.5, 0.5], 1.0, xd, None)
    assert F.get_status() == 0
    blob5 = C.cpu_blob(seed, layer, 5, H, I, shape.bits)
    shared = C.cpu_blob(seed, layer, S.SHARED_EXPERT_ID, H, I, shape.shared_bits)
    want = oracle_given([blob5], shared, [1.0], 1.0, x, np.zeros(H), shape)
    C.assert_close(out.cpu().numpy(), want, "repeated blob")
