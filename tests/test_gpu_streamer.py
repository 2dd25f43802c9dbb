"""Routed experts streamed from host memory (fmoe_streamer_*) against the oracle.

Two layers keep their routed experts in page-locked host memory and share a
few device slots, so that the tokens below evict and re-fetch experts.  For
each token and layer the streamer routes on the GPU, copies the misses into
their slots, decodes the shared expert and the hits while the copies run and
adds the misses afterwards.  Every result must match the oracle (the routing
bit for bit, the output within the layer tolerance, checked on out with and
without a residual), the hit/miss counts must equal those of a fresh LRU
directory fed the same routing decisions, and the bytes copied must be the
misses times the blob size.
"""
import numpy as np
import pytest
import torch

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


def make_streamed_layers(F, shape, seed, n_layers, with_shared):
    import synth.gpu as SG
    layers, hosts = [], []
    for l in range(n_layers):
        t = SG.make_layer(seed, l, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                          F.blob_offsets, F.expert_bytes, dev(), with_shared, True)
        stride = t["experts"].stride(0)
        host = torch.empty(shape.n_experts, stride, dtype=torch.uint8, pin_memory=True)
        host.copy_(t["experts"])
        stub = torch.zeros(1, stride, dtype=torch.uint8, device=dev())  # (the device table is not used)
        layers.append(F.Layer(t["w_router"], t["w_sgate"], stub, t["shared"], shape.hidden, shape.inter,
                              shape.top_k, shape.bits, shape.shared_bits))
        hosts.append(host)
        del t
    return layers, hosts


@pytest.mark.parametrize("shape,with_shared,n_slots", [
    (C.Shape("stream_h512_i128_e12_k4", 512, 128, 12, 4, 4), True, 6),
    (C.Shape("stream_h512_i128_e12_k4_noshared", 512, 128, 12, 4, 4), False, 5),
    (C.Shape("stream_h1024_i256_e16_k4_r2_s4", 1024, 256, 16, 4, 2, 4), True, 8),
], ids=lambda v: v.name if isinstance(v, C.Shape) else str(v))
def test_streamer_matches_oracle_across_evictions(F, shape, with_shared, n_slots):
    seed, n_layers, n_tokens = 53, 2, 8
    layers, hosts = make_streamed_layers(F, shape, seed, n_layers, with_shared)
    stride = hosts[0].shape[1]
    slots = torch.zeros(n_slots, stride, dtype=torch.uint8, device=dev())
    st = F.Streamer(layers, hosts, slots)
    copy_stream = torch.cuda.Stream()
    directory = F.ExpertCache(n_slots)  # the rule the streamer's directory must follow
    H = shape.hidden
    for t in range(n_tokens):
        for l in range(n_layers):
            wr = S.router_bf16(seed, l, shape.n_experts, H)
            x = C.parity_x(seed, l, t, wr, shape.top_k, H)[0]
            with_res = (t + l) % 2 == 0
            res = S.token_residual(seed, l, t, 1, H)[0] if with_res else np.zeros(H, dtype=np.float32)
            xd = torch.from_numpy(x).to(dev())
            rd = torch.from_numpy(res).to(dev()) if with_res else None
            out, idx, w = st.decode(l, xd, rd, copy_stream=copy_stream, return_routing=True)
            assert F.get_status() == 0
            r = C.oracle_layer(seed, l, shape, x, res, with_shared=with_shared)
            assert idx.tolist() == r["idx"].tolist(), f"token {t} layer {l}"
            C.assert_close(out.cpu().numpy(), r["out"], f"{shape.name} token {t} layer {l} residual={with_res}")
            directory.lookup(l, idx)
    s, d = st.stats(), directory.stats()
    assert (s["hits"], s["misses"]) == (d["hits"], d["misses"])
    assert s["hits"] + s["misses"] == n_tokens * n_layers * shape.top_k
    assert s["misses"] > n_slots  # experts were evicted and fetched again
    assert s["h2d_bytes"] == s["misses"] * F.expert_bytes(shape.hidden, shape.inter, shape.bits)


def test_streamer_same_stream_and_resident_agree(F):
    """Copies on the compute stream itself give the same outputs, and they
    equal the resident layer decode within fp32 rounding."""
    import synth.gpu as SG
    shape, seed = C.Shape("stream_h512_i128_e12_k4", 512, 128, 12, 4, 4), 59
    layers, hosts = make_streamed_layers(F, shape, seed, 1, True)
    stride = hosts[0].shape[1]
    t = SG.make_layer(seed, 0, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                      F.blob_offsets, F.expert_bytes, dev())
    resident = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter,
                       shape.top_k, shape.bits, shape.shared_bits)
    a = F.Streamer(layers, hosts, torch.zeros(4, stride, dtype=torch.uint8, device=dev()))
    b = F.Streamer(layers, hosts, torch.zeros(4, stride, dtype=torch.uint8, device=dev()))
    side = torch.cuda.Stream()
    wr = S.router_bf16(seed, 0, shape.n_experts, shape.hidden)
    for step in range(5):
        xd = torch.from_numpy(C.parity_x(seed, 0, step, wr, shape.top_k, shape.hidden)[0]).to(dev())
        ya = a.decode(0, xd)
        yb = b.decode(0, xd, copy_stream=side)
        yr = resident.decode(xd)
        assert F.get_status() == 0
        assert torch.equal(ya, yb)
        C.assert_close(ya.cpu().numpy(), yr.cpu().numpy(), f"step {step} vs resident")


def test_streamer_rejects_pageable_host_memory(F):
    shape, seed = C.Shape("stream_h512_i128_e12_k4", 512, 128, 12, 4, 4), 61
    layers, hosts = make_streamed_layers(F, shape, seed, 1, True)
    pageable = hosts[0].clone()  # not page-locked
    assert not pageable.is_pinned()
    slots = torch.zeros(4, hosts[0].shape[1], dtype=torch.uint8, device=dev())
    with pytest.raises(ValueError):
        F.Streamer(layers, [pageable], slots)
    import ctypes
    arr = (F.FmoeLayerC * 1)(layers[0].c)
    hp = (ctypes.c_void_p * 1)(pageable.data_ptr())
    h = ctypes.c_void_p()
    assert F.lib().fmoe_streamer_create(arr, 1, hp, slots.data_ptr(), 4, ctypes.byref(h)) == F.FMOE_EINVAL
    assert not h.value


def test_streamer_prepared_ahead_matches_oracle_and_serial(F):
    """Layers with independent inputs, each prepared while the previous one
    decodes (its misses copied during that decode): every output matches the
    oracle, the hit/miss sequence and the outputs equal the one-step decode's
    in the same order, and calls out of order are refused."""
    shape = C.Shape("stream_h512_i128_e12_k4", 512, 128, 12, 4, 4)
    seed, n_layers, n_tokens = 67, 2, 6
    layers, hosts = make_streamed_layers(F, shape, seed, n_layers, True)
    stride = hosts[0].shape[1]
    H = shape.hidden
    inputs = []
    for t in range(n_tokens):
        for l in range(n_layers):
            wr = S.router_bf16(seed, l, shape.n_experts, H)
            x = C.parity_x(seed, l, t, wr, shape.top_k, H)[0]
            inputs.append((l, torch.from_numpy(x).to(dev()), x))
    n_slots = 2 * shape.top_k  # the least a prepared-ahead layer needs
    piped = F.Streamer(layers, hosts, torch.zeros(n_slots, stride, dtype=torch.uint8, device=dev()))
    serial = F.Streamer(layers, hosts, torch.zeros(n_slots, stride, dtype=torch.uint8, device=dev()))
    copy_a, copy_b, route_s = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ws = layers[0].workspace(1)
    outs = [torch.empty(H, device=dev()) for _ in inputs]
    routes = [None] * len(inputs)
    l0, xd0, _ = inputs[0]
    routes[0] = piped.prepare(l0, xd0, route_stream=route_s, copy_stream=copy_a)
    for i, (l, xd, _) in enumerate(inputs):
        if i + 1 < len(inputs):
            ln, xn, _ = inputs[i + 1]
            routes[i + 1] = piped.prepare(ln, xn, route_stream=route_s, copy_stream=copy_a)
            # a third layer may not be prepared while two are pending
            with pytest.raises(F.FmoeError):
                piped.prepare(ln, xn, route_stream=route_s, copy_stream=copy_a)
        piped.finish(l, xd, out=outs[i], ws=ws)
    torch.cuda.synchronize()
    assert F.get_status() == 0
    for i, (l, xd, x) in enumerate(inputs):
        r = C.oracle_layer(seed, l, shape, x, np.zeros(H, dtype=np.float32))
        assert routes[i][0].tolist() == r["idx"].tolist()
        C.assert_close(outs[i].cpu().numpy(), r["out"], f"prepared-ahead input {i}")
        ys = serial.decode(l, xd, copy_stream=copy_b)
        assert torch.equal(ys, outs[i]), f"input {i}: prepared-ahead and one-step decodes differ"
    assert piped.stats() == serial.stats()
    # finishing a layer that is not the oldest prepared one is refused
    piped.prepare(0, inputs[0][1], route_stream=route_s, copy_stream=copy_a)
    with pytest.raises(F.FmoeError):
        piped.finish(1, inputs[1][1], ws=ws)
    with pytest.raises(F.FmoeError):  # and so is a one-step decode while a layer is prepared
        piped.decode(1, inputs[1][1], copy_stream=copy_a)
    piped.finish(0, inputs[0][1], ws=ws)
    torch.cuda.synchronize()
    assert F.get_status() == 0
