"""CUDA engine (through the C ABI) against the fp64 oracle, on seeded inputs.

Integer results (packed codes, selected experts) must match bit for bit; fp32
outputs must be within max-abs 2e-3 and relative L2 1e-4 of the oracle.
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
    assert torch.cuda.is_available()
    return F


@pytest.fixture(scope="module")
def SG(F):
    import synth.gpu as SG
    return SG


def dev():
    return torch.device("cuda:0")


def make_gpu_layer(F, SG, seed, layer, shape: C.Shape, with_shared=True, with_sgate=True):
    t = SG.make_layer(seed, layer, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                      F.blob_offsets, F.expert_bytes, dev(), with_shared, with_sgate)
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter, shape.top_k,
                shape.bits, shape.shared_bits)
    return L, t


# ---------------------------------------------------------------------------
# Generator and layout agreement
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hidden,inter,bits", [(512, 128, 4), (4096, 1024, 4), (4096, 1024, 2), (320, 192, 2)])
def test_device_generator_and_layout_match_host(F, SG, hidden, inter, bits):
    assert F.expert_bytes(hidden, inter, bits) == O.expert_bytes(hidden, inter, bits)
    lay = O.blob_layout(hidden, inter, bits)
    assert F.blob_offsets(hidden, inter, bits) == [lay["gate"][0], lay["gate"][1], lay["up"][0], lay["up"][1],
                                                   lay["down"][0], lay["down"][1]]
    n = 3
    eb = F.expert_bytes(hidden, inter, bits)
    stride = (eb + 255) // 256 * 256
    buf = torch.zeros(n, stride, dtype=torch.uint8, device=dev())
    SG.fill_experts(buf, stride, F.blob_offsets(hidden, inter, bits), 5, n, hidden, inter, bits, 99, 2)
    got = buf.cpu().numpy()
    for e in range(n):
        want = C.cpu_blob(99, 2, 5 + e, hidden, inter, bits)
        assert np.array_equal(got[e, :eb], want), f"expert {5 + e}"


# ---------------------------------------------------------------------------
# Quantiser: bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hidden,inter,bits", [(512, 128, 4), (512, 128, 2), (4096, 1024, 4), (4096, 1024, 2),
                                               (320, 192, 4)])
def test_quantize_bit_exact(F, hidden, inter, bits):
    wg = S.dense_matrix(3, 1, inter, hidden)
    wu = S.dense_matrix(3, 2, inter, hidden)
    wd = S.dense_matrix(3, 3, hidden, inter)
    # add a constant group and an exactly-representable grid group
    wg[0, :64] = 0.25
    wd[1, 64:128] = np.arange(64, dtype=np.float32) % 4 * np.float32(2 ** -8) - np.float32(2 ** -6)
    blob = F.quantize_expert(*(torch.from_numpy(m).to(dev()) for m in (wg, wu, wd)), bits)
    want = O.quantize_expert(wg, wu, wd, bits)
    assert np.array_equal(blob.cpu().numpy(), want)


@pytest.mark.parametrize("bits", [4, 2])
def test_quantize_exact_half_quotients(F, bits):
    """Groups whose fp32 quotient is an exact half only after the fp32
    subtraction rounds (the hand-worked fixture of the oracle's pins): the
    device quantiser gives the fixture's codes, bit for bit."""
    from tests import oracle_pins as P
    (grp,) = [g for g in P.load_quantizer_ties() if g[0] == bits]
    row = np.array(grp[2], dtype=np.uint32).view(np.float32)
    H, I = 128, 64
    wg = S.dense_matrix(4, 1, I, H)
    wu = S.dense_matrix(4, 2, I, H)
    wd = S.dense_matrix(4, 3, H, I)
    wg[5, 64:128] = row  # gate row 5, group 1
    wd[7, 0:64] = row    # down row 7, group 0
    blob = F.quantize_expert(*(torch.from_numpy(m).to(dev()) for m in (wg, wu, wd)), bits)
    want = O.quantize_expert(wg, wu, wd, bits)
    got = blob.cpu().numpy()
    assert np.array_equal(got, want)
    parts = O.split_blob(got, H, I, bits)
    for name, r, g in (("gate", 5, 1), ("down", 7, 0)):
        codes, sb = parts[name]
        assert int(sb[r, g]) == grp[1]
        q = O.unpack_codes(codes, bits)[r, g * 64:(g + 1) * 64]
        assert q.tolist() == grp[3]


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("E,H,K,T", [(16, 512, 4, 1), (512, 4096, 4, 1), (512, 4096, 4, 16), (64, 320, 8, 5),
                                     (8, 256, 8, 3), (1024, 1024, 1, 2)])
def test_route(F, E, H, K, T):
    seed, layer = 21, 0
    wr = S.router_bf16(seed, layer, E, H)
    wsg = S.sgate_bf16(seed, layer, H)
    x = C.parity_x(seed, layer, 0, wr, min(K, E - 1) if E > K else K, H, T) if E > K else \
        S.token_x(seed, layer, 0, T, H)
    idx, w, sg, logits = F.route(torch.from_numpy(wr.view(np.int16)).to(dev()),
                                 torch.from_numpy(wsg.view(np.int16)).to(dev()), torch.from_numpy(x).to(dev()),
                                 K, want_logits=True)
    idx, w, sg, logits = idx.cpu().numpy(), w.cpu().numpy(), sg.cpu().numpy(), logits.cpu().numpy()
    for t in range(T):
        r = O.route(wr, wsg, x[t], K)
        if E > K:
            assert idx[t].tolist() == r["idx"].tolist()
        else:
            assert sorted(idx[t].tolist()) == list(range(E))
        order = [int(np.where(r["idx"] == e)[0][0]) for e in idx[t]]
        C.assert_close(w[t], r["w"][order], f"w token {t}", max_abs=1e-6, rel_l2=1e-6)
        assert abs(sg[t] - r["sg"]) <= 1e-6
        C.assert_close(logits[t], r["logits"], f"logits token {t}", max_abs=1e-4, rel_l2=1e-6)


# ---------------------------------------------------------------------------
# Single expert
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("hidden,inter,bits", [(512, 128, 4), (512, 128, 2), (4096, 1024, 4), (4096, 1024, 2),
                                               (320, 192, 4), (320, 192, 2), (64, 64, 4), (8192, 1024, 4),
                                               (1024, 4096, 2)])
def test_expert_forward(F, SG, hidden, inter, bits):
    eb = F.expert_bytes(hidden, inter, bits)
    buf = torch.zeros((eb + 255) // 256 * 256, dtype=torch.uint8, device=dev())
    SG.fill_experts(buf, eb, F.blob_offsets(hidden, inter, bits), 0, 1, hidden, inter, bits, 7, 0, 77)
    x = S.token_x(7, 0, 0, 1, hidden)[0]
    y = F.expert_forward(buf, hidden, inter, bits, torch.from_numpy(x).to(dev())).cpu().numpy()
    want = O.expert_forward(C.cpu_blob(7, 0, 77, hidden, inter, bits), hidden, inter, bits, x)
    C.assert_close(y, want, f"expert {hidden}x{inter} {bits}-bit")
    assert F.get_status() == 0


def test_expert_forward_extreme_inputs(F, SG):
    """Inputs spanning many binades (tiny, large, zeros) still match."""
    hidden, inter, bits = 512, 128, 4
    eb = F.expert_bytes(hidden, inter, bits)
    buf = torch.zeros(eb, dtype=torch.uint8, device=dev())
    SG.fill_experts(buf, eb, F.blob_offsets(hidden, inter, bits), 0, 1, hidden, inter, bits, 8, 0, 3)
    blob = C.cpu_blob(8, 0, 3, hidden, inter, bits)
    rng = np.random.default_rng(0)
    for scale in (1e-20, 1e-3, 1.0, 1e4, 1e12):
        x = (rng.standard_normal(hidden) * scale).astype(np.float32)
        x[::7] = 0.0
        x[3] *= 1e3
        y = F.expert_forward(buf, hidden, inter, bits, torch.from_numpy(x).to(dev())).cpu().numpy()
        want = O.expert_forward(blob, hidden, inter, bits, x)
        C.assert_close(y, want, f"scale {scale}", max_abs=max(2e-3, 1e-6 * np.abs(want).max()))


# ---------------------------------------------------------------------------
# Whole layer
# ---------------------------------------------------------------------------

def run_layer_case(F, SG, shape, seed=5, layer=0, n_steps=2, with_shared=True, with_sgate=True):
    L, t = make_gpu_layer(F, SG, seed, layer, shape, with_shared, with_sgate)
    wr = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    for step in range(n_steps):
        x = C.parity_x(seed, layer, step, wr, shape.top_k, shape.hidden)[0]
        # odd steps pass no residual, so `out` is the MoE contribution alone and
        # the relative check is not diluted by an O(1) residual
        res = S.token_residual(seed, layer, step, 1, shape.hidden)[0] if step % 2 == 0 else None
        idx = torch.empty(1, shape.top_k, dtype=torch.int32, device=dev())
        w = torch.empty(1, shape.top_k, dtype=torch.float32, device=dev())
        out = L.decode(torch.from_numpy(x).to(dev()), None if res is None else torch.from_numpy(res).to(dev()),
                       idx_out=idx, w_out=w)
        assert F.get_status() == 0
        r = C.oracle_layer(seed, layer, shape, x, np.zeros(shape.hidden) if res is None else res, with_shared,
                           with_sgate)
        assert idx.cpu().numpy()[0].tolist() == r["idx"].tolist()
        C.assert_close(w.cpu().numpy()[0], r["w"], "w", max_abs=1e-6, rel_l2=1e-6)
        C.assert_close(out.cpu().numpy()[0], r["out"], f"{shape.name} out step {step}")


def test_layer_tiny(F, SG):
    run_layer_case(F, SG, C.TINY, n_steps=4)


def test_layer_full_4bit(F, SG):
    run_layer_case(F, SG, C.FULL4, n_steps=2)


def test_layer_full_2bit_routed(F, SG):
    run_layer_case(F, SG, C.FULL2, n_steps=2)


@pytest.mark.parametrize("shape,with_shared,with_sgate", [
    (C.Shape("ragged_h320_i192_e24_k3", 320, 192, 24, 3, 4), True, True),
    (C.Shape("no_shared_h512_i128_e16_k4", 512, 128, 16, 4, 4), False, True),
    (C.Shape("ungated_h512_i128_e16_k2", 512, 128, 16, 2, 2, 2), True, False),
    (C.Shape("k1_h256_i64_e8", 256, 64, 8, 1, 4), True, True),
    (C.Shape("k8_h1024_i1024_e64", 1024, 1024, 64, 8, 4), True, True),
    (C.Shape("e1024_h2048_i256_k4", 2048, 256, 1024, 4, 4), True, True),
])
def test_layer_edge_shapes(F, SG, shape, with_shared, with_sgate):
    run_layer_case(F, SG, shape, n_steps=2, with_shared=with_shared, with_sgate=with_sgate)


def test_layer_all_experts_selected(F, SG):
    """K = E: every expert is used; weights are the full softmax."""
    shape = C.Shape("k_eq_e_h256_i64_e8", 256, 64, 8, 8, 4)
    L, t = make_gpu_layer(F, SG, 6, 0, shape)
    x = S.token_x(6, 0, 0, 1, 256)[0]
    res = S.token_residual(6, 0, 0, 1, 256)[0]
    out = L.decode(torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev()))
    r = C.oracle_layer(6, 0, shape, x, res)
    C.assert_close(out.cpu().numpy()[0], r["out"], "k=e")


def test_layer_multi_token(F, SG):
    shape = C.TINY
    L, t = make_gpu_layer(F, SG, 9, 1, shape)
    wr = S.router_bf16(9, 1, shape.n_experts, shape.hidden)
    T = 5
    x = C.parity_x(9, 1, 0, wr, shape.top_k, shape.hidden, T)
    res = S.token_residual(9, 1, 0, T, shape.hidden)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device=dev())
    out = L.decode(torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev()), idx_out=idx)
    for k in range(T):
        r = C.oracle_layer(9, 1, shape, x[k], res[k])
        assert idx.cpu().numpy()[k].tolist() == r["idx"].tolist()
        C.assert_close(out.cpu().numpy()[k], r["out"], f"token {k}")


def test_layer_deterministic(F, SG):
    L, t = make_gpu_layer(F, SG, 5, 0, C.FULL4)
    x = torch.from_numpy(S.token_x(5, 0, 3, 1, 4096)).to(dev())
    res = torch.from_numpy(S.token_residual(5, 0, 3, 1, 4096)).to(dev())
    a = L.decode(x, res).clone()
    b = L.decode(x, res).clone()
    assert torch.equal(a, b)
    assert F.get_status() == 0


def test_stacked_layers_graph(F, SG):
    """Layers chained as in a stacked decode (each layer's output is the next
    layer's input and residual), replayed from one CUDA graph; every layer is
    checked against the oracle on the input the engine actually gave it."""
    shape = C.FULL4
    seed, n_layers, n_steps = 11, 3, 2
    layers = [make_gpu_layer(F, SG, seed, l, shape)[0] for l in range(n_layers)]
    H, K = shape.hidden, shape.top_k
    x0 = torch.empty(H, dtype=torch.float32, device=dev())
    hs = torch.empty(n_layers, H, dtype=torch.float32, device=dev())
    idx = torch.empty(n_layers, K, dtype=torch.int32, device=dev())
    ws = [L.workspace(1) for L in layers]
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for L, w in zip(layers, ws):  # resolve the stream's device before capture
            L.decode(x0, x0, out=hs[0], ws=w)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            src = x0
            for l, L in enumerate(layers):
                L.decode(src, src, out=hs[l], idx_out=idx[l], ws=ws[l])
                src = hs[l]
    wr = [S.router_bf16(seed, l, shape.n_experts, H) for l in range(n_layers)]
    for step in range(n_steps):
        x0.copy_(torch.from_numpy(C.parity_x(seed, 0, step, wr[0], K, H)[0]))
        g.replay()
        torch.cuda.synchronize()
        assert F.get_status() == 0
        ins = [x0.cpu().numpy().astype(np.float64)] + [hs[l].cpu().numpy().astype(np.float64)
                                                         for l in range(n_layers - 1)]
        for l in range(n_layers):
            x = ins[l].astype(np.float32)
            r = C.oracle_layer(seed, l, shape, x, x)
            got = idx[l].cpu().numpy().tolist()
            lg = O.router_logits(wr[l], x)
            if O.top5_min_gap(lg, K) >= C.NEAR_TIE:
                assert got == r["idx"].tolist(), f"layer {l} step {step}"
            else:  # a near-tie: the selection must still be a valid top-K
                assert min(lg[got]) >= np.sort(lg)[-K] - C.NEAR_TIE
                continue
            out = hs[l].cpu().numpy()
            C.assert_close(out, r["out"], f"stacked layer {l} step {step}")
            ma, _ = C.errors(out.astype(np.float64) - x, r["out"] - x)
            assert ma <= C.MAX_ABS, f"layer {l} step {step}: MoE part max-abs {ma:.3e}"
    del g


@pytest.mark.parametrize("shape", [C.FULL4, C.TINY], ids=["full4", "tiny"])
def test_dependent_launch_matches_cooperative(F, SG, shape):
    """Back-to-back chained decodes of three layers that share ONE workspace
    (so each grid's counters are the previous grid's), run as programmatic
    dependent launches (eagerly and from a graph) and as cooperative launches:
    all outputs, indices and weights are bit-identical, and layer 0 agrees
    with the oracle."""
    seed, n_layers = 17, 3
    layers = [make_gpu_layer(F, SG, seed, l, shape)[0] for l in range(n_layers)]
    H, K = shape.hidden, shape.top_k
    ws = layers[0].workspace(1)
    x0 = torch.from_numpy(C.parity_x(seed, 0, 0, S.router_bf16(seed, 0, shape.n_experts, H), K, H)[0]).to(dev())

    def chain(hs, idx, w):
        src = x0
        for l, L in enumerate(layers):
            L.decode(src, src, out=hs[l], idx_out=idx[l], w_out=w[l], ws=ws)
            src = hs[l]

    def bufs():
        return (torch.full((n_layers, H), float("nan"), device=dev()),
                torch.full((n_layers, K), -1, dtype=torch.int32, device=dev()),
                torch.full((n_layers, K), float("nan"), device=dev()))

    runs = {}
    prev = F.set_dependent_launch(True)
    try:
        for mode in (True, False):
            F.set_dependent_launch(mode)
            eager = bufs()
            for _ in range(3):
                chain(*eager)
            assert F.get_status() == 0
            graphed = bufs()
            stream = torch.cuda.Stream()
            stream.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(stream):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    chain(*graphed)
                for _ in range(3):
                    g.replay()
            stream.synchronize()
            assert F.get_status() == 0
            del g
            runs[mode] = (eager, graphed)
    finally:
        F.set_dependent_launch(prev)
    ref = runs[False][0]
    for mode in (True, False):
        for got in runs[mode]:
            for a, b in zip(got, ref):
                assert torch.equal(a, b), f"dependent={mode}"
    r = C.oracle_layer(seed, 0, shape, x0.cpu().numpy(), x0.cpu().numpy())
    C.assert_close(ref[0][0].cpu().numpy(), r["out"], "chain layer 0")


def test_routing_epoch_wraps(F, SG):
    """The router logits and the activations are published as words tagged
    with the workspace's launch epoch + 1.  Started two launches before the
    epoch would pass 0x7FFFFFFE, three decodes must all be right: the second
    clears the tagged words and restarts the epoch at 0, so the third (tag 1)
    reads no stale word."""
    shape, seed = C.FULL4, 23
    L, _ = make_gpu_layer(F, SG, seed, 0, shape)
    H, K = shape.hidden, shape.top_k
    wr = S.router_bf16(seed, 0, shape.n_experts, H)
    xs = C.parity_x(seed, 0, 0, wr, K, H, 3)
    res = S.token_residual(seed, 0, 0, 3, H)
    ws = L.workspace(1)
    epoch = ws[:4].view(torch.int32)
    epoch.fill_(0x7FFFFFFD)
    expect_epoch = [0x7FFFFFFE, 0, 1]  # then the wrap to 0
    n_tagged = (1025 * 8 + 255) // 256 * 256 // 8 + 10240
    for i in range(3):
        idx = torch.empty(1, K, dtype=torch.int32, device=dev())
        out = L.decode(torch.from_numpy(xs[i]).to(dev()), torch.from_numpy(res[i]).to(dev()), idx_out=idx, ws=ws)
        assert F.get_status() == 0
        assert int(epoch.cpu()[0]) == expect_epoch[i], f"decode {i}"
        tags = ws[256:256 + n_tagged * 8].view(torch.int64).cpu().numpy()
        if i == 1:  # the wrap cleared every tagged word
            assert (tags == 0).all()
        else:  # this launch's words carry its tag
            assert ((tags >> 32) == expect_epoch[i]).sum() == shape.n_experts + 1 + (K + 1) * shape.inter
        r = C.oracle_layer(seed, 0, shape, xs[i], res[i])
        assert idx.cpu().numpy()[0].tolist() == r["idx"].tolist(), f"decode {i}"
        C.assert_close(out.cpu().numpy()[0], r["out"], f"decode {i} across the epoch wrap")


def test_workspace_shared_by_grouped_and_single_token(F, SG):
    """One workspace used in turn by single-token and grouped decodes of the
    layer: every single-token result equals the one from a fresh workspace
    (the grouped decode never writes the tagged router words)."""
    shape, seed, T = C.FULL4, 29, 16
    L, _ = make_gpu_layer(F, SG, seed, 0, shape)
    H = shape.hidden
    xs = torch.from_numpy(S.token_x(seed, 0, 0, T, H)).to(dev())
    res = torch.from_numpy(S.token_residual(seed, 0, 0, T, H)).to(dev())
    fresh = torch.zeros(L.workspace_bytes(1), dtype=torch.uint8, device=dev())
    want = [L.decode(xs[t], res[t], ws=fresh).clone() for t in range(3)]
    ws = torch.zeros(L.workspace_bytes(T), dtype=torch.uint8, device=dev())
    for t in range(3):
        L.decode(xs, res, ws=ws)
        assert torch.equal(L.decode(xs[t], res[t], ws=ws), want[t]), f"token {t}"
        assert F.get_status() == 0


# ---------------------------------------------------------------------------
# Grouped decode (T >= 2 tokens in one call)
# ---------------------------------------------------------------------------

def run_grouped_case(F, SG, shape, T, seed=31, layer=0, with_shared=True, with_sgate=True, identical=False,
                     residual=True):
    L, t = make_gpu_layer(F, SG, seed, layer, shape, with_shared, with_sgate)
    wr = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    x = C.parity_x(seed, layer, 0, wr, shape.top_k, shape.hidden, 1 if identical else T)
    if identical:
        x = np.repeat(x, T, axis=0)
    res = S.token_residual(seed, layer, 0, T, shape.hidden) if residual else np.zeros((T, shape.hidden), np.float32)
    if identical:
        res = np.repeat(res[:1], T, axis=0)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device=dev())
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device=dev())
    out = L.decode(torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev()) if residual else None,
                   idx_out=idx, w_out=w)
    assert F.get_status() == 0
    got = out.cpu().numpy()
    gi, gw = idx.cpu().numpy(), w.cpu().numpy()
    for k in range(T):
        if identical and k > 0:
            assert np.array_equal(got[k], got[0]) and np.array_equal(gi[k], gi[0])
            continue
        r = C.oracle_layer(seed, layer, shape, x[k], res[k], with_shared, with_sgate)
        assert gi[k].tolist() == r["idx"].tolist(), f"token {k}"
        C.assert_close(gw[k], r["w"], f"token {k} w", max_abs=1e-6, rel_l2=1e-6)
        C.assert_close(got[k], r["out"], f"{shape.name} T={T} token {k}")
    return L, x, res, got


def test_grouped_full_4bit_16_tokens(F, SG):
    # no residual: `out` is the layer's own contribution, so the relative
    # check is not diluted by an O(1) residual
    run_grouped_case(F, SG, C.FULL4, 16, residual=False)


def test_grouped_full_4bit_16_tokens_with_residual(F, SG):
    run_grouped_case(F, SG, C.FULL4, 16, seed=36)


def test_grouped_full_2bit_16_tokens(F, SG):
    run_grouped_case(F, SG, C.FULL2, 16, seed=32, residual=False)


def test_grouped_two_tokens_full(F, SG):
    run_grouped_case(F, SG, C.FULL4, 2, seed=33)


@pytest.mark.parametrize("shape,T,with_shared,with_sgate", [
    (C.Shape("shared_heavy_h512_i128_e8_k4", 512, 128, 8, 4, 4), 16, True, True),
    (C.Shape("ragged_h320_i192_e24_k3", 320, 192, 24, 3, 4), 7, True, True),
    (C.Shape("no_shared_h512_i128_e16_k4", 512, 128, 16, 4, 4), 16, False, True),
    (C.Shape("ungated_h512_i128_e16_k2_2bit", 512, 128, 16, 2, 2, 2), 9, True, False),
    (C.Shape("mixed_h1024_i256_e64_k8_r4_s2", 1024, 256, 64, 8, 4, 2), 16, True, True),
    (C.Shape("mixed_h1024_i256_e64_k1_r2_s4", 1024, 256, 64, 1, 2, 4), 3, True, True),
    (C.Shape("e1024_h2048_i256_k4", 2048, 256, 1024, 4, 4), 16, True, True),
    # H and I multiples of 512: the shared expert runs on the tensor cores
    (C.Shape("tc_h1024_i512_e64_k4", 1024, 512, 64, 4, 4), 16, True, True),
    (C.Shape("tc_h1024_i512_e32_k8_r2_s4", 1024, 512, 32, 8, 2, 4), 16, True, True),
    (C.Shape("tc_h2048_i512_e64_k2_r4_s2", 2048, 512, 64, 2, 4, 2), 5, True, True),
    (C.Shape("tc_ungated_h1024_i1024_e16_k4", 1024, 1024, 16, 4, 4), 3, True, False),
], ids=lambda v: v.name if isinstance(v, C.Shape) else str(v))
def test_grouped_edge_shapes(F, SG, shape, T, with_shared, with_sgate):
    run_grouped_case(F, SG, shape, T, with_shared=with_shared, with_sgate=with_sgate)


@pytest.mark.parametrize("shape", [C.Shape("identical_h1024_i256_e64_k4", 1024, 256, 64, 4, 4),
                                   C.Shape("identical_tc_h1024_i512_e64_k4", 1024, 512, 64, 4, 4)],
                         ids=lambda v: v.name)
def test_grouped_identical_tokens_share_every_expert(F, SG, shape):
    """All tokens equal: one slot per expert holding every token."""
    run_grouped_case(F, SG, shape, 16, identical=True)


def test_grouped_matches_single_token_calls(F, SG):
    """A batch gives each token the routing and (within the fp tolerance) the
    output of decoding that token alone."""
    L, x, res, got = run_grouped_case(F, SG, C.TINY, 12, seed=34)
    for k in range(12):
        idx = torch.empty(1, C.TINY.top_k, dtype=torch.int32, device=dev())
        one = L.decode(torch.from_numpy(x[k]).to(dev()), torch.from_numpy(res[k]).to(dev()), idx_out=idx)
        C.assert_close(got[k], one.cpu().numpy()[0], f"token {k} batch vs alone", max_abs=1e-5, rel_l2=1e-6)


def test_grouped_deterministic_and_graph_replay(F, SG):
    shape, T = C.FULL4, 16
    L, t = make_gpu_layer(F, SG, 35, 0, shape)
    x = torch.from_numpy(S.token_x(35, 0, 0, T, shape.hidden)).to(dev())
    res = torch.from_numpy(S.token_residual(35, 0, 0, T, shape.hidden)).to(dev())
    out = torch.empty(T, shape.hidden, dtype=torch.float32, device=dev())
    ws = L.workspace(T)
    a = L.decode(x, res, ws=ws).clone()
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        L.decode(x, res, out=out, ws=ws)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            L.decode(x, res, out=out, ws=ws)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(a, out)
    assert F.get_status() == 0
    del g


def test_grouped_dependent_and_plain_launches_agree(F, SG):
    """Two layers decoded back to back on 6 tokens (the second reads the
    first's output as input and residual) with one shared workspace, as
    programmatic dependent launches and as plain launches, eagerly and from
    a graph: outputs, indices and weights are bit-identical, and layer 0
    agrees with the oracle."""
    shape, T, seed = C.FULL4, 6, 37
    layers = [make_gpu_layer(F, SG, seed, l, shape)[0] for l in range(2)]
    H, K = shape.hidden, shape.top_k
    x = C.parity_x(seed, 0, 0, S.router_bf16(seed, 0, shape.n_experts, H), K, H, T)
    res = S.token_residual(seed, 0, 0, T, H)
    xd, rd = torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev())
    ws = layers[0].workspace(T)

    def chain(hs, idx, w):
        layers[0].decode(xd, rd, out=hs[0], idx_out=idx[0], w_out=w[0], ws=ws)
        layers[1].decode(hs[0], hs[0], out=hs[1], idx_out=idx[1], w_out=w[1], ws=ws)

    def bufs():
        return (torch.full((2, T, H), float("nan"), device=dev()),
                torch.full((2, T, K), -1, dtype=torch.int32, device=dev()),
                torch.full((2, T, K), float("nan"), device=dev()))

    runs = {}
    prev = F.set_dependent_launch(True)
    try:
        for mode in (True, False):
            F.set_dependent_launch(mode)
            eager = bufs()
            for _ in range(2):
                chain(*eager)
            torch.cuda.synchronize()
            assert F.get_status() == 0
            graphed = bufs()
            stream = torch.cuda.Stream()
            stream.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(stream):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    chain(*graphed)
                for _ in range(2):
                    g.replay()
            torch.cuda.synchronize()
            assert F.get_status() == 0
            del g
            runs[mode] = (eager, graphed)
    finally:
        F.set_dependent_launch(prev)
    ref = runs[True][0]
    for mode, (eager, graphed) in runs.items():
        for a, b in zip(ref, eager):
            assert torch.equal(a, b), f"dependent={mode} eager"
        for a, b in zip(ref, graphed):
            assert torch.equal(a, b), f"dependent={mode} graph"
    got, gi = ref[0][0].cpu().numpy(), ref[1][0].cpu().numpy()
    for k in range(T):
        r = C.oracle_layer(seed, 0, shape, x[k], res[k])
        assert gi[k].tolist() == r["idx"].tolist(), f"token {k}"
        C.assert_close(got[k], r["out"], f"token {k}")


@pytest.mark.parametrize("T", [1, 6])
def test_layer_exact_ties_pick_lowest_indices(F, SG, T):
    """Every router row equal: all logits tie exactly, and the decision is the
    K lowest expert indices with equal weights (single token and grouped)."""
    shape = C.Shape("ties_h512_i128_e40_k4", 512, 128, 40, 4, 4)
    seed, layer = 41, 0
    t = SG.make_layer(seed, layer, shape.hidden, shape.inter, shape.n_experts, shape.bits, shape.shared_bits,
                      F.blob_offsets, F.expert_bytes, dev())
    wr_host = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    wr_tied = np.repeat(wr_host[7:8], shape.n_experts, axis=0)
    w_router = t["w_router"].clone()
    w_router.copy_(torch.from_numpy(wr_tied.view(np.int16)).to(dev()))
    L = F.Layer(w_router, t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter, shape.top_k,
                shape.bits, shape.shared_bits)
    x = S.token_x(seed, layer, 0, T, shape.hidden)
    res = S.token_residual(seed, layer, 0, T, shape.hidden)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device=dev())
    w = torch.empty(T, shape.top_k, dtype=torch.float32, device=dev())
    out = L.decode(torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev()), idx_out=idx, w_out=w)
    assert F.get_status() == 0
    w_sg = S.sgate_bf16(seed, layer, shape.hidden)
    shared = C.cpu_blob(seed, layer, S.SHARED_EXPERT_ID, shape.hidden, shape.inter, shape.shared_bits)
    for k in range(T):
        assert idx.cpu().numpy()[k].tolist() == [0, 1, 2, 3]
        C.assert_close(w.cpu().numpy()[k], np.full(4, 0.25), "tied weights", max_abs=1e-7, rel_l2=1e-7)
        r = O.layer_decode(wr_tied, w_sg, lambda e: C.cpu_blob(seed, layer, e, shape.hidden, shape.inter, shape.bits),
                           shared, x[k], res[k], shape.top_k, shape.hidden, shape.inter, shape.bits, shape.shared_bits)
        assert r["idx"].tolist() == [0, 1, 2, 3]
        C.assert_close(out.cpu().numpy()[k], r["out"], f"tied token {k}")


# ---------------------------------------------------------------------------
# Input RMS norm (the next layer's norm fused into the layer start)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape,T", [(C.TINY, 1), (C.FULL4, 1), (C.FULL2, 1), (C.TINY, 7), (C.FULL4, 16),
                                     (C.Shape("norm_h1024_i256_e64_k4", 1024, 256, 64, 4, 4), 5)],
                         ids=lambda v: v.name if isinstance(v, C.Shape) else str(v))
def test_layer_input_norm(F, SG, shape, T):
    seed, layer, eps = 51, 2, 1e-5
    L0, t = make_gpu_layer(F, SG, seed, layer, shape)
    nw = S.norm_bf16(seed, layer, shape.hidden)
    L = F.Layer(t["w_router"], t["w_sgate"], t["experts"], t["shared"], shape.hidden, shape.inter, shape.top_k,
                shape.bits, shape.shared_bits, norm_weight=SG.bf16_tensor(nw, dev()), norm_eps=eps)
    wr = S.router_bf16(seed, layer, shape.n_experts, shape.hidden)
    # un-normalised inputs of different scales (the norm removes most of the
    # scale); the near-tie screen looks at what the router will see
    x = np.empty((T, shape.hidden), dtype=np.float32)
    for k in range(T):
        for redraw in range(1000):
            xk = S.token_x(seed, layer, k, 1, shape.hidden, redraw)[0] * np.float32(0.5 + k)
            if O.top5_min_gap(O.router_logits(wr, O.rms_norm(xk, nw, eps)), shape.top_k) >= C.NEAR_TIE:
                x[k] = xk
                break
    res = S.token_residual(seed, layer, 0, T, shape.hidden)
    idx = torch.empty(T, shape.top_k, dtype=torch.int32, device=dev())
    out = L.decode(torch.from_numpy(x).to(dev()), torch.from_numpy(res).to(dev()), idx_out=idx)
    assert F.get_status() == 0
    for k in range(T):
        r = C.oracle_layer(seed, layer, shape, x[k], res[k], norm_w=nw, norm_eps=eps)
        assert idx.cpu().numpy()[k].tolist() == r["idx"].tolist(), f"token {k}"
        C.assert_close(out.cpu().numpy()[k], r["out"], f"{shape.name} T={T} token {k} (input norm)")
